"""Expert-parallel MoE (experts split over ranks) through the C ABI, against
the fp64 oracle MoE.

Each rank is a process of its own with a gloo process group and its own
tokens; the ranks share the one GPU of this machine, and the all-to-alls of
routed rows and results go through host memory between kernel launches, so
no kernel waits on another process.  On several GPUs the same code runs over
NCCL.
"""
import datetime
import json
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import mamba as om
from oracle import moe as omoe
from synthetic import MoEShape, moe_input, moe_params
from tests.helpers import TOL_BF16, cuda_or_skip, rel_l2, to_np

pytestmark = pytest.mark.gpu

FACTS = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, spec, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=300))
    import mamba_selective_scan_mixer_b200 as J
    from mamba_selective_scan_mixer_b200 import expert_parallel as ep
    dev = torch.device("cuda:0")
    es = MoEShape(d_model=spec["dm"], d_ff=spec["dff"], n_experts=FACTS["n_experts"], top_k=FACTS["top_k"])
    p = {k: v.to(dev) for k, v in moe_params(es, seed=spec["seed"]).items()}
    if spec["int8"]:
        p = J.quantize_experts_int8(p)
    moe = ep.ExpertParallelMoE(ep.shard_experts(p, rank, world), es)
    x = moe_input(es, spec["tokens"][rank], seed=spec["seed"] + 100 + rank).to(dev)
    res = moe_input(es, spec["tokens"][rank], seed=spec["seed"] + 200 + rank).to(dev)
    r = moe.forward(x, residual=res)
    torch.cuda.synchronize()
    J.device_status()
    torch.save({k: r[k].cpu() for k in ("out", "idx", "offsets", "perm")}, os.path.join(outdir, "rank%d.pt" % rank))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("spec", [
    dict(tokens=[300, 177], dm=512, dff=384, seed=1, int8=False),
    dict(tokens=[64, 64, 64, 64], dm=256, dff=256, seed=2, int8=False),   # 4 experts per rank, decode-sized
    dict(tokens=[200, 37], dm=512, dff=256, seed=3, int8=True),
])
def test_expert_parallel_moe_matches_oracle(spec):
    cuda_or_skip()
    world = len(spec["tokens"])
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank_main, args=(world, _free_port(), spec, d), nprocs=world, join=True,
                           start_method="spawn")
        parts = [torch.load(os.path.join(d, "rank%d.pt" % r)) for r in range(world)]
    es = MoEShape(d_model=spec["dm"], d_ff=spec["dff"], n_experts=FACTS["n_experts"], top_k=FACTS["top_k"])
    p = moe_params(es, seed=spec["seed"])
    p64 = {k: om.to64(v) for k, v in p.items()}
    if spec["int8"]:
        p64 = omoe.dequantized(omoe.experts_int8(p64))
    for r in range(world):
        x = moe_input(es, spec["tokens"][r], seed=spec["seed"] + 100 + r)
        res = moe_input(es, spec["tokens"][r], seed=spec["seed"] + 200 + r)
        want = omoe.moe_forward(p64, om.to64(x), es.top_k)
        np.testing.assert_array_equal(parts[r]["idx"].numpy(), want["idx"])
        np.testing.assert_array_equal(parts[r]["offsets"].numpy(), want["offsets"])
        np.testing.assert_array_equal(parts[r]["perm"].numpy(), want["perm"])
        assert rel_l2(to_np(parts[r]["out"]), want["out"] + om.to64(res)) < TOL_BF16
