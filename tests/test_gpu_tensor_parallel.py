"""Tensor-parallel prefill (d_inner split over ranks) through the C ABI,
against the fp64 oracle of the whole layer.

Each rank is a process of its own with a gloo process group; the ranks share
the one GPU of this machine, and the two all-reduces (the x_proj partial sums
and the out_proj partial sums) go through host memory between kernel
launches, so no kernel waits on another process.  On several GPUs the same
code runs over NCCL.
"""
import datetime
import os
import socket
import tempfile

import pytest
import torch
import torch.multiprocessing as mp

from oracle import mamba as om
from synthetic import MambaShape, mamba_input, mamba_params
from tests.helpers import TOL_BF16, TOL_F32, cuda_or_skip, rel_l2, to_np

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _case(spec):
    sh = MambaShape(d_model=spec["dm"], d_inner=spec["di"], dt_rank=spec["R"], dtype=spec["dtype"],
                    inner_norm=spec["norm"])
    p = mamba_params(sh, seed=spec["seed"], a_init=spec["a_init"], norm_init="random")
    u = mamba_input(sh, spec["batch"], spec["L"], seed=spec["seed"])
    res = mamba_input(sh, spec["batch"], spec["L"], seed=spec["seed"] + 1)
    g = torch.Generator().manual_seed(spec["seed"] + 2)
    cs0 = torch.randn(spec["batch"], sh.d_inner, 3, generator=g)
    if spec["dtype"] == "bf16":
        cs0 = cs0.to(torch.bfloat16).float()
    ss0 = torch.randn(spec["batch"], sh.d_inner, 16, generator=g)
    return sh, p, u, res, cs0, ss0


def _rank_main(rank, world, port, spec, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=300))
    import mamba_selective_scan_mixer_b200 as J
    from mamba_selective_scan_mixer_b200 import tensor_parallel as tp
    dev = torch.device("cuda:0")
    sh, p, u, res, cs0, ss0 = _case(spec)
    k = sh.d_inner // world
    c0, c1 = rank * k, (rank + 1) * k
    mix = J.MambaMixer({n: v.to(dev) for n, v in tp.shard_params(p, rank, world).items()},
                       sh.with_(d_inner=k))
    out, cs, ss = tp.prefill_tp(mix, u.to(dev), residual=res.to(dev),
                                conv_state_in=cs0[:, c0:c1].contiguous().to(dev),
                                ssm_state_in=ss0[:, c0:c1].contiguous().to(dev))
    torch.cuda.synchronize()
    J.device_status()
    torch.save({"out": out.cpu(), "cs": cs.cpu(), "ss": ss.cpu()}, os.path.join(outdir, "rank%d.pt" % rank))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("spec", [
    dict(world=2, dm=256, di=512, R=32, dtype="bf16", norm=True, batch=2, L=300, seed=5, a_init="structured"),
    dict(world=4, dm=256, di=1024, R=32, dtype="bf16", norm=True, batch=1, L=700, seed=6, a_init="random"),
    dict(world=2, dm=64, di=128, R=4, dtype="f32", norm=False, batch=1, L=256, seed=7, a_init="structured"),
])
def test_tensor_parallel_prefill_matches_oracle(spec):
    cuda_or_skip()
    world = spec["world"]
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank_main, args=(world, _free_port(), spec, d), nprocs=world, join=True,
                           start_method="spawn")
        parts = [torch.load(os.path.join(d, "rank%d.pt" % r)) for r in range(world)]
    sh, p, u, res, cs0, ss0 = _case(spec)
    ref = om.mamba_prefill(om.params64(p), to_np(u), sh, conv_state0=to_np(cs0), ssm_state0=to_np(ss0))
    tol = TOL_BF16 if spec["dtype"] == "bf16" else TOL_F32
    for r in range(world):   # the all-reduced output is the same on every rank
        assert rel_l2(to_np(parts[r]["out"]), ref["out"] + to_np(res)) < tol
    ss = torch.cat([q["ss"] for q in parts], dim=1)
    cs = torch.cat([q["cs"] for q in parts], dim=1)
    assert rel_l2(to_np(ss), ref["ssm_state"]) < tol
    assert rel_l2(to_np(cs), ref["conv_state"]) < tol
