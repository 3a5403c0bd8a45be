"""Context-parallel prefill (sequences split over ranks by time) through the
C ABI, against the fp64 oracle and the one-process prefill.

Each rank is a process of its own with a gloo process group: the ranks share
the one GPU of this machine, and the exchanges between them (the 3-row conv
halo and the (P, h) carries) go through host memory between kernel
launches, so no kernel ever waits on another process.  On several GPUs the
same code runs over NCCL.
"""
import datetime
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import mamba as om
from synthetic import MambaShape, mamba_input, mamba_params
from tests.helpers import TOL_BF16, cuda_or_skip, rel_l2, to_np

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _case(spec):
    sh = MambaShape(d_model=256, d_inner=512, dt_rank=32, dtype="bf16", inner_norm=True)
    p = mamba_params(sh, seed=spec["seed"], a_init=spec["a_init"])
    u = mamba_input(sh, spec["batch"], sum(spec["lens"]), seed=spec["seed"])
    g = torch.Generator().manual_seed(spec["seed"] + 1)
    res = mamba_input(sh, spec["batch"], sum(spec["lens"]), seed=spec["seed"] + 2) if spec["residual"] else None
    cs0 = ss0 = None
    if spec["states"]:
        cs0 = torch.randn(spec["batch"], sh.d_inner, 3, generator=g).to(torch.bfloat16).float()
        ss0 = torch.randn(spec["batch"], sh.d_inner, 16, generator=g)
    return sh, p, u, res, cs0, ss0


def _rank_main(rank, world, port, spec, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=300))
    import mamba_selective_scan_mixer_b200 as J
    from mamba_selective_scan_mixer_b200 import context_parallel as cp
    dev = torch.device("cuda:0")
    sh, p, u, res, cs0, ss0 = _case(spec)
    t0 = sum(spec["lens"][:rank])
    t1 = t0 + spec["lens"][rank]
    mix = J.MambaMixer({k: v.to(dev) for k, v in p.items()}, sh)
    ul = u[:, t0:t1].contiguous().to(dev)
    rl = None if res is None else res[:, t0:t1].contiguous().to(dev)
    out, cs, ss = cp.prefill_cp(mix, ul, residual=rl, conv_state_in=None if cs0 is None else cs0.to(dev),
                                ssm_state_in=None if ss0 is None else ss0.to(dev))
    torch.cuda.synchronize()
    J.device_status()
    torch.save({"out": out.cpu(), "cs": cs.cpu(), "ss": ss.cpu()}, os.path.join(outdir, "rank%d.pt" % rank))
    dist.barrier()
    dist.destroy_process_group()


def _run(spec):
    world = len(spec["lens"])
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank_main, args=(world, _free_port(), spec, d), nprocs=world, join=True,
                           start_method="spawn")
        parts = [torch.load(os.path.join(d, "rank%d.pt" % r)) for r in range(world)]
    out = torch.cat([q["out"] for q in parts], dim=1)
    return out, parts[-1]["cs"], parts[-1]["ss"], parts


@pytest.mark.parametrize("spec", [
    # uneven slices, caches before the first slice, residual, per-channel dt carried across slices
    dict(lens=[100, 37, 163], batch=2, seed=3, a_init="structured", residual=True, states=True),
    dict(lens=[300, 300], batch=1, seed=4, a_init="random", residual=False, states=False),
])
def test_context_parallel_prefill_matches_oracle(spec):
    cuda_or_skip()
    sh, p, u, res, cs0, ss0 = _case(spec)
    out, cs, ss, _ = _run(spec)
    ref = om.mamba_prefill(om.params64(p), to_np(u), sh, conv_state0=None if cs0 is None else to_np(cs0),
                           ssm_state0=None if ss0 is None else to_np(ss0))
    want = ref["out"] + (0 if res is None else to_np(res))
    assert rel_l2(to_np(out), want) < TOL_BF16
    assert rel_l2(to_np(ss), ref["ssm_state"]) < TOL_BF16
    assert rel_l2(to_np(cs), ref["conv_state"]) < TOL_BF16
    # the carries matter here: without them the later slices are wrong
    import mamba_selective_scan_mixer_b200 as J
    dev = torch.device("cuda:0")
    mix = J.MambaMixer({k: v.to(dev) for k, v in p.items()}, sh)
    t0 = spec["lens"][0]
    alone, _, _ = mix.prefill(u[:, t0:].contiguous().to(dev))
    assert rel_l2(to_np(alone), ref["out"][:, t0:]) > 10 * TOL_BF16


@pytest.mark.slow
def test_context_parallel_prefill_128k_four_ranks():
    """131072 tokens over 4 ranks of 32768 against the oracle (C scan) and the one-process prefill."""
    cuda_or_skip()
    spec = dict(lens=[32768] * 4, batch=1, seed=7, a_init="structured", residual=False, states=False)
    sh, p, u, _, _, _ = _case(spec)
    out, cs, ss, _ = _run(spec)
    ref = om.mamba_prefill(om.params64(p), to_np(u), sh, scan="c")
    assert rel_l2(to_np(out), ref["out"]) < TOL_BF16
    assert rel_l2(to_np(ss), ref["ssm_state"]) < TOL_BF16
    assert rel_l2(to_np(cs), ref["conv_state"]) < TOL_BF16
    import mamba_selective_scan_mixer_b200 as J
    dev = torch.device("cuda:0")
    mix = J.MambaMixer({k: v.to(dev) for k, v in p.items()}, sh)
    one, _, ss1 = mix.prefill(u.to(dev))
    assert rel_l2(to_np(out), to_np(one)) < TOL_BF16
    assert rel_l2(to_np(ss), to_np(ss1)) < 1e-4
