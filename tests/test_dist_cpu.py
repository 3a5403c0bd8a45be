"""The N > 1 host path of bench.py on CPU: world-size-2 gloo ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ms = 2.0 + 3.0 * rank                         # per-rank device time
    mx = bench.max_over_ranks(ms, world)
    bench.barrier(world)
    q.put((rank, mx, bench.aggregate_tokens_per_s(world, 131072, mx), bench.rank_seed(rank)))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_replicas_take_the_slowest_rank(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = 2.0 + 3.0 * (world - 1)
    assert all(r[1] == slowest for r in res)
    assert all(abs(r[2] - world * 131072 / (slowest / 1e3)) < 1e-6 for r in res)
    assert len({r[3] for r in res}) == world      # every replica works on its own sequence


def _cp_exchange_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from mamba_selective_scan_mixer_b200 import context_parallel as cp
    L = 5 + rank                                              # uneven slices
    u = torch.arange(2 * L * 4, dtype=torch.float32).reshape(2, L, 4) + 1000.0 * rank
    halo = cp.exchange_halo(u)
    carry = torch.full((2, 3, 16), float(rank))
    g = cp._all_gather(carry)
    q.put((rank, None if halo is None else halo.tolist(), g[:, 0, 0, 0].tolist(), u[:, -3:].tolist()))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_exchange(world):
    """The halo of rank r is rank r-1's last three rows; carries come back in rank order."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_exchange_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][1] is None
    for r in range(1, world):
        assert res[r][1] == res[r - 1][3]
    for r in range(world):
        assert res[r][2] == [float(j) for j in range(world)]


def _tp_reduce_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from mamba_selective_scan_mixer_b200 import tensor_parallel as tp
    t = torch.full((3, 5), float(rank + 1))
    tp._all_reduce(t)
    q.put((rank, t.tolist()))
    dist.destroy_process_group()


def test_tensor_parallel_all_reduce_sums_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 3
    procs = [ctx.Process(target=_tp_reduce_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, t in res:
        assert t == [[6.0] * 5] * 3


def test_tensor_parallel_shards_cover_the_channels():
    """The shards of every channel-indexed weight put back together are the
    original weights (in_proj: x rows, then z rows, of each shard)."""
    import torch
    from mamba_selective_scan_mixer_b200 import tensor_parallel as tp
    from synthetic import MambaShape, mamba_params
    sh = MambaShape(d_model=32, d_inner=64, dt_rank=8, dtype="f32")
    p = mamba_params(sh, seed=1, a_init="random", norm_init="random", d_init="random")
    world, k = 4, 16
    sh_ = [tp.shard_params(p, r, world) for r in range(world)]
    x = torch.cat([s["in_proj"][:k] for s in sh_])
    z = torch.cat([s["in_proj"][k:] for s in sh_])
    assert torch.equal(torch.cat([x, z]), p["in_proj"])
    for n in ("conv_w", "conv_b", "dt_proj", "dt_bias", "A", "D"):
        assert torch.equal(torch.cat([s[n] for s in sh_]), p[n])
    for n in ("x_proj", "out_proj"):
        assert torch.equal(torch.cat([s[n] for s in sh_], dim=1), p[n])
    for n in ("norm_dt", "norm_B", "norm_C"):
        assert all(torch.equal(s[n], p[n]) for s in sh_)


def test_expert_parallel_shards_cover_the_experts():
    import torch
    from mamba_selective_scan_mixer_b200 import expert_parallel as ep
    from synthetic import MoEShape, moe_params
    p = moe_params(MoEShape(d_model=16, d_ff=8, n_experts=16, top_k=2), seed=0)
    sh = [ep.shard_experts(p, r, 4) for r in range(4)]
    for n in ("w_gate", "w_up", "w_down"):
        assert torch.equal(torch.cat([s[n] for s in sh]), p[n])
    assert all(torch.equal(s["router"], p["router"]) for s in sh)
