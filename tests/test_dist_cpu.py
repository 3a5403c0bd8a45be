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
