"""Host-side logic of the library that needs no GPU: the planner that gives
each channel group of the bf16 prefill's scan its own number of time chunks
(through the test entry jamba_test_scan_plan), the k-split choices of the
decode-size GEMMs (jamba_test_gemm_splits) and the time chunks of the
host-memory prefill (jamba_test_host_chunks).

A CTA of the scan costs its chunk plus the head it replays: the steps until
its slowest channel has lost the incoming state, at most the chunk.  The
planner minimises the largest CTA cost with at most `slots` CTAs in the
launch; these tests check the plan's shape, that it fits, that slower
groups never get fewer chunks, that no group could drop a chunk without
exceeding the plan's largest cost, and (on small cases) that no other chunk
assignment has a smaller largest cost."""
import ctypes
import itertools

import numpy as np
import pytest


@pytest.fixture(scope="module")
def lib():
    from mamba_selective_scan_mixer_b200 import build, _abi
    build.build()
    return _abi.lib()


def _plan(lib, batch, L, heads, slots):
    g = len(heads)
    h = (ctypes.c_float * g)(*heads)
    chunks = (ctypes.c_int * g)()
    lens = (ctypes.c_int * g)()
    n = ctypes.c_int(-1)
    assert lib.jamba_test_scan_plan(batch, L, g, h, slots, chunks, lens, ctypes.byref(n)) == 0
    return n.value, list(chunks)[:n.value], list(lens)[:n.value]


def _len(L, n):
    return (-(-L // n) + 15) // 16 * 16


def _cost(L, n, head):
    ln = _len(L, n)
    return ln + min(head, ln)


def _check(L, batch, heads, slots, n, chunks, lens):
    assert n == len(heads)
    for c, ln in zip(chunks, lens):
        assert c >= 1 and ln % 16 == 0
        assert (c - 1) * ln < L <= c * ln
    assert sum(chunks) * batch <= slots
    assert all(a >= b for a, b in zip(chunks, chunks[1:]))   # heads sorted slowest first
    worst = max(ln + min(h, ln) for h, ln in zip(heads, lens))
    for c, h in zip(chunks, heads):
        if c > 1:
            assert _cost(L, c - 1, h) > worst
    return worst


def test_plan_at_jamba_width_128k(lib):
    """32 groups of 256 channels, 131072 steps, 444 CTA slots (three per SM),
    heads from 20000 down to 200 steps"""
    heads = list(np.geomspace(20000.0, 200.0, 32))
    n, chunks, lens = _plan(lib, 1, 131072, heads, 444)
    worst = _check(131072, 1, heads, 444, n, chunks, lens)
    assert chunks[0] > chunks[-1]                     # slow groups get shorter chunks
    assert worst < 2 * 131072 * 32 / 444              # well under replaying every chunk in full


def test_plan_is_optimal_on_small_cases(lib):
    """every assignment of 1..8 chunks to 3 groups: none has a smaller largest
    cost within the slots than the plan"""
    for L, heads, slots in ((1200, [900.0, 300.0, 40.0], 9), (2048, [5000.0, 5000.0, 10.0], 8),
                            (4000, [700.0, 350.0, 350.0], 12)):
        n, chunks, lens = _plan(lib, 1, L, heads, slots)
        worst = _check(L, 1, heads, slots, n, chunks, lens)
        best = min(max(_cost(L, c, h) for c, h in zip(cs, heads))
                   for cs in itertools.product(range(1, 9), repeat=3) if sum(cs) <= slots)
        assert worst <= best + 1, (L, chunks, worst, best)


def test_plan_batch_rows_share_the_slots(lib):
    heads = [3000.0, 1000.0, 100.0, 50.0]
    n, chunks, lens = _plan(lib, 3, 20000, heads, 120)
    _check(20000, 3, heads, 120, n, chunks, lens)


def test_plan_falls_back_to_uniform_chunks(lib):
    heads = [100.0] * 32
    assert _plan(lib, 1, 16, heads, 444)[0] == 0          # too short to split
    assert _plan(lib, 8, 131072, heads, 444)[0] == 0      # batch rows and groups already fill the slots


def test_plan_rejects_bad_arguments(lib):
    h = (ctypes.c_float * 65)(*([1.0] * 65))
    c = (ctypes.c_int * 65)()
    n = ctypes.c_int()
    assert lib.jamba_test_scan_plan(1, 1000, 65, h, 444, c, c, ctypes.byref(n)) == 1   # more than 64 groups
    assert lib.jamba_test_scan_plan(1, 1000, 4, None, 444, c, c, ctypes.byref(n)) == 1


def _splits(lib, M, N, K, bn, min_k, groups=1):
    s, s8 = ctypes.c_int(), ctypes.c_int()
    assert lib.jamba_test_gemm_splits(M, N, K, bn, min_k, groups, ctypes.byref(s), ctypes.byref(s8)) == 0
    return s.value, s8.value


def test_k_splits_fill_one_wave(lib):
    """x_proj and out_proj at decode sizes: tiles x splits stay within one wave
    of the 148 SMs, every split keeps its minimum of 64-deep steps, and a GEMM
    whose tiles already fill the SMs is not split"""
    sms = 148
    for M, N, K, bn, mk in ((288, 64, 8192, 64, 4), (4096, 64, 8192, 64, 8), (131072, 288, 8192, 144, 8),
                            (288, 1, 2048, 64, 4), (4096, 65, 1024, 64, 8), (128, 64, 64, 64, 4)):
        s, _ = _splits(lib, M, N, K, bn, mk)
        tiles = -(-M // 128) * -(-N // bn)
        k_tiles = -(-K // 64)
        assert 1 <= s <= 32
        if tiles >= sms:
            assert s == 1
        else:
            assert tiles * s <= sms
            per = -(-k_tiles // s)
            assert (s - 1) * per < k_tiles          # no empty split
            assert s == 1 or per >= mk
    assert _splits(lib, 4096, 64, 8192, 64, 8)[0] == 4   # decode out_proj: 32 weight tiles x 4


def test_int8_k_splits(lib):
    """ExpertsInt8 fp32 expert GEMM at decode batches: 1 to 4 splits of an even
    number of 64-deep steps; none when the experts hold many rows"""
    for M, groups, N, K in ((128, 16, 4096, 14336), (64, 16, 4096, 14336), (16, 16, 4096, 14336)):
        _, s8 = _splits(lib, M, N, K, 64, 4, groups)
        assert 1 <= s8 <= 4 and (K // 64) % (2 * s8) == 0
    assert _splits(lib, 32768, 4096, 14336, 64, 4, 16)[1] == 1


def _chunks(lib, seqlen, chunk):
    buf = (ctypes.c_int * 4096)()
    n = ctypes.c_int()
    assert lib.jamba_test_host_chunks(seqlen, chunk, buf, 4096, ctypes.byref(n)) == 0
    return list(buf)[:n.value]


def test_host_prefill_chunks(lib):
    """the host-memory prefill's time chunks cover the sequence exactly, none
    longer than the chunk; from four chunks on, the first two and last two
    ramp (chunk/4, chunk/2) so the unoverlapped first copy-in and last
    copy-out are short"""
    assert _chunks(lib, 131072, 16384) == [4096, 8192] + [16384] * 6 + [8192, 8192, 4096]
    for seqlen, chunk in ((200, 48), (300, 64), (4200, 1024), (131072, 16384), (100, 1000), (65, 64), (1, 16384)):
        lens = _chunks(lib, seqlen, chunk)
        c = min(chunk, seqlen)
        assert sum(lens) == seqlen and all(1 <= n <= c for n in lens)
        if seqlen >= 4 * c and c >= 64:
            assert lens[:2] == [c // 4, c // 2] and lens[-2:] == [c // 2, c // 4]
        else:
            assert lens[:-1] == [c] * (len(lens) - 1)
    buf = (ctypes.c_int * 2)()
    n = ctypes.c_int()
    assert lib.jamba_test_host_chunks(1000, 10, buf, 2, ctypes.byref(n)) == 1 and n.value == 100
