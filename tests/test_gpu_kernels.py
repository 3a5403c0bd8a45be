"""Per-kernel parity: each CUDA kernel, called through the C ABI, against the
fp64 oracle on the same seeded inputs.  Sizes span several tiles and end on
ragged tails."""
import numpy as np
import pytest
import torch

from oracle import mamba as om
from synthetic import scan_inputs
from tests.helpers import TOL_BF16, TOL_F32, bf16_steps, cuda_or_skip, rel_l2, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    d = cuda_or_skip()
    import mamba_selective_scan_mixer_b200 as J
    J.lib()
    return d


def _gen(seed):
    g = torch.Generator()
    g.manual_seed(seed)
    return g


# ------------------------------------------------------------------ GEMM

@pytest.mark.parametrize("m,n,k", [(128, 256, 64), (300, 520, 264), (1, 72, 8), (513, 288, 1032),
                                   (2048, 1024, 4096), (77, 144, 200)])
def test_gemm_bf16_tensor_cores(dev, m, n, k):
    import mamba_selective_scan_mixer_b200 as J
    g = _gen(m * 7 + n)
    a = torch.randn(m, k, generator=g).to(torch.bfloat16)
    b = torch.randn(n, k, generator=g).to(torch.bfloat16)
    want = om.linear(to_np(a), to_np(b))
    got32 = J.gemm(a.to(dev), b.to(dev), out_dtype=torch.float32)
    assert rel_l2(to_np(got32), want) < 1e-5
    got16 = J.gemm(a.to(dev), b.to(dev))
    assert rel_l2(to_np(got16), want) < TOL_BF16
    # every element, not only the norm: bf16 rounding of an fp32-exact value
    np.testing.assert_allclose(to_np(got16), want, rtol=2 ** -7, atol=1e-3 * np.abs(want).max())


def test_gemm_bf16_residual(dev):
    import mamba_selective_scan_mixer_b200 as J
    g = _gen(3)
    a = torch.randn(260, 512, generator=g).to(torch.bfloat16)
    b = torch.randn(384, 512, generator=g).to(torch.bfloat16)
    r = torch.randn(260, 384, generator=g).to(torch.bfloat16)
    want = om.linear(to_np(a), to_np(b)) + to_np(r)
    got = J.gemm(a.to(dev), b.to(dev), residual=r.to(dev))
    assert rel_l2(to_np(got), want) < TOL_BF16


@pytest.mark.parametrize("m,n,k", [(1, 64, 64), (257, 130, 70)])
def test_gemm_f32_cuda_cores(dev, m, n, k):
    import mamba_selective_scan_mixer_b200 as J
    g = _gen(m + n + k)
    a = torch.randn(m, k, generator=g)
    b = torch.randn(n, k, generator=g)
    got = J.gemm(a.to(dev), b.to(dev))
    assert rel_l2(to_np(got), om.linear(to_np(a), to_np(b))) < TOL_F32


# ------------------------------------------------------------------ conv

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("L,with_state", [(1, True), (2, False), (130, True), (300, False)])
def test_conv_prefill(dev, dtype, L, with_state):
    import mamba_selective_scan_mixer_b200 as J
    g = _gen(L)
    B, C = 2, 136
    xz = torch.randn(B, L, 2 * C, generator=g).to(dtype)   # x is the first half of each row
    w = (0.5 * torch.randn(C, 4, generator=g)).to(dtype)
    b = (0.5 * torch.randn(C, generator=g)).to(dtype)
    st = torch.randn(B, C, 3, generator=g).to(dtype).float() if with_state else None
    out, st_out = J.causal_conv1d(xz.to(dev)[..., :C], w.to(dev), b.to(dev),
                                  None if st is None else st.to(dev))
    pre, want_st = om.causal_conv1d(to_np(xz)[..., :C], to_np(w), to_np(b), None if st is None else to_np(st))
    tol = TOL_BF16 if dtype == torch.bfloat16 else TOL_F32
    assert rel_l2(to_np(out), om.silu(pre)) < tol
    np.testing.assert_array_equal(to_np(st_out), want_st)   # cached inputs are copied exactly


@pytest.mark.parametrize("batch,L,di", [(3, 37, 256), (1, 3, 128), (2, 100, 384), (5, 7, 256), (1, 300, 256)])
def test_in_proj_conv1d(dev, batch, L, di):
    """in_proj with the conv in its epilogue: against the oracle (x|z
    projection, conv over the bf16 x, caches), row by row for the conv output
    (rows 0-2 of each 32-row slab are finished by a second kernel; short
    sequences put their starts at every lane), and bit for bit against
    jamba_gemm followed by jamba_causal_conv1d, which round and add in the
    same order.  The cache in holds arbitrary fp32 values."""
    import mamba_selective_scan_mixer_b200 as J
    g = _gen(1000 + L)
    dm = 256
    u = torch.randn(batch, L, dm, generator=g).to(torch.bfloat16)
    w_in = (0.05 * torch.randn(2 * di, dm, generator=g)).to(torch.bfloat16)
    w = (0.5 * torch.randn(di, 4, generator=g)).to(torch.bfloat16)
    b = (0.5 * torch.randn(di, generator=g)).to(torch.bfloat16)
    st = torch.randn(batch, di, 3, generator=g)
    st_out = torch.empty(batch, di, 3, device=dev)
    xc, xz, _ = J.in_proj_conv1d(u.to(dev), w_in.to(dev), w.to(dev), b.to(dev), state_in=st.to(dev),
                                 state_out=st_out)
    xz64 = to_np(u) @ to_np(w_in).T
    pre, want_st = om.causal_conv1d(xz64[..., :di], to_np(w), to_np(b), to_np(st))
    want = om.silu(pre)
    got = to_np(xc)
    assert rel_l2(got, want) < TOL_BF16
    row_err = (np.linalg.norm(got - want, axis=2) / np.linalg.norm(want, axis=2)).ravel()
    assert row_err.max() < 2e-2, (int(row_err.argmax()), float(row_err.max()))
    assert rel_l2(to_np(xz)[..., di:], xz64[..., di:]) < TOL_BF16
    assert rel_l2(to_np(st_out), want_st) < TOL_BF16
    # the unfused path on the same device: identical bits
    xz2 = J.gemm(u.to(dev).view(batch * L, dm), w_in.to(dev)).view(batch, L, 2 * di)
    xc2, st2 = J.causal_conv1d(xz2[..., :di], w.to(dev), b.to(dev), st.to(dev))
    assert torch.equal(xc, xc2)
    assert torch.equal(xz[..., di:], xz2[..., di:])
    assert torch.equal(st_out, st2)


def test_in_proj_conv1d_refuses_short_or_narrow(dev):
    import mamba_selective_scan_mixer_b200 as J
    from mamba_selective_scan_mixer_b200 import _abi
    for L, di in ((2, 256), (40, 96), (40, 272)):
        u = torch.zeros(1, L, 64, dtype=torch.bfloat16, device=dev)
        w_in = torch.zeros(2 * di, 64, dtype=torch.bfloat16, device=dev)
        w = torch.zeros(di, 4, dtype=torch.bfloat16, device=dev)
        b = torch.zeros(di, dtype=torch.bfloat16, device=dev)
        with pytest.raises(_abi.JambaError) as e:
            J.in_proj_conv1d(u, w_in, w, b)
        assert e.value.status == 2   # JAMBA_ERR_UNSUPPORTED


# ------------------------------------------------------------------ scan

def _scan_case(dev, batch, L, di, seed, dtype="bf16", bc="bf16", a_init="structured", h0=False, chunk=0,
               dt_mean=-4.0):
    import mamba_selective_scan_mixer_b200 as J
    s = scan_inputs(batch, L, di, 16, seed=seed, dtype=dtype, a_init=a_init, dt_mean=dt_mean)
    if bc != dtype:
        s["B"], s["C"] = s["B"].float(), s["C"].float()
    g = _gen(seed + 1)
    hin = torch.randn(batch, di, 16, generator=g) if h0 else None
    args = {k: v.to(dev) for k, v in s.items()}
    y, h = J.selective_scan(args["x"], args["z"], args["dt"], args["B"], args["C"], args["A"], args["D"],
                            None if hin is None else hin.to(dev), chunk=chunk)
    want_y, want_h = om.selective_scan_c(to_np(s["x"]), to_np(s["dt"]), to_np(s["A"]), to_np(s["B"]),
                                         to_np(s["C"]), to_np(s["D"]), to_np(s["z"]),
                                         None if hin is None else to_np(hin))
    return to_np(y), to_np(h), want_y, want_h


@pytest.mark.parametrize("batch,L,di,chunk", [(1, 64, 256, 16), (2, 300, 272, 64), (1, 1000, 512, 0),
                                              (3, 17, 8, 16), (1, 4096, 256, 256)])
def test_scan_bf16(dev, batch, L, di, chunk):
    y, h, wy, wh = _scan_case(dev, batch, L, di, seed=L + di, chunk=chunk)
    assert rel_l2(y, wy) < TOL_BF16
    assert rel_l2(h, wh) < 1e-5


@pytest.mark.parametrize("a_init", ["structured", "random"])
@pytest.mark.parametrize("h0", [False, True])
def test_scan_f32(dev, a_init, h0):
    y, h, wy, wh = _scan_case(dev, 2, 333, 264, seed=5, dtype="f32", bc="f32", a_init=a_init, h0=h0, chunk=48)
    assert rel_l2(y, wy) < TOL_F32
    assert rel_l2(h, wh) < TOL_F32


def test_scan_bf16_x_fp32_bc_random_A(dev):
    y, h, wy, wh = _scan_case(dev, 1, 700, 520, seed=9, dtype="bf16", bc="f32", a_init="random", h0=True,
                              chunk=64)
    assert rel_l2(y, wy) < TOL_BF16
    assert rel_l2(h, wh) < 1e-5


def test_scan_long_memory_never_decays(dev):
    """tiny dt: the carried state never underflows, every chunk takes the buffered path"""
    y, h, wy, wh = _scan_case(dev, 1, 2048, 256, seed=11, dtype="f32", bc="f32", chunk=64, dt_mean=-9.0)
    assert rel_l2(y, wy) < TOL_F32
    assert rel_l2(h, wh) < TOL_F32


@pytest.mark.parametrize("chunk", [16, 32, 112])
def test_scan_chunk_invariance(dev, chunk):
    """the same inputs under different chunkings agree with each other and the oracle"""
    y1, h1, wy, wh = _scan_case(dev, 1, 500, 256, seed=13, dtype="f32", bc="f32", chunk=chunk)
    y2, h2, _, _ = _scan_case(dev, 1, 500, 256, seed=13, dtype="f32", bc="f32", chunk=496)
    assert rel_l2(y1, y2) < 1e-6 and rel_l2(h1, h2) < 1e-6
    assert rel_l2(y1, wy) < TOL_F32


def _bf16_elementwise_bad(got, want):
    """Elements further from the exact value than one bf16 step (2^-7
    relative) plus an fp32-accumulation allowance: a correct fp32 scan
    rounded to bf16 has none."""
    scale = np.sqrt(np.mean(want ** 2))
    return int((np.abs(got - want) > 2.0 ** -7 * np.abs(want) + 1e-5 * scale).sum())


@pytest.mark.parametrize("dt_kind", ["iid", "per_channel"])
@pytest.mark.parametrize("chunk", [0, 512, 2048])
def test_scan_bf16_elementwise_many_chunks(dev, dt_kind, chunk):
    """Every sampled output within one bf16 step of the exact scan, over many
    chunks (several waves of CTAs at chunk 512) and both dt regimes: i.i.d.
    per step (short carried-state heads) and fixed per channel, log-uniform
    in [1e-3, 1e-1] as the dt_bias initialisation gives (heads as long as a
    chunk)."""
    import mamba_selective_scan_mixer_b200 as J
    L, di = 32768, 2048
    s = scan_inputs(1, L, di, 16, seed=31)
    if dt_kind == "per_channel":
        g = _gen(32)
        dt0 = torch.exp(torch.empty(di).uniform_(np.log(1e-3), np.log(1e-1), generator=g))
        s["dt"] = (dt0[None, None, :] * torch.exp(0.3 * torch.randn(1, L, di, generator=g))).float()
    args = {k: v.to(dev) for k, v in s.items()}
    y, h = J.selective_scan(args["x"], args["z"], args["dt"], args["B"], args["C"], args["A"], args["D"],
                            chunk=chunk)
    cols = np.arange(5, di, 37)   # a few channels of every warp of every CTA
    n = lambda k: to_np(s[k])
    wy, wh = om.selective_scan_c(n("x")[:, :, cols], n("dt")[:, :, cols], n("A")[cols], n("B"), n("C"),
                                 n("D")[cols], n("z")[:, :, cols])
    assert _bf16_elementwise_bad(to_np(y)[:, :, cols], wy) == 0
    assert rel_l2(to_np(h)[:, cols], wh) < 1e-5


def test_scan_repeated_calls_reuse_workspace(dev):
    import mamba_selective_scan_mixer_b200 as J
    s = {k: v.to(dev) for k, v in scan_inputs(1, 640, 256, 16, seed=21).items()}
    ws = torch.empty(64 << 20, dtype=torch.uint8, device=dev)
    outs = [J.selective_scan(s["x"], s["z"], s["dt"], s["B"], s["C"], s["A"], s["D"], chunk=64, ws=ws)[0]
            for _ in range(3)]
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    J.device_status()


def test_scan_state_in_place_and_partial_overlap(dev):
    """h_out == h0 runs in place (the last time chunk writes after the first
    has published that it read h0) and matches separate buffers up to the
    carries' rounding order; an h_out that overlaps h0 without being it is
    refused with INVALID_ARG before any launch."""
    import ctypes
    import mamba_selective_scan_mixer_b200 as J
    from mamba_selective_scan_mixer_b200 import _abi
    s = {k: v.to(dev) for k, v in scan_inputs(1, 256, 256, 16, seed=22).items()}
    y = torch.empty_like(s["x"])
    h = torch.zeros(2, 256, 16, device=dev)
    n = ctypes.c_size_t()
    J.lib().jamba_selective_scan_workspace_size(1, 256, 256, 16, 64, ctypes.byref(n))
    ws = torch.empty(n.value, dtype=torch.uint8, device=dev)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    h.normal_()
    run = lambda h0, ho: J.lib().jamba_selective_scan(
        P(s["x"]), 256, P(s["z"]), 256, P(s["dt"]), 256, P(s["B"]), 16, P(s["C"]), 16, _abi.JAMBA_BF16, P(s["A"]),
        P(s["D"]), P(h0), P(y), 256, P(ho), 1, 256, 256, 16, _abi.JAMBA_BF16, 64, P(ws), ctypes.c_size_t(n.value), None)
    h_sep = torch.empty(256, 16, device=dev)
    assert run(h[0], h_sep) == 0                                  # separate buffers (4 time chunks of 64)
    y_sep = y.clone()
    h_in_place = h[0].clone()
    assert run(h_in_place, h_in_place) == 0                       # in place
    torch.cuda.synchronize()
    J.device_status()
    assert rel_l2(to_np(h_in_place), to_np(h_sep)) < 1e-6
    assert bf16_steps(to_np(y), to_np(y_sep)) <= 1
    assert run(h[0], h.view(-1)[2048:6144].view(256, 16)) == 1    # partial overlap: JAMBA_ERR_INVALID_ARG
    J.device_status()


# ------------------------------------------------------------------ norm

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_rmsnorm(dev, dtype):
    import mamba_selective_scan_mixer_b200 as J
    g = _gen(4)
    x = torch.randn(37, 4096, generator=g).to(dtype)
    w = 1 + 0.2 * torch.randn(4096, generator=g)
    got = J.rmsnorm(x.to(dev), w.to(dev), 1e-6)
    want = om.rmsnorm(to_np(x), to_np(w), 1e-6)
    assert rel_l2(to_np(got), want) < (TOL_BF16 if dtype == torch.bfloat16 else TOL_F32)
