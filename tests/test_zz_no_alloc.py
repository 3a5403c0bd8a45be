"""The selective-scan entry point that allocates nothing.

Some callers may not call cudaMalloc while they run (a library used inside
another framework whose allocator owns the device memory).  For them
jamba_selective_scan_static keeps its scratch in a static device array of
libjamba.so.  This file checks, through the C ABI, that two calls in a row
give the same results as jamba_selective_scan (the workspace entry point)
within the tolerances used everywhere else in the tests.  It sits last in
collection order so that a stop-at-first-failure run has run every other
test before it.
"""
import ctypes

import pytest
import torch

from synthetic import scan_inputs
from tests.helpers import TOL_BF16, TOL_F32, cuda_or_skip, rel_l2, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def J():
    cuda_or_skip()
    import mamba_selective_scan_mixer_b200 as J
    J.lib()
    return J


def _static_call(J, s, h0, status):
    """Direct C-ABI call of jamba_selective_scan_static; returns (y, h_out)."""
    from mamba_selective_scan_mixer_b200 import _abi
    x, z, dt, B, C, A, D = (s[k] for k in ("x", "z", "dt", "B", "C", "A", "D"))
    batch, L, di = x.shape
    y = torch.empty_like(x)
    h_out = torch.empty(batch, di, 16, dtype=torch.float32, device=x.device)
    dty = {torch.bfloat16: _abi.JAMBA_BF16, torch.float32: _abi.JAMBA_F32}
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = _abi.lib().jamba_selective_scan_static(
        p(x), di, p(z), di, p(dt), di, p(B), 16, p(C), 16, dty[B.dtype], p(A), p(D), p(h0), p(y), di, p(h_out),
        batch, L, di, 16, dty[x.dtype], p(status), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, _abi.lib().jamba_last_error()
    return y, h_out


@pytest.mark.parametrize("dtype,a_init,batch,L,di,tol", [
    ("bf16", "structured", 2, 3000, 520, TOL_BF16),   # power-form kernel, ragged channel group
    ("f32", "random", 1, 1500, 256, TOL_F32),         # general kernel
])
def test_static_scratch_scan_matches_workspace_scan(J, dtype, a_init, batch, L, di, tol):
    dev = torch.device("cuda:0")
    s = {k: v.to(dev) for k, v in scan_inputs(batch, L, di, 16, seed=L, dtype=dtype, a_init=a_init).items()}
    g = torch.Generator()
    g.manual_seed(L)
    h0 = torch.randn(batch, di, 16, generator=g).to(dev)
    ref_y, ref_h = J.selective_scan(s["x"], s["z"], s["dt"], s["B"], s["C"], s["A"], s["D"], h0)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(2):   # the second call starts from the first call's leftovers in the array
        y, h = _static_call(J, s, h0, status)
        torch.cuda.synchronize()
        assert rel_l2(to_np(y), to_np(ref_y)) < tol
        assert rel_l2(to_np(h), to_np(ref_h)) < tol
    assert int(status.item()) == 0


def test_static_scratch_scan_without_status_word(J):
    """status = NULL: the library's own word, read and cleared by jamba_device_status."""
    dev = torch.device("cuda:0")
    s = {k: v.to(dev) for k, v in scan_inputs(1, 2000, 512, 16, seed=5, dtype="bf16").items()}
    ref_y, ref_h = J.selective_scan(s["x"], s["z"], s["dt"], s["B"], s["C"], s["A"], s["D"])
    for _ in range(2):
        y, h = _static_call(J, s, None, None)
        torch.cuda.synchronize()
        assert rel_l2(to_np(y), to_np(ref_y)) < TOL_BF16
        assert rel_l2(to_np(h), to_np(ref_h)) < TOL_BF16
    J.device_status()   # raises on a latched timeout


def test_static_scratch_scan_at_the_group_limit(J):
    """682 channel groups fit the array: batch 21 at d_inner 8192 (672 groups) runs
    with one time chunk per group and matches the workspace scan."""
    dev = torch.device("cuda:0")
    s = {k: v.to(dev) for k, v in scan_inputs(21, 48, 8192, 16, seed=21, dtype="bf16").items()}
    ref_y, ref_h = J.selective_scan(s["x"], s["z"], s["dt"], s["B"], s["C"], s["A"], s["D"])
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    y, h = _static_call(J, s, None, status)
    torch.cuda.synchronize()
    assert rel_l2(to_np(y), to_np(ref_y)) < TOL_BF16
    assert rel_l2(to_np(h), to_np(ref_h)) < TOL_BF16
    assert int(status.item()) == 0


@pytest.mark.parametrize("batch", [22, 86])
def test_static_scratch_scan_rejects_sizes_beyond_the_array(J, batch):
    from mamba_selective_scan_mixer_b200 import _abi
    dev = torch.device("cuda:0")
    t = torch.zeros(16, device=dev)
    p = ctypes.c_void_p(t.data_ptr())
    # batch 22 at d_inner 8192: 704 channel groups, 48 KiB of records each even with one chunk
    st = _abi.lib().jamba_selective_scan_static(p, 8192, p, 8192, p, 8192, p, 16, p, 16, _abi.JAMBA_BF16, p, p,
                                                None, p, 8192, None, batch, 64, 8192, 16, _abi.JAMBA_BF16, None,
                                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 2   # JAMBA_ERR_UNSUPPORTED, nothing launched
    assert b"static scratch" in _abi.lib().jamba_last_error()
