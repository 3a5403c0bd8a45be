"""Failure detection on the GPU without a fault: a bounded device wait that
runs out, through the C ABI.

The scan's CTAs wait (bounded) on the flag a predecessor chunk publishes.
jamba_test_scan_missing_predecessor launches every chunk but the first, so
that flag is never set: each waiting CTA must give up after the given limit,
latch JAMBA_ERR_TIMEOUT in the device error word and return, leaving the
context usable.  No access leaves the caller's tensors or the workspace.
"""
import ctypes
import time

import pytest
import torch

from oracle import mamba as om
from synthetic import scan_inputs
from tests.helpers import TOL_BF16, cuda_or_skip, rel_l2, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def J():
    cuda_or_skip()
    import mamba_selective_scan_mixer_b200 as J
    J.lib()
    return J


def _missing_predecessor(s, chunk, wait_ns):
    from mamba_selective_scan_mixer_b200 import _abi
    x, z, dt, B, C, A, D = (s[k] for k in ("x", "z", "dt", "B", "C", "A", "D"))
    batch, L, di = x.shape
    y = torch.empty_like(x)
    h_out = torch.empty(batch, di, 16, dtype=torch.float32, device=x.device)
    n = ctypes.c_size_t()
    _abi.check(_abi.lib().jamba_selective_scan_workspace_size(batch, L, di, 16, chunk, ctypes.byref(n)))
    ws = torch.empty(n.value, dtype=torch.uint8, device=x.device)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return _abi.lib().jamba_test_scan_missing_predecessor(
        p(x), di, p(z), di, p(dt), di, p(B), 16, p(C), 16, _abi.JAMBA_BF16, p(A), p(D), p(y), di, p(h_out),
        batch, L, di, 16, _abi.JAMBA_BF16, chunk, wait_ns, p(ws), n.value, stream), stream


def test_scan_wait_on_unpublished_predecessor_times_out_and_recovers(J):
    from mamba_selective_scan_mixer_b200 import _abi
    dev = torch.device("cuda:0")
    # i.i.d. dt around 0.02: every chunk's carried state outlives its 512 steps,
    # so each look-back walks back to chunk 0, whose flag nobody sets
    s = {k: v.to(dev) for k, v in scan_inputs(1, 4096, 512, 16, seed=41, dtype="bf16").items()}
    assert _abi.lib().jamba_device_status(None) == 0          # clean start
    t0 = time.perf_counter()
    st, stream = _missing_predecessor(s, chunk=512, wait_ns=2_000_000)   # 2 ms limit
    assert st == 0, _abi.lib().jamba_last_error()
    code = _abi.lib().jamba_device_status(stream)          # synchronizes: every CTA has returned
    elapsed = time.perf_counter() - t0
    assert code == 5, (code, _abi.lib().jamba_last_error())  # JAMBA_ERR_TIMEOUT
    assert b"gave up" in _abi.lib().jamba_last_error()
    assert elapsed < 3.0   # far below the 4 s default limit: the test limit was used
    # the word was read and cleared, the context still works, and the next scan is right
    assert _abi.lib().jamba_device_status(stream) == 0
    y, h = J.selective_scan(s["x"], s["z"], s["dt"], s["B"], s["C"], s["A"], s["D"], chunk=512)
    J.device_status()
    s64 = {k: om.to64(v) for k, v in s.items()}
    wy, wh = om.selective_scan_c(s64["x"], s64["dt"], s64["A"], s64["B"], s64["C"], s64["D"], s64["z"])
    assert rel_l2(to_np(y), wy) < TOL_BF16
    assert rel_l2(to_np(h), wh) < TOL_BF16


def test_missing_predecessor_test_hook_rejects_a_single_chunk(J):
    from mamba_selective_scan_mixer_b200 import _abi
    dev = torch.device("cuda:0")
    s = {k: v.to(dev) for k, v in scan_inputs(1, 256, 256, 16, seed=42, dtype="bf16").items()}
    st, _ = _missing_predecessor(s, chunk=256, wait_ns=1_000_000)
    assert st == 1   # JAMBA_ERR_INVALID_ARG, nothing launched
