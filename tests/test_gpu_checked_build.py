"""The checked build of the library (libjamba_checked.so, compiled with
-DJAMBA_CHECKS): every index a kernel reads from device data (routed-row
positions, expert group offsets, the channel permutation of the reordered
caches, attention cache lengths) is tested on the device before use; a failed
test latches JAMBA_ERR_BOUNDS in the status word and the access is skipped.

- The GPU parity suites of the kernels, the mixer, the MoE and attention run
  again in a child process that loads the checked build (JAMBA_CHECKED=1); the
  conftest reads the status word after every test there, so a check that
  fires on valid inputs fails that test.
- An expert group table whose counts overrun the rows (a caller's bad counts
  on the expert-parallel path) is clamped by both builds, so no access leaves
  the tensors, and reported by the checked build only.
"""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from oracle import moe as omoe
from synthetic import MoEShape, moe_input, moe_params
from tests.helpers import TOL_BF16, cuda_or_skip, rel_l2, to_np

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECKED = os.environ.get("JAMBA_CHECKED", "0") == "1"


@pytest.fixture(scope="module")
def dev():
    d = cuda_or_skip()
    import mamba_selective_scan_mixer_b200 as J
    J.lib()
    return d


def test_the_loaded_library_is_the_requested_build(dev):
    from mamba_selective_scan_mixer_b200 import _abi
    assert _abi.lib().jamba_checked_build() == (1 if CHECKED else 0)
    assert os.path.basename(_abi.LIB_PATH) == ("libjamba_checked.so" if CHECKED else "libjamba.so")


def test_group_counts_past_the_rows(dev):
    """Local experts over 40 received rows whose group counts add up to 80:
    group 0 takes all 40 rows, group 1 is clipped to nothing.  Both builds
    compute exactly that; only the checked build reports the table."""
    import mamba_selective_scan_mixer_b200 as J
    from mamba_selective_scan_mixer_b200 import _abi
    shape = MoEShape(d_model=256, d_ff=128, n_experts=4, top_k=2)
    p = {k: v.to(dev) for k, v in moe_params(shape, seed=41).items()}
    R = 40
    rows_in = moe_input(shape, R, seed=41).to(dev)
    counts = torch.tensor([R, R, 0, 0], dtype=torch.int32, device=dev)
    rows_out = torch.full((R, shape.d_model), float("nan"), device=dev)
    cfg = _abi.MoeConfig(shape.d_model, shape.d_ff, shape.n_experts, shape.top_k, _abi.JAMBA_BF16, _abi.JAMBA_BF16)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    w = _abi.MoeWeights(P(p["router"]), P(p["w_gate"]), P(p["w_up"]), P(p["w_down"]), None, None, None)
    n = ctypes.c_size_t()
    _abi.check(_abi.lib().jamba_moe_ep_experts_workspace_size(ctypes.byref(cfg), R, 1, ctypes.byref(n)))
    ws = torch.empty(max(n.value, 256), dtype=torch.uint8, device=dev)
    _abi.check(_abi.lib().jamba_moe_ep_experts(ctypes.byref(cfg), ctypes.byref(w), P(rows_in), R, P(counts), 1,
                                               P(rows_out), P(ws), ws.numel(), None))
    torch.cuda.synchronize()
    if CHECKED:
        with pytest.raises(_abi.JambaError) as e:
            J.device_status()
        assert e.value.status == _abi.JAMBA_ERR_BOUNDS
    else:
        J.device_status()
    want = omoe.swiglu_expert(to_np(rows_in), to_np(p["w_gate"][0]), to_np(p["w_up"][0]), to_np(p["w_down"][0]))
    got = to_np(rows_out)
    assert np.isfinite(got).all()
    assert rel_l2(got, want) < TOL_BF16


@pytest.mark.skipif(CHECKED, reason="runs the suites under the checked build; not again inside it")
def test_parity_suites_under_the_checked_build(dev):
    from mamba_selective_scan_mixer_b200 import build
    if not os.path.exists(build.LIB_CHECKED):
        pytest.fail("libjamba_checked.so is not built (python -m mamba_selective_scan_mixer_b200.build --checked)")
    env = dict(os.environ, JAMBA_CHECKED="1")
    files = ["tests/test_gpu_kernels.py", "tests/test_gpu_mixer.py", "tests/test_gpu_moe.py",
             "tests/test_gpu_attention.py", "tests/test_gpu_checked_build.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", *files, "-m", "gpu and not slow", "-q", "-x",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
