"""C-ABI checks that need no GPU: the library loads, exports every function
include/jamba.h declares, and rejects bad arguments before touching a device."""
import ctypes
import os
import subprocess
import sys

import pytest

from tests.helpers import ROOT, header_symbols


@pytest.fixture(scope="module")
def lib():
    from mamba_selective_scan_mixer_b200 import build, _abi
    build.build()
    return _abi.lib()


def test_header_declares_the_entry_points():
    names = header_symbols()
    for n in ("jamba_mamba_create", "jamba_mamba_prefill", "jamba_mamba_step", "jamba_moe_forward",
              "jamba_selective_scan", "jamba_mamba_destroy", "jamba_mamba_workspace_size"):
        assert n in names


def test_library_exports_every_header_symbol(lib):
    missing = [n for n in header_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_header_symbol():
    from mamba_selective_scan_mixer_b200._abi import SIGNATURES
    declared = set(header_symbols()) - {"jamba_last_error", "jamba_checked_build"}   # not jamba_status
    assert declared == set(SIGNATURES), declared ^ set(SIGNATURES)


def test_exports_with_nm(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", os.path.join(ROOT, "mamba_selective_scan_mixer_b200",
                                                                      "libjamba.so")],
                         capture_output=True, text=True).stdout
    for n in header_symbols():
        assert (" T " + n) in out, n


def test_checked_build_exports_the_same_symbols_and_says_so(lib):
    """libjamba_checked.so (-DJAMBA_CHECKS) exports every header symbol and
    jamba_checked_build() tells the two builds apart (no GPU needed)."""
    from mamba_selective_scan_mixer_b200 import build
    path = build.build(checked=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    for n in header_symbols():
        assert (" T " + n) in out, n
    chk = ctypes.CDLL(path)
    assert chk.jamba_checked_build() == 1
    assert lib.jamba_checked_build() == 0


def test_create_rejects_bad_config_without_gpu(lib):
    from mamba_selective_scan_mixer_b200 import _abi
    h = ctypes.c_void_p()
    cfg = _abi.MambaConfig(64, 128, 8, 4, 4, _abi.JAMBA_F32, 0, 1e-6)   # d_state 8: unsupported
    w = _abi.MambaWeights(*([ctypes.c_void_p(4096)] * 12))
    assert lib.jamba_mamba_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == 2
    assert b"d_state" in lib.jamba_last_error()
    cfg = _abi.MambaConfig(64, 128, 16, 3, 4, _abi.JAMBA_F32, 0, 1e-6)   # d_conv 3
    assert lib.jamba_mamba_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == 2
    cfg = _abi.MambaConfig(64, 128, 16, 4, 4, _abi.JAMBA_F32, 0, 1e-6)
    w2 = _abi.MambaWeights(*([ctypes.c_void_p(4096)] * 8 + [None] + [ctypes.c_void_p(4096)] * 3))
    assert lib.jamba_mamba_create(ctypes.byref(cfg), ctypes.byref(w2), ctypes.byref(h)) == 1
    assert b"out_proj" in lib.jamba_last_error()
    w3 = _abi.MambaWeights(*([ctypes.c_void_p(4100)] + [ctypes.c_void_p(4096)] * 11))  # misaligned
    assert lib.jamba_mamba_create(ctypes.byref(cfg), ctypes.byref(w3), ctypes.byref(h)) == 1
    assert lib.jamba_mamba_create(None, ctypes.byref(w), ctypes.byref(h)) == 1


def test_scan_and_moe_reject_bad_shapes_without_gpu(lib):
    from mamba_selective_scan_mixer_b200 import _abi
    n = ctypes.c_size_t()
    assert lib.jamba_selective_scan_workspace_size(1, 16, 64, 8, 0, ctypes.byref(n)) == 2
    assert lib.jamba_selective_scan_workspace_size(1, 0, 64, 16, 0, ctypes.byref(n)) == 1
    assert lib.jamba_selective_scan_workspace_size(1, 64, 64, 16, 24, ctypes.byref(n)) == 1
    p = ctypes.c_void_p(4096)
    st = lib.jamba_selective_scan(p, 64, p, 64, p, 64, p, 16, p, 16, 1, p, p, None, p, 64, None,
                                  1, 64, 64, 8, 1, 0, p, 1 << 20, None)
    assert st == 2
    BF, I8 = _abi.JAMBA_BF16, _abi.JAMBA_INT8
    cfg = _abi.MoeConfig(4096, 14336, 16, 3, BF, BF)      # top_k 3
    assert lib.jamba_moe_workspace_size(ctypes.byref(cfg), 128, ctypes.byref(n)) == 2
    cfg = _abi.MoeConfig(4096, 14336, 16, 2, _abi.JAMBA_F32, BF)       # fp32 MoE
    assert lib.jamba_moe_workspace_size(ctypes.byref(cfg), 128, ctypes.byref(n)) == 2
    cfg = _abi.MoeConfig(4096, 14336, 16, 2, BF, _abi.JAMBA_F32)       # fp32 expert weights
    assert lib.jamba_moe_workspace_size(ctypes.byref(cfg), 128, ctypes.byref(n)) == 2
    cfg = _abi.MoeConfig(4096, 14336, 16, 2, BF, I8)                   # ExpertsInt8
    assert lib.jamba_moe_workspace_size(ctypes.byref(cfg), 128, ctypes.byref(n)) == 0
    cfg = _abi.MoeConfig(4096, 14336, 16, 2, BF, BF)
    assert lib.jamba_moe_workspace_size(ctypes.byref(cfg), 32768, ctypes.byref(n)) == 0
    # routed rows 65536: gathered input, SwiGLU activations and fp32 expert outputs dominate
    assert n.value >= 65536 * (4096 * 2 + 14336 * 2 + 4096 * 4)
    # int8 MoE without scales, and the quantiser's argument checks, fail before any launch
    w = _abi.MoeWeights(p, p, p, p, None, None, None)
    cfg = _abi.MoeConfig(4096, 14336, 16, 2, BF, I8)
    st = lib.jamba_moe_forward(ctypes.byref(cfg), ctypes.byref(w), p, None, p, 64, p, p, p, p, p, 1 << 30, None)
    assert st == 1
    assert lib.jamba_quantize_int8_rows(p, BF, 16, 12, p, p, None) == 1     # cols not a multiple of 8
    assert lib.jamba_quantize_int8_rows(p, BF, 0, 16, p, p, None) == 1      # no rows
    assert lib.jamba_quantize_int8_rows(p, I8, 16, 16, p, p, None) == 2     # int8 input
    assert lib.jamba_quantize_int8_rows(ctypes.c_void_p(4100), BF, 16, 16, p, p, None) == 1  # misaligned


def test_product_path_fails_loudly_without_library(tmp_path):
    code = ("import mamba_selective_scan_mixer_b200._abi as a; a.LIB_PATH = '/nonexistent/libjamba.so';\n"
            "try:\n    a.lib()\nexcept ImportError as e:\n    print('raised', e)\n")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT)
    assert "raised" in r.stdout, r.stdout + r.stderr


def test_binding_refuses_host_tensors():
    """no CPU path: every binding call with a host tensor raises before the library runs"""
    import torch
    import mamba_selective_scan_mixer_b200 as J
    bf = torch.bfloat16
    a = torch.zeros(128, 64, dtype=bf)
    calls = [
        lambda: J.gemm(a, a),
        lambda: J.rmsnorm(a, torch.ones(64)),
        lambda: J.causal_conv1d(torch.zeros(1, 8, 64, dtype=bf), torch.zeros(64, 4, dtype=bf), torch.zeros(64, dtype=bf)),
        lambda: J.in_proj_conv1d(torch.zeros(1, 8, 64, dtype=bf), torch.zeros(256, 64, dtype=bf),
                                 torch.zeros(128, 4, dtype=bf), torch.zeros(128, dtype=bf)),
        lambda: J.quantize_int8_rows(a),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA tensors only"):
            call()


def test_no_product_module_imports_the_oracle():
    pkg = os.path.join(ROOT, "mamba_selective_scan_mixer_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".hpp", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f


def test_attention_entry_points_validate_without_gpu(lib):
    """Config and argument checks of the attention entry points (no launch reached)."""
    from mamba_selective_scan_mixer_b200 import _abi
    n = ctypes.c_size_t()
    BF = _abi.JAMBA_BF16
    good = _abi.AttnConfig(4096, 32, 8, 128, BF)
    assert lib.jamba_attn_prefill_workspace_size(ctypes.byref(good), 1, 32768, ctypes.byref(n)) == 0
    # q|k|v rows (6144 wide) + V transposed + attention output, bf16
    assert n.value >= 32768 * (6144 + 1024 + 4096) * 2
    assert lib.jamba_attn_step_workspace_size(ctypes.byref(good), 64, 2048, ctypes.byref(n)) == 0
    for bad, code in ((_abi.AttnConfig(4096, 32, 8, 64, BF), 2),        # head_dim 64
                      (_abi.AttnConfig(4096, 32, 7, 128, BF), 1),       # 7 does not divide 32
                      (_abi.AttnConfig(4096, 32, 8, 128, _abi.JAMBA_F32), 2),
                      (_abi.AttnConfig(4000, 32, 8, 128, BF), 2)):      # d_model not a multiple of 64
        assert lib.jamba_attn_prefill_workspace_size(ctypes.byref(bad), 1, 128, ctypes.byref(n)) == code
    assert lib.jamba_attn_prefill_workspace_size(ctypes.byref(good), 1, 0, ctypes.byref(n)) == 1
    p = ctypes.c_void_p(4096)
    w = _abi.AttnWeights(p, p)
    ws = ctypes.c_void_p(8192)
    # out aliasing x, one cache without the other, max_len below seqlen, null lengths: rejected up front
    assert lib.jamba_attn_prefill(ctypes.byref(good), ctypes.byref(w), p, None, p, 1, 128, None, None, 0,
                                  ws, 1 << 30, None) == 1
    q = ctypes.c_void_p(1 << 20)
    assert lib.jamba_attn_prefill(ctypes.byref(good), ctypes.byref(w), p, None, q, 1, 128, p, None, 256,
                                  ws, 1 << 30, None) == 1
    assert lib.jamba_attn_prefill(ctypes.byref(good), ctypes.byref(w), p, None, q, 1, 128, p, p, 64,
                                  ws, 1 << 30, None) == 1
    assert lib.jamba_attn_prefill(ctypes.byref(good), ctypes.byref(w), p, None, q, 1, 128, None, None, 0,
                                  ws, 16, None) == 3                      # workspace too small
    assert lib.jamba_attn_step(ctypes.byref(good), ctypes.byref(w), p, None, q, 4, p, p, 256, None,
                               ws, 1 << 30, None) == 1
    assert lib.jamba_attn_step(ctypes.byref(good), ctypes.byref(w), ctypes.c_void_p(4100), None, q, 4, p, p,
                               256, p, ws, 1 << 30, None) == 1            # misaligned x
