"""ctypes declarations of include/jamba.h and the loader of libjamba.so.

Argument marshalling only: every step of the computation runs in the CUDA
library.  Importing this module does not load the library; the first call
does, and raises if libjamba.so has not been built.  With JAMBA_CHECKED=1 in
the environment the checked build (libjamba_checked.so: device-side index
checks that report JAMBA_ERR_BOUNDS) is loaded instead.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
CHECKED = os.environ.get("JAMBA_CHECKED", "0") == "1"
LIB_PATH = os.path.join(HERE, "libjamba_checked.so" if CHECKED else "libjamba.so")

JAMBA_OK = 0
STATUS_NAMES = {0: "JAMBA_OK", 1: "JAMBA_ERR_INVALID_ARG", 2: "JAMBA_ERR_UNSUPPORTED",
                3: "JAMBA_ERR_WORKSPACE", 4: "JAMBA_ERR_CUDA", 5: "JAMBA_ERR_TIMEOUT",
                6: "JAMBA_ERR_OOM", 7: "JAMBA_ERR_BOUNDS"}
JAMBA_ERR_BOUNDS = 7
JAMBA_F32 = 0
JAMBA_BF16 = 1
JAMBA_INT8 = 2


class JambaError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, status), msg))
        self.status = status


class MambaConfig(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("d_inner", ctypes.c_int), ("d_state", ctypes.c_int),
                ("d_conv", ctypes.c_int), ("dt_rank", ctypes.c_int), ("dtype", ctypes.c_int),
                ("inner_rmsnorm", ctypes.c_int), ("eps", ctypes.c_float)]


class MambaWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("in_proj", "conv_w", "conv_b", "x_proj", "dt_proj", "dt_bias", "A", "D",
                 "out_proj", "norm_dt", "norm_B", "norm_C")]


class MoeConfig(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("d_ff", ctypes.c_int), ("n_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("dtype", ctypes.c_int), ("expert_dtype", ctypes.c_int)]


class MoeWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("router", "w_gate", "w_up", "w_down",
                                               "s_gate", "s_up", "s_down")]


class AttnConfig(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("n_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("dtype", ctypes.c_int)]


class AttnWeights(ctypes.Structure):
    _fields_ = [("w_qkv", ctypes.c_void_p), ("w_o", ctypes.c_void_p)]


P = ctypes.c_void_p
I = ctypes.c_int
SZ = ctypes.c_size_t
F = ctypes.c_float

# name -> argument types (all return jamba_status as int, except jamba_last_error)
SIGNATURES = {
    "jamba_device_status": [P],
    "jamba_mamba_create": [ctypes.POINTER(MambaConfig), ctypes.POINTER(MambaWeights), ctypes.POINTER(P)],
    "jamba_mamba_destroy": [P],
    "jamba_mamba_workspace_size": [P, I, I, ctypes.POINTER(SZ)],
    "jamba_mamba_prefill": [P, P, P, P, I, I, P, P, P, P, P, SZ, P],
    "jamba_mamba_step": [P, P, P, P, I, P, P, P, SZ, P],
    "jamba_mamba_host_workspace_size": [P, I, I, ctypes.POINTER(SZ)],
    "jamba_mamba_prefill_host": [P, P, P, P, I, I, I, P, P, P, P, P, SZ, P],
    "jamba_mamba_prefill_tp_begin": [P, P, I, I, P, P, P, P, SZ, P],
    "jamba_mamba_prefill_tp_finish": [P, P, I, I, P, P, P, P, SZ, P],
    "jamba_mamba_prefill_tp_end": [P, P, P, P, I, I, P],
    "jamba_mamba_cp_workspace_size": [P, I, I, ctypes.POINTER(SZ)],
    "jamba_mamba_prefill_cp_begin": [P, P, P, I, I, P, P, P, P, P, P, SZ, P],
    "jamba_mamba_prefill_cp_finish": [P, P, P, I, I, I, P, P, P, P, P, SZ, P],
    "jamba_selective_scan_workspace_size": [I, I, I, I, I, ctypes.POINTER(SZ)],
    "jamba_selective_scan": [P, I, P, I, P, I, P, I, P, I, I, P, P, P, P, I, P, I, I, I, I, I, I, P, SZ, P],
    "jamba_selective_scan_static": [P, I, P, I, P, I, P, I, P, I, I, P, P, P, P, I, P, I, I, I, I, I, P, P],
    "jamba_test_scan_plan": [I, I, I, P, I, P, P, P],
    "jamba_test_gemm_splits": [I, I, I, I, I, I, P, P],
    "jamba_test_host_chunks": [I, I, P, I, P],
    "jamba_test_scan_missing_predecessor": [P, I, P, I, P, I, P, I, P, I, I, P, P, P, I, P, I, I, I, I, I, I,
                                            ctypes.c_ulonglong, P, SZ, P],
    "jamba_rmsnorm": [P, P, P, I, I, F, I, P],
    "jamba_causal_conv1d": [P, I, P, P, P, P, P, I, I, I, I, P],
    "jamba_in_proj_conv1d": [P, P, P, P, P, P, P, P, I, I, I, I, P],
    "jamba_gemm": [P, P, P, I, P, I, I, I, I, I, P],
    "jamba_quantize_int8_rows": [P, I, ctypes.c_longlong, I, P, P, P],
    "jamba_moe_workspace_size": [ctypes.POINTER(MoeConfig), I, ctypes.POINTER(SZ)],
    "jamba_moe_forward": [ctypes.POINTER(MoeConfig), ctypes.POINTER(MoeWeights), P, P, P, I, P, P, P, P,
                          P, SZ, P],
    "jamba_moe_ep_dispatch": [ctypes.POINTER(MoeConfig), P, P, I, P, P, P, P, P, P, SZ, P],
    "jamba_moe_ep_experts_workspace_size": [ctypes.POINTER(MoeConfig), I, I, ctypes.POINTER(SZ)],
    "jamba_moe_ep_experts": [ctypes.POINTER(MoeConfig), ctypes.POINTER(MoeWeights), P, I, P, I, P, P, SZ, P],
    "jamba_moe_ep_combine": [ctypes.POINTER(MoeConfig), P, P, I, P, P, P, SZ, P],
    "jamba_attn_prefill_workspace_size": [ctypes.POINTER(AttnConfig), I, I, ctypes.POINTER(SZ)],
    "jamba_attn_prefill": [ctypes.POINTER(AttnConfig), ctypes.POINTER(AttnWeights), P, P, P, I, I, P, P, I,
                           P, SZ, P],
    "jamba_attn_step_workspace_size": [ctypes.POINTER(AttnConfig), I, I, ctypes.POINTER(SZ)],
    "jamba_attn_step": [ctypes.POINTER(AttnConfig), ctypes.POINTER(AttnWeights), P, P, P, I, P, P, I, P,
                        P, SZ, P],
}

_lib = None


def lib():
    """The loaded library; raises if it is missing (there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("%s is not built (python -m mamba_selective_scan_mixer_b200.build%s)"
                              % (os.path.basename(LIB_PATH), " --checked" if CHECKED else ""))
        L = ctypes.CDLL(LIB_PATH)
        L.jamba_last_error.restype = ctypes.c_char_p
        L.jamba_last_error.argtypes = []
        L.jamba_checked_build.restype = ctypes.c_int
        L.jamba_checked_build.argtypes = []
        for name, args in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = ctypes.c_int
            f.argtypes = args
        _lib = L
    return _lib


def check(status):
    if status != JAMBA_OK:
        raise JambaError(status, lib().jamba_last_error().decode())
    return status
