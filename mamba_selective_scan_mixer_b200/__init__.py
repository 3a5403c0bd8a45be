"""B200 (sm_100a) Jamba Mamba mixer and top-2 MoE behind a C ABI (include/jamba.h).

The compute path is libjamba.so; this package only marshals torch tensors to
it.  There is no CPU or PyTorch fallback: calls raise if the library is not
built or the tensors are not on a CUDA device.
"""
from ._abi import JambaError, LIB_PATH, SIGNATURES, lib  # noqa: F401
from .ops import (Attention, MambaMixer, MoE, causal_conv1d, device_status, gemm, in_proj_conv1d, layer_pair,  # noqa: F401,E501
                  quantize_experts_int8, quantize_int8_rows, rmsnorm, selective_scan,
                  selective_scan_static)
