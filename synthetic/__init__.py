"""Seeded synthetic inputs shared by the oracle and the CUDA path.

This package holds workload sizes and random draws only: no step of the Mamba
mixer, of the MoE or of the attention layer is computed here.  Both sides of
every parity check take their inputs from these functions, so the two never
share arithmetic.
"""
from .workloads import (AttnShape, MambaShape, MoEShape, WORKLOADS, workload)  # noqa: F401
from .generators import (mamba_params, mamba_input, scan_inputs,  # noqa: F401
                         moe_params, moe_input, decode_inputs, block_norm_params,
                         attn_params, attn_input)
