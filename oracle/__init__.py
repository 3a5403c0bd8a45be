"""fp64 CPU oracle for the Jamba Mamba mixer and its top-2 MoE.

TEST INFRASTRUCTURE.  This package exists to check the CUDA library; it is
not part of the product path.  Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference arm may import, call, link or
execute anything in it.  It imports nothing from the CUDA package and the
CUDA package imports nothing from it; the only code both sides use is the
seeded input generators in ``synthetic/``.

Everything is float64 numpy, written step by step in the order the method
defines, with numpy matmul as the only library primitive and a plain C loop
(``scan_seq.c``) for the sequential scan at long sequence lengths.

Sources (titles and sections of the pages the method is taken from):
  * "Jamba: A Hybrid Transformer-Mamba Language Model" (paper summary page),
    section 2 "Model architecture": Mamba layers with RMSNorm inside, no
    positional encoding, SwiGLU MLPs, MoE with n experts and top-K routing;
    section 3.1: n = 16, K = 2; section 6.4: RMSNorm on the Mamba layer's
    inner activations.
  * The Mamba layer the paper cites (section 2, ref [17]) is taken in its
    standard form: in_proj -> causal depthwise conv1d -> SiLU -> x_proj ->
    dt_proj + softplus -> selective scan
    h_t = exp(dt_t * A) * h_{t-1} + dt_t * B_t * x_t,
    y_t = C_t . h_t + D * x_t -> SiLU(z) gate -> out_proj.

Parity status per function is listed in each module header.
"""
from . import attention, mamba, moe  # noqa: F401
