"""Workload sizes.

Widths follow the Jamba paper (Lieber et al., "Jamba: A Hybrid
Transformer-Mamba Language Model", section 3.1: n = 16 experts, top-K = 2)
and the Mamba layer it cites (section 2, ref [17]); the per-workload sizes
(d_model 4096, d_inner 8192, d_state 16, d_conv 4, dt_rank 256, d_ff 14336,
the batch and sequence lengths) are the benchmark configurations this
library is measured on.
"""
from dataclasses import dataclass, replace


@dataclass(frozen=True)
class MambaShape:
    d_model: int
    d_inner: int
    d_state: int = 16
    d_conv: int = 4
    dt_rank: int = 256
    dtype: str = "bf16"          # "bf16" or "f32": weights and activations
    inner_norm: bool = True      # RMSNorm on dt_low / B / C
    eps: float = 1e-6

    def with_(self, **kw):
        return replace(self, **kw)


@dataclass(frozen=True)
class MoEShape:
    d_model: int = 4096
    d_ff: int = 14336
    n_experts: int = 16
    top_k: int = 2
    dtype: str = "bf16"

    def with_(self, **kw):
        return replace(self, **kw)


@dataclass(frozen=True)
class AttnShape:
    d_model: int = 4096
    n_heads: int = 32
    n_kv_heads: int = 8
    head_dim: int = 128
    dtype: str = "bf16"

    def with_(self, **kw):
        return replace(self, **kw)


JAMBA_MAMBA = MambaShape(d_model=4096, d_inner=8192, d_state=16, d_conv=4,
                         dt_rank=256, dtype="bf16", inner_norm=True)

WORKLOADS = {
    # tiny fp32 mixer: prefill of 256 tokens then 16 decode steps
    "tiny_fp32": dict(mamba=MambaShape(d_model=64, d_inner=128, dt_rank=4,
                                       dtype="f32", inner_norm=False),
                      batch=1, seqlen=256, steps=16),
    # Jamba-width prefill, 4096 tokens
    "prefill_4k": dict(mamba=JAMBA_MAMBA, batch=1, seqlen=4096),
    # Jamba-width prefill at 128K context
    "prefill_128k": dict(mamba=JAMBA_MAMBA, batch=1, seqlen=131072),
    # selective scan + gate alone at 128K context
    "scan_128k": dict(batch=1, seqlen=131072, d_inner=8192, d_state=16),
    # one-token decode, batch 64, caches from a 2048-token prefill
    "decode_b64": dict(mamba=JAMBA_MAMBA, batch=64, prefill=2048, steps=1024),
    # RMSNorm -> Mamba -> residual -> RMSNorm -> top-2-of-16 MoE -> residual
    "layer_pair": dict(mamba=JAMBA_MAMBA, moe=MoEShape(), batch=4, seqlen=8192),
    # the block's GQA attention layer: prefill of 32768 tokens (batch 1)
    "attn_32k": dict(attn=AttnShape(), batch=1, seqlen=32768),
}


def workload(name):
    return dict(WORKLOADS[name])
