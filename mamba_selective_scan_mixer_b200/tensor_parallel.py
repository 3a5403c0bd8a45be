"""Tensor-parallel Mamba prefill: the d_inner channels split over ranks.

Rank r owns channels [r * d_inner / world, (r + 1) * d_inner / world): its
shares of in_proj (the x and z rows of those channels), conv, x_proj
(columns), dt_proj (rows), dt_bias, A, D and out_proj (columns); the norm
weights are whole on every rank.  Conv, dt_proj and the scan are per channel;
x_proj and out_proj contract over d_inner, so each rank produces a partial
sum and the ranks all-reduce it: once for the x_proj output [T, R + 2N]
(before the inner norms) and once for the mixer output [T, d_model].  Every
step of the computation runs in libjamba.so (jamba_mamba_prefill_tp_begin /
_finish / _end); the collectives are torch.distributed's (NCCL between GPUs;
gloo through host copies).
"""
import torch
import torch.distributed as dist


def shard_params(p, rank, world):
    """This rank's weights from the full parameter dict (tensors on any device)."""
    di = p["D"].shape[0]
    if di % world or (di // world) % 8:
        raise ValueError("d_inner must split into equal shards of a multiple of 8 channels")
    k = di // world
    c0, c1 = rank * k, (rank + 1) * k
    q = {
        "in_proj": torch.cat([p["in_proj"][c0:c1], p["in_proj"][di + c0:di + c1]]).contiguous(),
        "conv_w": p["conv_w"][c0:c1].contiguous(),
        "conv_b": p["conv_b"][c0:c1].contiguous(),
        "x_proj": p["x_proj"][:, c0:c1].contiguous(),
        "dt_proj": p["dt_proj"][c0:c1].contiguous(),
        "dt_bias": p["dt_bias"][c0:c1].contiguous(),
        "A": p["A"][c0:c1].contiguous(),
        "D": p["D"][c0:c1].contiguous(),
        "out_proj": p["out_proj"][:, c0:c1].contiguous(),
    }
    for k_ in ("norm_dt", "norm_B", "norm_C"):
        q[k_] = p[k_]
    return q


def _all_reduce(t, group=None):
    """Sum over ranks, in place on t (through host memory on gloo)."""
    if dist.get_backend(group) == "gloo":
        h = t.detach().to("cpu")
        dist.all_reduce(h, group=group)
        t.copy_(h)
    else:
        dist.all_reduce(t, group=group)
    return t


def prefill_tp(mixer, u, group=None, residual=None, conv_state_in=None, ssm_state_in=None, out=None):
    """Prefill of u [B, L, d_model] (the same tokens on every rank) by this
    rank's channel shard.  conv_state_in / ssm_state_in and the returned
    caches are this rank's channels.  Returns (out, conv_state_out,
    ssm_state_out); out (with the residual) is the same on every rank."""
    part, cs = mixer.prefill_tp_begin(u, conv_state_in=conv_state_in)
    _all_reduce(part, group)
    out_part, ss = mixer.prefill_tp_finish(part, ssm_state_in=ssm_state_in)
    _all_reduce(out_part, group)
    return mixer.prefill_tp_end(out_part, residual=residual, out=out), cs, ss
