"""Context-parallel Mamba prefill: one sequence split over ranks by time.

Rank r holds tokens [t_r, t_r+1) of every batch row.  The scan is
associative: after a slice the state is P * h_in + h_loc, with P the
product of the slice's decays exp(dt A) and h_loc the slice's end state from
zero.  So each rank runs jamba_mamba_prefill_cp_begin on its slice (every
step up to a state-only scan from zero), the ranks all-gather their
(P, h_loc) carries, and each rank runs jamba_mamba_prefill_cp_finish, which
folds the carries of the ranks before it into the state entering its slice
and scans the slice from there.  The causal conv needs the 3 input rows
before the slice: the last 3 rows of every rank's u are all-gathered first.

The collectives are torch.distributed's (NCCL over NVLink between GPUs;
gloo, through host copies, where the process group is gloo).  Per batch row
the exchange is 3 x d_model input rows and 2 x d_inner x 16 fp32 carries per
rank: 1 MiB at Jamba width.  Every step of the computation runs in
libjamba.so.
"""
import torch
import torch.distributed as dist


def _all_gather(t, group=None):
    """[world, *t.shape] on t's device, in rank order."""
    world = dist.get_world_size(group)
    if dist.get_backend(group) == "gloo":
        src = t.detach().to("cpu").contiguous()
        parts = [torch.empty_like(src) for _ in range(world)]
        dist.all_gather(parts, src, group=group)
        return torch.stack(parts).to(t.device)
    out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
    dist.all_gather_into_tensor(out, t.contiguous(), group=group)
    return out


def exchange_halo(u, group=None, width=3):
    """The `width` input rows before this rank's slice ([B, width, d_model]),
    from the previous rank; None on rank 0."""
    if u.shape[1] < width:
        raise ValueError("context-parallel prefill needs at least %d tokens per rank" % width)
    tails = _all_gather(u[:, -width:].contiguous(), group)
    rank = dist.get_rank(group)
    return None if rank == 0 else tails[rank - 1].contiguous()


def prefill_cp(mixer, u, group=None, residual=None, conv_state_in=None, ssm_state_in=None, out=None):
    """Prefill of this rank's slice u [B, L_r, d_model] of sequences split by time.

    conv_state_in / ssm_state_in: caches before the first slice (read on rank
    0 only, where the state seeds rank 0's carry; None = zeros).  Returns
    (out, conv_state_out, ssm_state_out): the
    slice's output and the caches after the slice (the sequences' final
    caches on the last rank).
    """
    rank = dist.get_rank(group)
    u_halo = exchange_halo(u, group, mixer.shape.d_conv - 1)
    first = rank == 0
    conv_out, carry_p, carry_h = mixer.prefill_cp_begin(u, u_halo=u_halo,
                                                        conv_state_in=conv_state_in if first else None,
                                                        ssm_state_in=ssm_state_in if first else None)
    carries_p = _all_gather(carry_p, group)
    carries_h = _all_gather(carry_h, group)
    out, ss = mixer.prefill_cp_finish(rank, carries_p, carries_h, ssm_state_in=ssm_state_in if first else None,
                                      residual=residual, out=out)
    return out, conv_out, ss
