"""Expert-parallel top-K MoE: the experts split over ranks.

Rank r owns experts [r E / world, (r + 1) E / world) and routes its own
tokens.  jamba_moe_ep_dispatch routes them and lays the routed rows out in
(expert, token, slot) order, so the rows bound for rank r are one contiguous
range; the ranks exchange the per-expert row counts and then the rows
(all-to-all), jamba_moe_ep_experts runs this rank's experts on the rows it
received (grouped by source rank, then expert, with no reordering), the
outputs travel back by the reverse all-to-all, and jamba_moe_ep_combine forms
the weighted top-K sum.  Every step of the computation runs in libjamba.so;
the collectives are torch.distributed's (NCCL between GPUs, gloo through host
copies).  The all-to-all sizes must be known on the host, so each forward
reads this rank's E + 1 expert offsets back once.
"""
import ctypes

import torch
import torch.distributed as dist

from . import _abi
from ._abi import check, lib
from .ops import _Workspace, _cuda, _contig, _p, _stream


def shard_experts(params, rank, world):
    """This rank's expert weights (and scales, for int8 experts) plus the whole router."""
    E = params["router"].shape[0]
    if E % world:
        raise ValueError("the experts must split evenly over the ranks")
    k = E // world
    q = {"router": params["router"]}
    for n in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
        if n in params:
            q[n] = params[n][rank * k:(rank + 1) * k].contiguous()
    return q


def _a2a(out, inp, out_split, in_split, group):
    if dist.get_backend(group) == "gloo":
        o = torch.empty(out.shape, dtype=out.dtype)
        dist.all_to_all_single(o, inp.detach().to("cpu").contiguous(), out_split, in_split, group=group)
        out.copy_(o)
    else:
        dist.all_to_all_single(out, inp.contiguous(), out_split, in_split, group=group)
    return out


class ExpertParallelMoE:
    """params: this rank's shard (shard_experts); shape: the whole MoE (n_experts = E)."""

    def __init__(self, params, shape, group=None):
        self.shape = shape
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.params = {k: v.contiguous() for k, v in params.items()}
        _cuda(*self.params.values())
        E = shape.n_experts
        if E % self.world:
            raise ValueError("the experts must split evenly over the ranks")
        self.E_local = E // self.world
        int8 = self.params["w_gate"].dtype == torch.int8
        edt = _abi.JAMBA_INT8 if int8 else _abi.JAMBA_BF16
        self.cfg = _abi.MoeConfig(shape.d_model, shape.d_ff, E, shape.top_k, _abi.JAMBA_BF16, edt)
        self.cfg_local = _abi.MoeConfig(shape.d_model, shape.d_ff, self.E_local, shape.top_k, _abi.JAMBA_BF16, edt)
        self.w_local = _abi.MoeWeights(*[_p(self.params.get(k)) for k in
                                         ("router", "w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down")])
        self.ws = _Workspace()
        self.ws_exp = _Workspace()

    def forward(self, x, residual=None, stream=None):
        """x [T, d_model] (this rank's tokens) -> dict(out, idx, w, offsets, perm)."""
        _cuda(x, residual)
        _contig(x, "x")
        sh, dev, g = self.shape, x.device, self.group
        T, K, E, El, W = x.shape[0], sh.top_k, sh.n_experts, self.E_local, self.world
        idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        w = torch.empty(T, K, dtype=torch.float32, device=dev)
        offs = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(T * K, dtype=torch.int32, device=dev)
        send = torch.empty(T * K, sh.d_model, dtype=x.dtype, device=dev)
        n = ctypes.c_size_t()
        check(lib().jamba_moe_workspace_size(ctypes.byref(self.cfg), T, ctypes.byref(n)))
        ws = self.ws.get(n.value, dev)
        check(lib().jamba_moe_ep_dispatch(ctypes.byref(self.cfg), _p(self.params["router"]), _p(x), T, _p(idx),
                                          _p(w), _p(offs), _p(perm), _p(send), _p(ws), ws.numel(),
                                          _stream(stream)))
        off_h = offs.cpu()                                     # the all-to-all sizes live on the host
        counts = (off_h[1:] - off_h[:-1]).to(torch.int32)     # rows per expert, this rank's tokens
        send_split = [int(off_h[(r + 1) * El] - off_h[r * El]) for r in range(W)]
        recv_counts = torch.empty(W * El, dtype=torch.int32, device=dev)
        _a2a(recv_counts, counts.to(dev), [El] * W, [El] * W, g)
        rc = recv_counts.view(W, El).cpu()
        recv_split = [int(v) for v in rc.sum(1)]
        R = sum(recv_split)
        rows_in = torch.empty(R, sh.d_model, dtype=x.dtype, device=dev)
        _a2a(rows_in, send, recv_split, send_split, g)
        rows_out = torch.empty(R, sh.d_model, dtype=torch.float32, device=dev)
        check(lib().jamba_moe_ep_experts_workspace_size(ctypes.byref(self.cfg_local), R, W, ctypes.byref(n)))
        wse = self.ws_exp.get(n.value, dev)
        check(lib().jamba_moe_ep_experts(ctypes.byref(self.cfg_local), ctypes.byref(self.w_local), _p(rows_in), R,
                                         _p(recv_counts), W, _p(rows_out), _p(wse), wse.numel(), _stream(stream)))
        back = torch.empty(T * K, sh.d_model, dtype=torch.float32, device=dev)
        _a2a(back, rows_out, send_split, recv_split, g)
        out = torch.empty_like(x)
        check(lib().jamba_moe_ep_combine(ctypes.byref(self.cfg), _p(back), _p(w), T, _p(residual), _p(out), _p(ws),
                                         ws.numel(), _stream(stream)))
        return dict(out=out, idx=idx, w=w, offsets=offs, perm=perm)
