"""Torch-tensor front end of the C ABI (marshalling only).

Tensors must already live on the CUDA device; workspaces are allocated with
torch and passed down as raw pointers.  Names follow include/jamba.h.
"""
import ctypes

import torch

from . import _abi
from ._abi import check, lib

_DT = {torch.bfloat16: _abi.JAMBA_BF16, torch.float32: _abi.JAMBA_F32}
_TORCH_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libjamba works on CUDA tensors only")


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _contig(t, name):
    if t is not None and not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


class _Workspace:
    def __init__(self):
        self.buf = None

    def get(self, nbytes, device):
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != device:
            self.buf = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
        return self.buf


def device_status(stream=None):
    """Synchronizes the stream and raises if a kernel's bounded wait gave up."""
    check(lib().jamba_device_status(_stream(stream)))


class MambaMixer:
    """One Mamba mixer layer (prefill and decode) over borrowed weight tensors.

    params: dict with in_proj, conv_w, conv_b, x_proj, dt_proj, dt_bias, A, D,
    out_proj, norm_dt, norm_B, norm_C (the layout of jamba_mamba_weights).
    """

    def __init__(self, params, shape):
        self.shape = shape
        self.dtype = _TORCH_DT[shape.dtype]
        self.params = {k: v.contiguous() for k, v in params.items()}
        _cuda(*self.params.values())
        self.device = self.params["in_proj"].device
        cfg = _abi.MambaConfig(shape.d_model, shape.d_inner, shape.d_state, shape.d_conv, shape.dt_rank,
                               _DT[self.dtype], int(shape.inner_norm), float(shape.eps))
        w = _abi.MambaWeights(*[ctypes.c_void_p(self.params[k].data_ptr()) for k in
                                ("in_proj", "conv_w", "conv_b", "x_proj", "dt_proj", "dt_bias", "A", "D",
                                 "out_proj", "norm_dt", "norm_B", "norm_C")])
        self._cfg = cfg
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            check(lib().jamba_mamba_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)))
        self.handle = h
        self.ws = _Workspace()

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value and _abi._lib is not None:
            _abi._lib.jamba_mamba_destroy(h)
            self.handle = None

    def workspace_size(self, batch, seqlen):
        n = ctypes.c_size_t()
        check(lib().jamba_mamba_workspace_size(self.handle, batch, seqlen, ctypes.byref(n)))
        return n.value

    def new_states(self, batch):
        sh = self.shape
        return (torch.zeros(batch, sh.d_inner, sh.d_conv - 1, device=self.device),
                torch.zeros(batch, sh.d_inner, sh.d_state, device=self.device))

    def release_workspace(self):
        """Drop the cached device workspace (after the last call that used it
        has completed); the next call allocates one of its own size again."""
        self.ws = _Workspace()

    def prefill(self, u, residual=None, conv_state_in=None, ssm_state_in=None, conv_state_out=None,
                ssm_state_out=None, out=None, stream=None):
        """u [B, L, d_model] -> (out, conv_state_out, ssm_state_out)."""
        _cuda(u, residual)
        _contig(u, "u")
        _contig(residual, "residual")
        B, L, _ = u.shape
        if out is None:
            out = torch.empty_like(u)
        if conv_state_out is None or ssm_state_out is None:
            cs, ss = self.new_states(B)
            conv_state_out = cs if conv_state_out is None else conv_state_out
            ssm_state_out = ss if ssm_state_out is None else ssm_state_out
        nbytes = self.workspace_size(B, L)
        ws = self.ws.get(nbytes, u.device)
        check(lib().jamba_mamba_prefill(self.handle, _p(u), _p(residual), _p(out), B, L, _p(conv_state_in),
                                        _p(ssm_state_in), _p(conv_state_out), _p(ssm_state_out), _p(ws),
                                        ws.numel(), _stream(stream)))
        return out, conv_state_out, ssm_state_out

    def prefill_tp_begin(self, u, conv_state_in=None, stream=None):
        """Tensor-parallel prefill, first part, on this rank's channel shard:
        returns (xproj_part [B*L, R+2N] fp32, conv_state_out)."""
        _cuda(u, conv_state_in)
        _contig(u, "u")
        B, L, _ = u.shape
        sh = self.shape
        part = torch.empty(B * L, sh.dt_rank + 2 * sh.d_state, device=u.device)
        cs = torch.empty(B, sh.d_inner, sh.d_conv - 1, device=u.device)
        ws = self.ws.get(self.workspace_size(B, L), u.device)
        check(lib().jamba_mamba_prefill_tp_begin(self.handle, _p(u), B, L, _p(conv_state_in), _p(cs), _p(part),
                                                 _p(ws), ws.numel(), _stream(stream)))
        self._tp = (B, L)
        return part, cs

    def prefill_tp_finish(self, xproj_sum, ssm_state_in=None, stream=None):
        """Second part from the all-reduced x_proj sum: returns (out_part [B*L,
        d_model] fp32, ssm_state_out)."""
        B, L = self._tp
        _cuda(xproj_sum, ssm_state_in)
        _contig(xproj_sum, "xproj_sum")
        sh = self.shape
        out = torch.empty(B * L, sh.d_model, device=self.device)
        ss = torch.empty(B, sh.d_inner, sh.d_state, device=self.device)
        ws = self.ws.get(self.workspace_size(B, L), self.device)
        check(lib().jamba_mamba_prefill_tp_finish(self.handle, _p(xproj_sum), B, L, _p(ssm_state_in), _p(ss),
                                                  _p(out), _p(ws), ws.numel(), _stream(stream)))
        return out, ss

    def prefill_tp_end(self, out_sum, residual=None, out=None, stream=None):
        """out = out_sum (+ residual) in the model dtype, [B, L, d_model]."""
        B, L = self._tp
        _cuda(out_sum, residual, out)
        _contig(out_sum, "out_sum")
        _contig(residual, "residual")
        out = torch.empty(B, L, self.shape.d_model, dtype=self.dtype, device=self.device) if out is None else out
        check(lib().jamba_mamba_prefill_tp_end(self.handle, _p(out_sum), _p(residual), _p(out), B, L,
                                               _stream(stream)))
        return out

    def cp_workspace_size(self, batch, seqlen):
        n = ctypes.c_size_t()
        check(lib().jamba_mamba_cp_workspace_size(self.handle, batch, seqlen, ctypes.byref(n)))
        return n.value

    def prefill_cp_begin(self, u, u_halo=None, conv_state_in=None, ssm_state_in=None, stream=None):
        """First half of a context-parallel prefill on this rank's slice u
        [B, L, d_model]: returns (conv_state_out, carry_p, carry_h).  The
        slice's activations stay in this mixer's workspace for
        prefill_cp_finish."""
        _cuda(u, u_halo, conv_state_in, ssm_state_in)
        _contig(u, "u")
        _contig(u_halo, "u_halo")
        B, L, _ = u.shape
        sh = self.shape
        conv_out = torch.empty(B, sh.d_inner, sh.d_conv - 1, device=u.device)
        carry_p = torch.empty(B, sh.d_inner, sh.d_state, device=u.device)
        carry_h = torch.empty_like(carry_p)
        ws = self.ws.get(self.cp_workspace_size(B, L), u.device)
        check(lib().jamba_mamba_prefill_cp_begin(self.handle, _p(u), _p(u_halo), B, L, _p(conv_state_in),
                                                 _p(ssm_state_in), _p(conv_out), _p(carry_p), _p(carry_h),
                                                 _p(ws), ws.numel(), _stream(stream)))
        self._cp = (B, L)
        return conv_out, carry_p, carry_h

    def prefill_cp_finish(self, rank, carries_p, carries_h, ssm_state_in=None, residual=None, out=None,
                          stream=None):
        """Second half: carries_* [world, B, d_inner, 16] of every rank in rank
        order.  Returns (out, ssm_state_out)."""
        B, L = self._cp
        _cuda(carries_p, carries_h, ssm_state_in, residual, out)
        _contig(carries_p, "carries_p")
        _contig(carries_h, "carries_h")
        _contig(residual, "residual")
        sh = self.shape
        out = torch.empty(B, L, sh.d_model, dtype=self.dtype, device=self.device) if out is None else out
        ss = torch.empty(B, sh.d_inner, sh.d_state, device=self.device)
        ws = self.ws.get(self.cp_workspace_size(B, L), self.device)
        check(lib().jamba_mamba_prefill_cp_finish(self.handle, _p(residual), _p(out), B, L, int(rank),
                                                  _p(carries_p), _p(carries_h), _p(ssm_state_in), _p(ss), _p(ws),
                                                  ws.numel(), _stream(stream)))
        return out, ss

    def prefill_host(self, u_host, residual_host=None, out_host=None, chunk=0, conv_state_in=None,
                     ssm_state_in=None, conv_state_out=None, ssm_state_out=None, stream=None):
        """Prefill from and to pinned host tensors [B, L, d_model]; the library
        pipelines the transfers with the compute in time chunks of `chunk`
        tokens (0: its default).  Returns (out_host, conv_state_out, ssm_state_out);
        the caches live on the device."""
        for t, name in ((u_host, "u_host"), (residual_host, "residual_host"), (out_host, "out_host")):
            if t is not None and (t.is_cuda or not t.is_pinned()):
                raise ValueError(name + " must be a pinned host tensor")
            _contig(t, name)
        B, L, _ = u_host.shape
        if out_host is None:
            out_host = torch.empty(u_host.shape, dtype=u_host.dtype, pin_memory=True)
        if conv_state_out is None or ssm_state_out is None:
            cs, ss = self.new_states(B)
            conv_state_out = cs if conv_state_out is None else conv_state_out
            ssm_state_out = ss if ssm_state_out is None else ssm_state_out
        _cuda(conv_state_in, ssm_state_in, conv_state_out, ssm_state_out)
        n = ctypes.c_size_t()
        check(lib().jamba_mamba_host_workspace_size(self.handle, B, int(chunk), ctypes.byref(n)))
        ws = self.ws.get(n.value, self.device)
        check(lib().jamba_mamba_prefill_host(self.handle, _p(u_host), _p(residual_host), _p(out_host), B, L,
                                             int(chunk), _p(conv_state_in), _p(ssm_state_in), _p(conv_state_out),
                                             _p(ssm_state_out), _p(ws), ws.numel(), _stream(stream)))
        return out_host, conv_state_out, ssm_state_out

    def step(self, u, conv_state, ssm_state, residual=None, out=None, stream=None):
        """u [B, d_model]; updates both caches in place; returns out [B, d_model]."""
        _cuda(u, conv_state, ssm_state, residual)
        _contig(u, "u")
        B = u.shape[0]
        if out is None:
            out = torch.empty_like(u)
        nbytes = self.workspace_size(B, 1)
        ws = self.ws.get(nbytes, u.device)
        check(lib().jamba_mamba_step(self.handle, _p(u), _p(residual), _p(out), B, _p(conv_state),
                                     _p(ssm_state), _p(ws), ws.numel(), _stream(stream)))
        return out


def selective_scan(x, z, dt, B, C, A, D, h0=None, chunk=0, want_state=True, y=None, ws=None, stream=None):
    """x, z, dt [batch, L, d_inner] (row strides taken from the tensors);
    B, C [batch, L, 16]; A [d_inner, 16]; D [d_inner]; h0 [batch, d_inner, 16] or None.
    Returns (y, h_out)."""
    _cuda(x, z, dt, B, C, A, D, h0)
    batch, L, di = x.shape
    N = A.shape[1]
    for t, n in ((x, "x"), (z, "z"), (dt, "dt"), (B, "B"), (C, "C")):
        if t.stride(-1) != 1 or t.stride(0) != L * t.stride(1):
            raise ValueError("%s: rows must be unit-stride and evenly spaced" % n)
    if y is None:
        y = torch.empty(batch, L, di, dtype=x.dtype, device=x.device)
    h_out = torch.empty(batch, di, N, dtype=torch.float32, device=x.device) if want_state else None
    n = ctypes.c_size_t()
    check(lib().jamba_selective_scan_workspace_size(batch, L, di, N, chunk, ctypes.byref(n)))
    if ws is None or ws.numel() < n.value:
        ws = torch.empty(max(n.value, 256), dtype=torch.uint8, device=x.device)
    check(lib().jamba_selective_scan(_p(x), x.stride(1), _p(z), z.stride(1), _p(dt), dt.stride(1), _p(B),
                                     B.stride(1), _p(C), C.stride(1), _DT[B.dtype], _p(A), _p(D), _p(h0),
                                     _p(y), y.stride(1), _p(h_out), batch, L, di, N, _DT[x.dtype], chunk,
                                     _p(ws), ws.numel(), _stream(stream)))
    return y, h_out


def selective_scan_static(x, z, dt, B, C, A, D, h0=None, want_state=True, y=None, status=None, stream=None):
    """selective_scan() through the entry point that allocates nothing (its
    scratch is a static device array inside libjamba.so).  Returns (y, h_out)."""
    _cuda(x, z, dt, B, C, A, D, h0, status)
    batch, L, di = x.shape
    N = A.shape[1]
    for t, n in ((x, "x"), (z, "z"), (dt, "dt"), (B, "B"), (C, "C")):
        if t.stride(-1) != 1 or t.stride(0) != L * t.stride(1):
            raise ValueError("%s: rows must be unit-stride and evenly spaced" % n)
    if y is None:
        y = torch.empty(batch, L, di, dtype=x.dtype, device=x.device)
    h_out = torch.empty(batch, di, N, dtype=torch.float32, device=x.device) if want_state else None
    check(lib().jamba_selective_scan_static(_p(x), x.stride(1), _p(z), z.stride(1), _p(dt), dt.stride(1), _p(B),
                                            B.stride(1), _p(C), C.stride(1), _DT[B.dtype], _p(A), _p(D), _p(h0),
                                            _p(y), y.stride(1), _p(h_out), batch, L, di, N, _DT[x.dtype],
                                            _p(status), _stream(stream)))
    return y, h_out


def rmsnorm(x, w, eps=1e-6, out=None, stream=None):
    _cuda(x, w)
    _contig(x, "x")
    out = torch.empty_like(x) if out is None else out
    cols = x.shape[-1]
    check(lib().jamba_rmsnorm(_p(x), _p(w), _p(out), x.numel() // cols, cols, float(eps), _DT[x.dtype],
                              _stream(stream)))
    return out


def causal_conv1d(x, w, b, state_in=None, want_state=True, stream=None):
    """x [batch, L, C] (row stride from the tensor) -> (SiLU(conv), state_out)."""
    _cuda(x, w, b, state_in)
    batch, L, C = x.shape
    out = torch.empty(batch, L, C, dtype=x.dtype, device=x.device)
    st = torch.empty(batch, C, 3, dtype=torch.float32, device=x.device) if want_state else None
    check(lib().jamba_causal_conv1d(_p(x), x.stride(1), _p(w), _p(b), _p(out), _p(state_in), _p(st), batch, L,
                                    C, _DT[x.dtype], _stream(stream)))
    return out, st


def in_proj_conv1d(u, w_in, conv_w, conv_b, state_in=None, state_out=None, xz=None, xc=None, stream=None):
    """bf16 u [batch, L, d_model] -> (xc [batch, L, d_inner] = SiLU(conv(x)),
    xz [batch, L, 2 d_inner] with z in its second half, state_out): in_proj
    with the conv in its epilogue."""
    _cuda(u, w_in, conv_w, conv_b, state_in, state_out, xz, xc)
    _contig(u, "u")
    _contig(w_in, "w_in")
    batch, L, dm = u.shape
    di = w_in.shape[0] // 2
    xz = torch.empty(batch, L, 2 * di, dtype=u.dtype, device=u.device) if xz is None else xz
    xc = torch.empty(batch, L, di, dtype=u.dtype, device=u.device) if xc is None else xc
    _contig(xz, "xz")
    _contig(xc, "xc")
    check(lib().jamba_in_proj_conv1d(_p(u), _p(w_in), _p(conv_w), _p(conv_b), _p(xz), _p(xc), _p(state_in),
                                     _p(state_out), batch, L, dm, di, _stream(stream)))
    return xc, xz, state_out


def gemm(a, b, residual=None, out_dtype=None, out=None, stream=None):
    """a [m, k] @ b[n, k]^T (+ residual) on the tensor cores (bf16) or CUDA cores (fp32)."""
    _cuda(a, b, residual, out)
    _contig(a, "a")
    _contig(b, "b")
    m, k = a.shape
    n = b.shape[0]
    od = out.dtype if out is not None else (out_dtype or a.dtype)
    if out is None:
        out = torch.empty(m, n, dtype=od, device=a.device)
    _contig(out, "out")
    check(lib().jamba_gemm(_p(a), _p(b), _p(out), n, _p(residual), m, n, k, _DT[a.dtype], _DT[od],
                           _stream(stream)))
    return out


def quantize_int8_rows(w, stream=None):
    """ExpertsInt8 codes of w [..., cols] (bf16 or fp32, CUDA): (q int8 like w, scale fp32 [...])."""
    _cuda(w)
    _contig(w, "w")
    cols = w.shape[-1]
    rows = w.numel() // cols
    q = torch.empty(w.shape, dtype=torch.int8, device=w.device)
    s = torch.empty(w.shape[:-1], dtype=torch.float32, device=w.device)
    check(lib().jamba_quantize_int8_rows(_p(w), _DT[w.dtype], rows, cols, _p(q), _p(s), _stream(stream)))
    return q, s


def quantize_experts_int8(params, stream=None):
    """MoE parameters with the expert matrices replaced by ExpertsInt8 codes
    (w_gate -> int8 codes + s_gate, ...); the router is kept as it is."""
    out = {"router": params["router"]}
    for k in ("gate", "up", "down"):
        out["w_" + k], out["s_" + k] = quantize_int8_rows(params["w_" + k].contiguous(), stream)
    return out


class MoE:
    """Top-K SwiGLU mixture of experts over borrowed weights.

    params: router, w_gate, w_up, w_down (bf16); with int8 expert matrices
    (ExpertsInt8, see quantize_experts_int8) also s_gate, s_up, s_down.
    """

    def __init__(self, params, shape):
        self.shape = shape
        self.params = {k: v.contiguous() for k, v in params.items()}
        _cuda(*self.params.values())
        int8 = self.params["w_gate"].dtype == torch.int8
        if int8 and not all(("s_" + k) in self.params for k in ("gate", "up", "down")):
            raise ValueError("int8 expert weights need s_gate, s_up and s_down")
        self.cfg = _abi.MoeConfig(shape.d_model, shape.d_ff, shape.n_experts, shape.top_k, _abi.JAMBA_BF16,
                                  _abi.JAMBA_INT8 if int8 else _abi.JAMBA_BF16)
        self.w = _abi.MoeWeights(*[_p(self.params.get(k)) for k in
                                   ("router", "w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down")])
        self.ws = _Workspace()

    def workspace_size(self, tokens):
        n = ctypes.c_size_t()
        check(lib().jamba_moe_workspace_size(ctypes.byref(self.cfg), tokens, ctypes.byref(n)))
        return n.value

    def forward(self, x, residual=None, out=None, stream=None):
        """x [T, d_model] -> dict(out, idx, w, offsets, perm)."""
        _cuda(x, residual)
        _contig(x, "x")
        T = x.shape[0]
        K, E = self.shape.top_k, self.shape.n_experts
        dev = x.device
        out = torch.empty_like(x) if out is None else out
        idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        w = torch.empty(T, K, dtype=torch.float32, device=dev)
        offs = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(T * K, dtype=torch.int32, device=dev)
        ws = self.ws.get(self.workspace_size(T), dev)
        check(lib().jamba_moe_forward(ctypes.byref(self.cfg), ctypes.byref(self.w), _p(x), _p(residual),
                                      _p(out), T, _p(idx), _p(w), _p(offs), _p(perm), _p(ws), ws.numel(),
                                      _stream(stream)))
        return dict(out=out, idx=idx, w=w, offsets=offs, perm=perm)


class Attention:
    """GQA attention layer (prefill and one-token decode) over borrowed weights.

    params: wq [n_heads*head_dim, d_model], wk and wv [n_kv_heads*head_dim,
    d_model], wo [d_model, n_heads*head_dim]; the q|k|v rows are stacked once
    into the fused w_qkv the library takes.
    """

    def __init__(self, params, shape):
        self.shape = shape
        _cuda(*params.values())
        self.w_qkv = torch.cat([params["wq"], params["wk"], params["wv"]], dim=0).contiguous()
        self.w_o = params["wo"].contiguous()
        self.cfg = _abi.AttnConfig(shape.d_model, shape.n_heads, shape.n_kv_heads, shape.head_dim,
                                   _DT[self.w_o.dtype])
        self.w = _abi.AttnWeights(_p(self.w_qkv), _p(self.w_o))
        self.ws = _Workspace()

    def new_cache(self, batch, max_len, device=None):
        """Zeroed K and V caches [batch, n_kv_heads, max_len, head_dim] and int32 lengths [batch]."""
        dev = device if device is not None else self.w_o.device
        sh = (batch, self.shape.n_kv_heads, max_len, self.shape.head_dim)
        return (torch.zeros(sh, dtype=self.w_o.dtype, device=dev), torch.zeros(sh, dtype=self.w_o.dtype, device=dev),
                torch.zeros(batch, dtype=torch.int32, device=dev))

    def prefill(self, x, residual=None, out=None, k_cache=None, v_cache=None, stream=None):
        """x [B, L, d_model] -> out; k_cache / v_cache (optional) receive positions 0..L-1."""
        _cuda(x, residual, out, k_cache, v_cache)
        _contig(x, "x")
        B, L, _ = x.shape
        out = torch.empty_like(x) if out is None else out
        max_len = k_cache.shape[2] if k_cache is not None else 0
        n = ctypes.c_size_t()
        check(lib().jamba_attn_prefill_workspace_size(ctypes.byref(self.cfg), B, L, ctypes.byref(n)))
        ws = self.ws.get(n.value, x.device)
        check(lib().jamba_attn_prefill(ctypes.byref(self.cfg), ctypes.byref(self.w), _p(x), _p(residual), _p(out),
                                       B, L, _p(k_cache), _p(v_cache), max_len, _p(ws), ws.numel(),
                                       _stream(stream)))
        return out

    def step(self, x, k_cache, v_cache, lengths, residual=None, out=None, stream=None):
        """x [B, d_model] at position lengths[b]; appends to the caches and advances lengths."""
        _cuda(x, k_cache, v_cache, lengths, residual, out)
        _contig(x, "x")
        if lengths.dtype != torch.int32:
            raise ValueError("lengths must be int32")
        B = x.shape[0]
        out = torch.empty_like(x) if out is None else out
        max_len = k_cache.shape[2]
        n = ctypes.c_size_t()
        check(lib().jamba_attn_step_workspace_size(ctypes.byref(self.cfg), B, max_len, ctypes.byref(n)))
        ws = self.ws.get(n.value, x.device)
        check(lib().jamba_attn_step(ctypes.byref(self.cfg), ctypes.byref(self.w), _p(x), _p(residual), _p(out), B,
                                    _p(k_cache), _p(v_cache), max_len, _p(lengths), _p(ws), ws.numel(),
                                    _stream(stream)))
        return out


def layer_pair(mixer, moe, x, g1, g2, eps=1e-6, stream=None):
    """RMSNorm -> Mamba -> residual -> RMSNorm -> MoE -> residual on x [B, L, d_model]."""
    B, L, dm = x.shape
    u = rmsnorm(x, g1, eps, stream=stream)
    h, _, _ = mixer.prefill(u, residual=x, stream=stream)
    v = rmsnorm(h, g2, eps, stream=stream)
    r = moe.forward(v.view(B * L, dm), residual=h.view(B * L, dm), stream=stream)
    r["h"] = h
    return r
