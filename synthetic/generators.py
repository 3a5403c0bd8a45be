"""Seeded random draws for every workload.

Recipe (one torch.Generator per call, seeded explicitly; draws in the order
listed; fp32 samples rounded to bf16 round-to-nearest-even where the
workload stores bf16):

* Mamba parameters, in this order: in_proj [2*d_inner, d_model],
  conv weight [d_inner, d_conv], conv bias [d_inner], x_proj
  [dt_rank + 2*d_state, d_inner], dt_proj [d_inner, dt_rank], all N(0, 0.02);
  then dt0 = exp(U[ln 1e-3, ln 1e-1]) per channel and dt_bias =
  dt0 + log(-expm1(-dt0)) (the inverse of softplus, so softplus(dt_bias) is
  log-uniform in [1e-3, 1e-1]); then out_proj [d_model, d_inner] N(0, 0.02).
  A[c, n] = -(n + 1), D = 1 and the inner-norm weights = 1 unless a test
  asks for randomised ones (drawn after the above, same generator).
* Mixer input u ~ N(0, 1), from its own generator (seed + 7919).
* Scan-only input: x, z, B, C ~ N(0, 1) in bf16; dt = softplus(N(-4, 1)) in
  fp32; A[c, n] = -(n + 1); D = 1.
* MoE: router [E, d_model], gate and up [E, d_ff, d_model], down
  [E, d_model, d_ff], all N(0, 0.02); input ~ N(0, 1).
* Attention: wq [n_heads*head_dim, d_model], wk and wv
  [n_kv_heads*head_dim, d_model], wo [d_model, n_heads*head_dim], all
  N(0, 0.02); input ~ N(0, 1).

dt_bias and the softplus of the scan-only dt are part of the input recipe
(how the benchmark initialises its tensors), not a step of the method.
Nothing here is computed by the method under test.
"""
import math

import torch

STD = 0.02


def _gen(seed, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(g, shape, std=1.0, mean=0.0, device="cpu"):
    t = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t


def _store(t, dtype):
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t.float()
    raise ValueError(dtype)


def mamba_params(shape, seed=0, device="cpu", a_init="structured",
                 norm_init="ones", d_init="ones"):
    """Parameters of one Mamba mixer, as the dict the C-ABI weights struct mirrors."""
    g = _gen(seed, device)
    di, dm, N, K, R = shape.d_inner, shape.d_model, shape.d_state, shape.d_conv, shape.dt_rank
    dt = shape.dtype
    p = {}
    p["in_proj"] = _store(_normal(g, (2 * di, dm), STD, device=device), dt)
    p["conv_w"] = _store(_normal(g, (di, K), STD, device=device), dt)
    p["conv_b"] = _store(_normal(g, (di,), STD, device=device), dt)
    p["x_proj"] = _store(_normal(g, (R + 2 * N, di), STD, device=device), dt)
    p["dt_proj"] = _store(_normal(g, (di, R), STD, device=device), dt)
    u = torch.rand(di, generator=g, dtype=torch.float64, device=device)
    dt0 = torch.exp(math.log(1e-3) + u * (math.log(1e-1) - math.log(1e-3)))
    p["dt_bias"] = (dt0 + torch.log(-torch.expm1(-dt0))).float()
    p["out_proj"] = _store(_normal(g, (dm, di), STD, device=device), dt)
    n1 = torch.arange(1, N + 1, dtype=torch.float32, device=device)
    if a_init == "structured":
        p["A"] = (-n1).expand(di, N).contiguous()
    elif a_init == "random":
        # independent negative rates per (channel, state)
        p["A"] = -torch.exp(_normal(g, (di, N), 0.5, device=device)) * n1
    else:
        raise ValueError(a_init)
    if d_init == "ones":
        p["D"] = torch.ones(di, dtype=torch.float32, device=device)
    else:
        p["D"] = 1.0 + _normal(g, (di,), 0.5, device=device)
    if norm_init == "ones":
        p["norm_dt"] = torch.ones(R, dtype=torch.float32, device=device)
        p["norm_B"] = torch.ones(N, dtype=torch.float32, device=device)
        p["norm_C"] = torch.ones(N, dtype=torch.float32, device=device)
    else:
        p["norm_dt"] = 1.0 + _normal(g, (R,), 0.2, device=device)
        p["norm_B"] = 1.0 + _normal(g, (N,), 0.2, device=device)
        p["norm_C"] = 1.0 + _normal(g, (N,), 0.2, device=device)
    return p


def mamba_input(shape, batch, seqlen, seed=0, device="cpu"):
    g = _gen(seed + 7919, device)
    return _store(_normal(g, (batch, seqlen, shape.d_model), device=device), shape.dtype)


def decode_inputs(shape, batch, steps, seed=0, device="cpu"):
    """Per-step decode tokens u_t ~ N(0, 1): [steps, batch, d_model]."""
    g = _gen(seed + 104729, device)
    return _store(_normal(g, (steps, batch, shape.d_model), device=device), shape.dtype)


def scan_inputs(batch, seqlen, d_inner, d_state=16, seed=0, device="cpu",
                dtype="bf16", a_init="structured", dt_mean=-4.0):
    g = _gen(seed, device)
    sh = (batch, seqlen, d_inner)
    x = _store(_normal(g, sh, device=device), dtype)
    z = _store(_normal(g, sh, device=device), dtype)
    B = _store(_normal(g, (batch, seqlen, d_state), device=device), dtype)
    C = _store(_normal(g, (batch, seqlen, d_state), device=device), dtype)
    dt = torch.nn.functional.softplus(_normal(g, sh, 1.0, dt_mean, device=device))
    n1 = torch.arange(1, d_state + 1, dtype=torch.float32, device=device)
    if a_init == "structured":
        A = (-n1).expand(d_inner, d_state).contiguous()
    else:
        A = -torch.exp(_normal(g, (d_inner, d_state), 0.5, device=device)) * n1
    D = torch.ones(d_inner, dtype=torch.float32, device=device)
    return dict(x=x, z=z, dt=dt.float(), B=B, C=C, A=A, D=D)


def moe_params(shape, seed=0, device="cpu"):
    g = _gen(seed + 31337, device)
    E, dm, dff = shape.n_experts, shape.d_model, shape.d_ff
    dt = shape.dtype
    return dict(
        router=_store(_normal(g, (E, dm), STD, device=device), dt),
        w_gate=_store(_normal(g, (E, dff, dm), STD, device=device), dt),
        w_up=_store(_normal(g, (E, dff, dm), STD, device=device), dt),
        w_down=_store(_normal(g, (E, dm, dff), STD, device=device), dt),
    )


def moe_input(shape, tokens, seed=0, device="cpu"):
    g = _gen(seed + 65537, device)
    return _store(_normal(g, (tokens, shape.d_model), device=device), shape.dtype)


def attn_params(shape, seed=0, device="cpu"):
    g = _gen(seed + 271828, device)
    H, G, D, dm = shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.d_model
    dt = shape.dtype
    return dict(
        wq=_store(_normal(g, (H * D, dm), STD, device=device), dt),
        wk=_store(_normal(g, (G * D, dm), STD, device=device), dt),
        wv=_store(_normal(g, (G * D, dm), STD, device=device), dt),
        wo=_store(_normal(g, (dm, H * D), STD, device=device), dt),
    )


def attn_input(shape, batch, seqlen, seed=0, device="cpu"):
    g = _gen(seed + 314159, device)
    return _store(_normal(g, (batch, seqlen, shape.d_model), device=device), shape.dtype)


def block_norm_params(d_model, seed=0, device="cpu", init="ones"):
    """Weights of the two block RMSNorms around the mixer and the MoE."""
    if init == "ones":
        return (torch.ones(d_model, device=device), torch.ones(d_model, device=device))
    g = _gen(seed + 271828, device)
    return (1.0 + _normal(g, (d_model,), 0.2, device=device),
            1.0 + _normal(g, (d_model,), 0.2, device=device))
