"""fp64 oracle of the Mamba mixer (prefill and one-token decode).

TEST INFRASTRUCTURE: see the package header for who may import this.

The Jamba paper (summary page "Jamba: A Hybrid Transformer-Mamba Language
Model", section 2) builds its Mamba layers on the selective state-space layer
of its ref [17] and adds RMSNorm inside the layer (section 2 and section 6.4,
figure 9).  The layer computed here, with u of shape [batch, L, d_model]:

  xz       = u W_in^T                         x = xz[..., :d_inner], z = xz[..., d_inner:]
  xc       = SiLU(conv_b + sum_k conv_w[:, k] * x[t - (d_conv-1) + k])   (causal, depthwise)
  p        = xc W_x^T                         dt_low, B, C = split(p, [dt_rank, d_state, d_state])
  (inner RMSNorm, when enabled, on dt_low, on B and on C separately)
  dt       = softplus(dt_low W_dt^T + dt_bias)
  h_t      = exp(dt_t A) * h_{t-1} + dt_t B_t x_t          (per channel c, state n)
  y_t      = (C_t . h_t + D x_t) * SiLU(z_t)
  out      = y W_out^T

Readings taken where the pages are silent (each listed in the design notes):
discretisation exp(dt A) for A and Euler dt*B*x for the input term; A given
directly (negative), not as a log; D multiplies the post-conv x; the conv is
a cross-correlation with d_conv-1 zeros (or the cache) on the left and the
last tap on the current token; the conv cache holds the last d_conv-1
pre-conv inputs, oldest first; the three inner norms use eps = 1e-6.

Parity pins (tests/test_oracle_pins.py): A = 0 cumulative-sum closed form,
brute-force unrolled sum for L <= 5, constant-input geometric series, C = 0,
linearity in x, a hand-worked three-step example (tests/golden), the chunked
associative form for several chunk sizes, conv delta kernels and
torch.nn.functional.conv1d, linear vs a pure-Python triple loop, RMSNorm and
softplus / SiLU identities, and decode step == prefill of L + 1.  The whole
composition is pinned by a three-token mixer example worked out by hand
(tests/golden/mixer_hand_example.json: every intermediate from the x|z split
to both caches, in closed form) and, inside the layer pair, by the same
layer written with scalar Python loops.
"""
import numpy as np


def to64(t):
    """torch tensor (any dtype, any device) or array -> float64 numpy."""
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu").double().numpy()


def silu(v):
    return v / (1.0 + np.exp(-v))


def softplus(v):
    # log(1 + e^v), evaluated without overflow
    return np.logaddexp(0.0, v)


def rmsnorm(x, w, eps):
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * w."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * w


def linear(x, W):
    """x [..., K] times W [N, K]^T."""
    return x @ W.T


def causal_conv1d(x, w, b, state0=None):
    """Depthwise causal conv along time, before the activation.

    x [B, L, C]; w [C, K]; b [C]; state0 [B, C, K-1] (oldest first) or None
    for zeros.  Returns (out [B, L, C], new_state [B, C, K-1]).
    """
    Bsz, L, Cn = x.shape
    K = w.shape[1]
    if state0 is None:
        state0 = np.zeros((Bsz, Cn, K - 1))
    xpad = np.concatenate([np.transpose(state0, (0, 2, 1)), x], axis=1)  # [B, L+K-1, C]
    out = np.broadcast_to(b, (Bsz, L, Cn)).copy()
    for k in range(K):
        out += w[:, k] * xpad[:, k:k + L, :]
    new_state = np.transpose(xpad[:, L:L + K - 1, :], (0, 2, 1)).copy()
    return out, new_state


def selective_scan(x, dt, A, Bm, Cm, D, z=None, h0=None):
    """Sequential selective scan with D skip and SiLU(z) gate.

    x, dt, z: [B, L, C]; A: [C, N]; Bm, Cm: [B, L, N]; D: [C];
    h0: [B, C, N] or None (zeros).  Returns (y [B, L, C], h_L [B, C, N]).
    """
    Bsz, L, Cn = x.shape
    N = A.shape[1]
    h = np.zeros((Bsz, Cn, N)) if h0 is None else np.array(h0, dtype=np.float64)
    y = np.empty((Bsz, L, Cn))
    for t in range(L):
        d = dt[:, t, :, None]                                   # [B, C, 1]
        h = np.exp(d * A[None]) * h + d * Bm[:, t, None, :] * x[:, t, :, None]
        y[:, t] = np.einsum("bcn,bn->bc", h, Cm[:, t]) + D * x[:, t]
    if z is not None:
        y = y * silu(z)
    return y, h


def selective_scan_chunked(x, dt, A, Bm, Cm, D, z=None, h0=None, chunk=64):
    """The same scan evaluated chunk by chunk with the associative carry.

    Each chunk is scanned from a zero state, giving local outputs, the local
    end state and the chunk's decay products P_t = prod exp(dt A); chunks are
    then chained with (P2, h2) o (P1, h1) = (P2 P1, P2 h1 + h2) and every
    local output gets the carried-in term C_t . (P_t * h_in).
    """
    Bsz, L, Cn = x.shape
    N = A.shape[1]
    h_in = np.zeros((Bsz, Cn, N)) if h0 is None else np.array(h0, dtype=np.float64)
    y = np.empty((Bsz, L, Cn))
    for s in range(0, L, chunk):
        e = min(L, s + chunk)
        h = np.zeros((Bsz, Cn, N))
        P = np.ones((Bsz, Cn, N))
        for t in range(s, e):
            d = dt[:, t, :, None]
            a = np.exp(d * A[None])
            h = a * h + d * Bm[:, t, None, :] * x[:, t, :, None]
            P = a * P
            y_loc = np.einsum("bcn,bn->bc", h, Cm[:, t])
            carry = np.einsum("bcn,bn->bc", P * h_in, Cm[:, t])
            y[:, t] = y_loc + carry + D * x[:, t]
        h_in = P * h_in + h
    if z is not None:
        y = y * silu(z)
    return y, h_in


def selective_scan_c(x, dt, A, Bm, Cm, D, z=None, h0=None):
    """selective_scan() through the plain C loop in scan_seq.c (long L)."""
    from . import native
    return native.scan(x, dt, A, Bm, Cm, D, z, h0)


def params64(p):
    return {k: to64(v) for k, v in p.items()}


def mamba_prefill(p, u, shape, conv_state0=None, ssm_state0=None, scan="numpy",
                  keep=False):
    """Mamba mixer over a whole sequence.

    p: parameter dict (float64 arrays, see params64); u: [B, L, d_model].
    Returns dict(out, conv_state [B, d_inner, d_conv-1], ssm_state
    [B, d_inner, d_state]) plus the intermediates when keep=True.
    """
    di, N, R = shape.d_inner, shape.d_state, shape.dt_rank
    xz = linear(u, p["in_proj"])
    x, z = xz[..., :di], xz[..., di:]
    xc_pre, conv_state = causal_conv1d(x, p["conv_w"], p["conv_b"], conv_state0)
    xc = silu(xc_pre)
    proj = linear(xc, p["x_proj"])
    dt_low, Bm, Cm = proj[..., :R], proj[..., R:R + N], proj[..., R + N:R + 2 * N]
    if shape.inner_norm:
        dt_low = rmsnorm(dt_low, p["norm_dt"], shape.eps)
        Bm = rmsnorm(Bm, p["norm_B"], shape.eps)
        Cm = rmsnorm(Cm, p["norm_C"], shape.eps)
    dt = softplus(linear(dt_low, p["dt_proj"]) + p["dt_bias"])
    scan_fn = {"numpy": selective_scan, "c": selective_scan_c}[scan]
    y, h = scan_fn(xc, dt, p["A"], Bm, Cm, p["D"], z, ssm_state0)
    out = linear(y, p["out_proj"])
    res = dict(out=out, conv_state=conv_state, ssm_state=h)
    if keep:
        res.update(xz=xz, xc=xc, proj=proj, dt_low=dt_low, B=Bm, C=Cm, dt=dt, y=y)
    return res


def mamba_step(p, u_t, shape, conv_state, ssm_state):
    """One-token decode: u_t [B, d_model] with the conv and ssm caches.

    The conv window is [cache (d_conv-1 oldest first), x_t]; the cache then
    drops its oldest entry and appends x_t.  The scan advances one step from
    the cached state.  Returns (out_t [B, d_model], conv_state', ssm_state').
    """
    di, N, R = shape.d_inner, shape.d_state, shape.dt_rank
    xz = linear(u_t, p["in_proj"])                        # [B, 2 d_inner]
    x, z = xz[:, :di], xz[:, di:]
    window = np.concatenate([conv_state, x[:, :, None]], axis=2)   # [B, C, d_conv]
    xc = silu(p["conv_b"] + np.sum(window * p["conv_w"][None], axis=2))
    new_conv = window[:, :, 1:].copy()
    proj = linear(xc, p["x_proj"])
    dt_low, Bm, Cm = proj[:, :R], proj[:, R:R + N], proj[:, R + N:R + 2 * N]
    if shape.inner_norm:
        dt_low = rmsnorm(dt_low, p["norm_dt"], shape.eps)
        Bm = rmsnorm(Bm, p["norm_B"], shape.eps)
        Cm = rmsnorm(Cm, p["norm_C"], shape.eps)
    dt = softplus(linear(dt_low, p["dt_proj"]) + p["dt_bias"])       # [B, C]
    h = np.exp(dt[:, :, None] * p["A"][None]) * ssm_state \
        + dt[:, :, None] * Bm[:, None, :] * xc[:, :, None]
    y = (np.einsum("bcn,bn->bc", h, Cm) + p["D"] * xc) * silu(z)
    return linear(y, p["out_proj"]), new_conv, h
