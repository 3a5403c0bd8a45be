"""Pins the fp64 oracle to facts that do not come from the oracle itself.

Closed forms, brute force on tiny inputs, hand-worked examples from
tests/golden and identities of the mathematics.  Each check is chosen so that
a plausible slip in the oracle (a dropped term, a wrong sign or index, a
transposed operand) fails it.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import mamba as om
from oracle import moe as omoe
from oracle import native
from synthetic import MambaShape, mamba_params, mamba_input

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand_scan(rng, B=2, L=9, C=5, N=4, a_neg=True):
    x = rng.standard_normal((B, L, C))
    dt = np.log1p(np.exp(rng.standard_normal((B, L, C)) - 2.0))
    A = -np.exp(rng.standard_normal((C, N))) if a_neg else rng.standard_normal((C, N))
    Bm = rng.standard_normal((B, L, N))
    Cm = rng.standard_normal((B, L, N))
    D = rng.standard_normal(C)
    z = rng.standard_normal((B, L, C))
    return x, dt, A, Bm, Cm, D, z


# ----------------------------------------------------------------- scan pins

def test_scan_hand_example():
    g = _golden("scan_hand_example.json")
    ln2 = math.log(2.0)
    x = np.array(g["x"])[None, :, None]
    L = x.shape[1]
    dt = np.full((1, L, 1), ln2)
    A = np.array(g["A"])[None, :]
    Bm = np.tile(np.array(g["B"]), (1, L, 1))
    Cm = np.tile(np.array(g["C"]), (1, L, 1))
    D = np.array([g["D"]])
    want = np.array(g["y_ln2_coef"]) * ln2 + np.array(g["y_const"])
    want_h = np.array(g["h_last_ln2_coef"]) * ln2
    for fn in (om.selective_scan, om.selective_scan_c):
        y, h = fn(x, dt, A, Bm, Cm, D)
        np.testing.assert_allclose(y[0, :, 0], want, rtol=1e-14)
        np.testing.assert_allclose(h[0, 0], want_h, rtol=1e-14)


def test_scan_A_zero_is_cumsum():
    rng = np.random.default_rng(1)
    x, dt, A, Bm, Cm, D, z = _rand_scan(rng)
    A = np.zeros_like(A)
    # h_t[c, n] = sum_{s<=t} dt_s[c] B_s[n] x_s[c]
    contrib = dt[..., None] * Bm[:, :, None, :] * x[..., None]      # [B, L, C, N]
    hcum = np.cumsum(contrib, axis=1)
    want = (np.einsum("blcn,bln->blc", hcum, Cm) + D * x) * (z / (1 + np.exp(-z)))
    for fn in (om.selective_scan, om.selective_scan_c):
        y, h = fn(x, dt, A, Bm, Cm, D, z)
        np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(h, hcum[:, -1], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("L", [1, 2, 3, 5])
def test_scan_bruteforce_unrolled(L):
    """y_t = sum_{s<=t} sum_n C_t[n] (prod_{r=s+1..t} e^{dt_r A_n}) dt_s B_s[n] x_s + D x_t."""
    rng = np.random.default_rng(10 + L)
    x, dt, A, Bm, Cm, D, z = _rand_scan(rng, B=1, L=L, C=3, N=3)
    want = np.zeros((1, L, 3))
    for c in range(3):
        for t in range(L):
            acc = 0.0
            for s in range(t + 1):
                for n in range(3):
                    decay = 1.0
                    for r in range(s + 1, t + 1):
                        decay *= math.exp(dt[0, r, c] * A[c, n])
                    acc += Cm[0, t, n] * decay * dt[0, s, c] * Bm[0, s, n] * x[0, s, c]
            want[0, t, c] = acc + D[c] * x[0, t, c]
    for fn in (om.selective_scan, om.selective_scan_c):
        y, _ = fn(x, dt, A, Bm, Cm, D)
        np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-13)


def test_scan_constant_input_geometric_series():
    L, C, N = 40, 2, 3
    dtv, xv = 0.3, 1.7
    A = np.array([[-0.5, -1.0, -2.0], [-0.1, -0.2, -3.0]])
    Bv = np.array([0.4, -1.1, 2.0])
    x = np.full((1, L, C), xv)
    dt = np.full((1, L, C), dtv)
    Bm = np.tile(Bv, (1, L, 1))
    Cm = np.tile(np.array([1.0, 0.0, 0.0]), (1, L, 1))
    D = np.zeros(C)
    _, h = om.selective_scan(x, dt, A, Bm, Cm, D)
    a = np.exp(dtv * A)                                   # [C, N]
    want = dtv * Bv[None] * xv * (1 - a ** L) / (1 - a)
    np.testing.assert_allclose(h[0], want, rtol=1e-13)


def test_scan_C_zero_gives_skip_times_gate():
    rng = np.random.default_rng(3)
    x, dt, A, Bm, Cm, D, z = _rand_scan(rng)
    y, _ = om.selective_scan(x, dt, A, Bm, np.zeros_like(Cm), D, z)
    np.testing.assert_allclose(y, D * x * z / (1 + np.exp(-z)), rtol=1e-14)


def test_scan_linear_in_x():
    rng = np.random.default_rng(4)
    x, dt, A, Bm, Cm, D, z = _rand_scan(rng)
    x2 = rng.standard_normal(x.shape)
    y1, h1 = om.selective_scan(x, dt, A, Bm, Cm, D, z)
    y2, h2 = om.selective_scan(x2, dt, A, Bm, Cm, D, z)
    y3, h3 = om.selective_scan(2.0 * x - 3.0 * x2, dt, A, Bm, Cm, D, z)
    np.testing.assert_allclose(y3, 2.0 * y1 - 3.0 * y2, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(h3, 2.0 * h1 - 3.0 * h2, rtol=1e-11, atol=1e-11)


def test_scan_initial_state_is_zero_input_prefix():
    """Starting from h0 equals scanning a prefix that produced h0."""
    rng = np.random.default_rng(5)
    x, dt, A, Bm, Cm, D, z = _rand_scan(rng, L=12)
    y_all, h_all = om.selective_scan(x, dt, A, Bm, Cm, D, z)
    _, h_mid = om.selective_scan(x[:, :5], dt[:, :5], A, Bm[:, :5], Cm[:, :5], D)
    y_tail, h_tail = om.selective_scan(x[:, 5:], dt[:, 5:], A, Bm[:, 5:], Cm[:, 5:], D,
                                       z[:, 5:], h0=h_mid)
    np.testing.assert_allclose(y_tail, y_all[:, 5:], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(h_tail, h_all, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("chunk", [1, 7, 64, 300])
def test_scan_chunked_equals_sequential(chunk):
    rng = np.random.default_rng(6)
    x, dt, A, Bm, Cm, D, z = _rand_scan(rng, B=2, L=150, C=4, N=16)
    h0 = rng.standard_normal((2, 4, 16))
    y1, h1 = om.selective_scan(x, dt, A, Bm, Cm, D, z, h0)
    y2, h2 = om.selective_scan_chunked(x, dt, A, Bm, Cm, D, z, h0, chunk=chunk)
    np.testing.assert_allclose(y2, y1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(h2, h1, rtol=1e-12, atol=1e-12)


def test_scan_c_matches_numpy_on_random():
    rng = np.random.default_rng(7)
    x, dt, A, Bm, Cm, D, z = _rand_scan(rng, B=2, L=64, C=6, N=16)
    h0 = rng.standard_normal((2, 6, 16))
    y1, h1 = om.selective_scan(x, dt, A, Bm, Cm, D, z, h0)
    y2, h2 = native.scan(x, dt, A, Bm, Cm, D, z, h0)
    np.testing.assert_allclose(y2, y1, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(h2, h1, rtol=1e-13, atol=1e-13)


# ----------------------------------------------------------------- conv pins

def test_conv_hand_example():
    g = _golden("conv_hand_example.json")
    x = np.array(g["x"])[None, :, None]
    w = np.array(g["w"])[None, :]
    out, st = om.causal_conv1d(x, w, np.array([g["b"]]))
    np.testing.assert_allclose(out[0, :, 0], g["out_pre_activation"], rtol=0, atol=0)
    np.testing.assert_allclose(st[0, 0], g["state_after"], rtol=0, atol=0)


def test_conv_delta_kernels():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((2, 10, 3))
    ident = np.tile([0.0, 0.0, 0.0, 1.0], (3, 1))
    out, _ = om.causal_conv1d(x, ident, np.zeros(3))
    np.testing.assert_array_equal(out, x)
    shift = np.tile([1.0, 0.0, 0.0, 0.0], (3, 1))
    out, st = om.causal_conv1d(x, shift, np.zeros(3))
    np.testing.assert_array_equal(out[:, 3:], x[:, :-3])
    np.testing.assert_array_equal(out[:, :3], 0.0)
    np.testing.assert_array_equal(st, np.transpose(x[:, -3:], (0, 2, 1)))


def test_conv_vs_torch_conv1d():
    rng = np.random.default_rng(9)
    B, L, C, K = 2, 17, 5, 4
    x = rng.standard_normal((B, L, C))
    w = rng.standard_normal((C, K))
    b = rng.standard_normal(C)
    out, _ = om.causal_conv1d(x, w, b)
    t = torch.nn.functional.conv1d(torch.from_numpy(x).permute(0, 2, 1),
                                   torch.from_numpy(w)[:, None, :], torch.from_numpy(b),
                                   padding=K - 1, groups=C)[..., :L]
    np.testing.assert_allclose(out, t.permute(0, 2, 1).numpy(), rtol=1e-13, atol=1e-13)


def test_conv_state_continues_sequence():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((1, 9, 4))
    w = rng.standard_normal((4, 4))
    b = rng.standard_normal(4)
    full, st_full = om.causal_conv1d(x, w, b)
    a, st = om.causal_conv1d(x[:, :2], w, b)         # shorter than the window
    rest, st2 = om.causal_conv1d(x[:, 2:], w, b, st)
    np.testing.assert_allclose(np.concatenate([a, rest], 1), full, rtol=1e-14)
    np.testing.assert_array_equal(st2, st_full)


# ------------------------------------------------------ elementwise and norms

def test_linear_vs_triple_loop():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((3, 4))
    W = rng.standard_normal((5, 4))
    want = [[sum(x[i, k] * W[j, k] for k in range(4)) for j in range(5)] for i in range(3)]
    np.testing.assert_allclose(om.linear(x, W), np.array(want), rtol=1e-14)
    np.testing.assert_array_equal(om.linear(x, np.eye(4)), x)


def test_rmsnorm_identities():
    rng = np.random.default_rng(13)
    w = rng.standard_normal(8)
    c = np.full((2, 8), -3.5)                       # constant vector -> w * sign
    np.testing.assert_allclose(om.rmsnorm(c, w, 0.0), -np.tile(w, (2, 1)), rtol=1e-15)
    x = rng.standard_normal((3, 8))
    np.testing.assert_allclose(om.rmsnorm(7.0 * x, w, 0.0), om.rmsnorm(x, w, 0.0), rtol=1e-14)
    # unit weights: mean of squares of the output is 1
    y = om.rmsnorm(x, np.ones(8), 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-14)
    # eps enters under the root
    e = 0.25
    np.testing.assert_allclose(om.rmsnorm(x, np.ones(8), e),
                               x / np.sqrt(np.mean(x * x, -1, keepdims=True) + e), rtol=1e-15)


def test_softplus_silu_identities():
    v = np.linspace(-30, 30, 61)
    sp = om.softplus(v)
    np.testing.assert_allclose(sp, [math.log1p(math.exp(t)) for t in v], rtol=1e-14)
    np.testing.assert_allclose(sp - om.softplus(-v), v, rtol=1e-13, atol=1e-13)
    assert om.softplus(np.array([0.0]))[0] == pytest.approx(math.log(2.0), rel=1e-15)
    s = om.silu(v)
    np.testing.assert_allclose(s - om.silu(-v), v, rtol=1e-13, atol=1e-13)
    assert om.silu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(s, [t / (1 + math.exp(-t)) for t in v], rtol=1e-14)


# --------------------------------------------------------------- mixer pins

def _tiny_shape(inner_norm):
    return MambaShape(d_model=8, d_inner=12, d_state=16, d_conv=4, dt_rank=3,
                      dtype="f32", inner_norm=inner_norm)


@pytest.mark.parametrize("inner_norm", [False, True])
def test_step_equals_prefill_of_L_plus_1(inner_norm):
    sh = _tiny_shape(inner_norm)
    p = om.params64(mamba_params(sh, seed=3, a_init="random", norm_init="random",
                                 d_init="random"))
    u = om.to64(mamba_input(sh, batch=2, seqlen=10, seed=3))
    full = om.mamba_prefill(p, u, sh)
    part = om.mamba_prefill(p, u[:, :7], sh)
    cs, ss = part["conv_state"], part["ssm_state"]
    for t in range(7, 10):
        o, cs, ss = om.mamba_step(p, u[:, t], sh, cs, ss)
        np.testing.assert_allclose(o, full["out"][:, t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(cs, full["conv_state"], rtol=1e-14)
    np.testing.assert_allclose(ss, full["ssm_state"], rtol=1e-12, atol=1e-13)


def test_prefill_continues_from_states():
    sh = _tiny_shape(True)
    p = om.params64(mamba_params(sh, seed=4))
    u = om.to64(mamba_input(sh, batch=1, seqlen=12, seed=4))
    full = om.mamba_prefill(p, u, sh)
    a = om.mamba_prefill(p, u[:, :5], sh)
    b = om.mamba_prefill(p, u[:, 5:], sh, a["conv_state"], a["ssm_state"])
    np.testing.assert_allclose(b["out"], full["out"][:, 5:], rtol=1e-12, atol=1e-13)


def test_prefill_step_order_by_hand():
    """The composed layer against the same steps written out with torch fp64."""
    sh = _tiny_shape(True)
    p = mamba_params(sh, seed=5, norm_init="random", d_init="random")
    u = mamba_input(sh, batch=1, seqlen=6, seed=5).double()[0]
    P = {k: v.double() for k, v in p.items()}
    di, N, R = sh.d_inner, sh.d_state, sh.dt_rank
    xz = u @ P["in_proj"].T
    x, z = xz[:, :di], xz[:, di:]
    conv = torch.nn.functional.conv1d(x.T[None], P["conv_w"][:, None, :], P["conv_b"],
                                      padding=3, groups=di)[0, :, :6].T
    xc = torch.nn.functional.silu(conv)
    pr = xc @ P["x_proj"].T
    rn = lambda a, w: a * torch.rsqrt((a * a).mean(-1, keepdim=True) + sh.eps) * w
    dtl, Bm, Cm = rn(pr[:, :R], P["norm_dt"]), rn(pr[:, R:R + N], P["norm_B"]), \
        rn(pr[:, R + N:], P["norm_C"])
    dt = torch.nn.functional.softplus(dtl @ P["dt_proj"].T + P["dt_bias"])
    h = torch.zeros(di, N, dtype=torch.float64)
    ys = []
    for t in range(6):
        h = torch.exp(dt[t, :, None] * P["A"]) * h + dt[t, :, None] * Bm[t][None] * xc[t, :, None]
        ys.append((h @ Cm[t] + P["D"] * xc[t]) * torch.nn.functional.silu(z[t]))
    want = torch.stack(ys) @ P["out_proj"].T
    got = om.mamba_prefill(om.params64(p), om.to64(u[None]), sh)["out"][0]
    np.testing.assert_allclose(got, want.numpy(), rtol=1e-12, atol=1e-13)


def _hand_value(expr):
    """Evaluates one hand-derived value of a golden file: numbers, ln2, ln3, + - * / and parentheses."""
    import ast
    names = {"ln2": math.log(2.0), "ln3": math.log(3.0)}
    ops = {ast.Add: lambda a, b: a + b, ast.Sub: lambda a, b: a - b,
           ast.Mult: lambda a, b: a * b, ast.Div: lambda a, b: a / b}

    def ev(n):
        if isinstance(n, ast.Expression):
            return ev(n.body)
        if isinstance(n, ast.Constant) and isinstance(n.value, (int, float)):
            return float(n.value)
        if isinstance(n, ast.Name) and n.id in names:
            return names[n.id]
        if isinstance(n, ast.UnaryOp) and isinstance(n.op, ast.USub):
            return -ev(n.operand)
        if isinstance(n, ast.BinOp) and type(n.op) in ops:
            return ops[type(n.op)](ev(n.left), ev(n.right))
        raise ValueError("not a hand value: " + expr)

    return ev(ast.parse(expr, mode="eval"))


def _hand_array(v):
    return np.vectorize(_hand_value, otypes=[np.float64])(np.array(v, dtype=object))


def test_mixer_hand_example():
    """The whole mixer on a worked example derived by hand step by step (tests/golden).

    Pins the wiring of the composition: which half of xz is x and which is z,
    the conv orientation and bias, SiLU after the conv, the [dt_low | B | C]
    split with a norm on each piece, dt_proj + dt_bias + softplus, the scan,
    D on the post-conv x, the SiLU(z) gate and out_proj, plus both caches.
    """
    g = _golden("mixer_hand_example.json")
    p = {k: _hand_array(v) for k, v in g["params"].items()}
    u = _hand_array(g["u"])[None]
    sh = MambaShape(d_model=2, d_inner=1, d_state=2, d_conv=4, dt_rank=2, dtype="f32",
                    inner_norm=True, eps=0.0)
    r = om.mamba_prefill(p, u, sh, keep=True)
    e = {k: _hand_array(v) for k, v in g["expect"].items()}
    close = dict(rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(r["xz"][0, :, 0], e["x"], **close)
    np.testing.assert_allclose(r["xz"][0, :, 1], e["z"], **close)
    np.testing.assert_allclose(r["xc"][0, :, 0], e["xc"], **close)
    np.testing.assert_allclose(r["dt_low"][0], e["dt_low"], **close)
    np.testing.assert_allclose(r["B"][0], e["B"], **close)
    np.testing.assert_allclose(r["C"][0], e["C"], **close)
    np.testing.assert_allclose(r["dt"][0, :, 0], e["dt"], **close)
    np.testing.assert_allclose(r["y"][0, :, 0], e["y"], **close)
    np.testing.assert_allclose(r["out"][0], e["out"], **close)
    np.testing.assert_allclose(r["conv_state"][0, 0], e["conv_state"], **close)
    np.testing.assert_allclose(r["ssm_state"][0, 0], e["ssm_state"], **close)
    # the sequential C loop reaches the same scan
    r_c = om.mamba_prefill(p, u, sh, scan="c")
    np.testing.assert_allclose(r_c["out"][0], e["out"], **close)
    # and decoding the three tokens one at a time from empty caches does too
    cs, ss = np.zeros((1, 1, 3)), np.zeros((1, 1, 2))
    for t in range(3):
        o, cs, ss = om.mamba_step(p, u[:, t], sh, cs, ss)
        np.testing.assert_allclose(o[0], e["out"][t], **close)
    np.testing.assert_allclose(ss[0, 0], e["ssm_state"], **close)


# ------------------------------------------------------------- layer-pair pins

def _py_layer_pair(mp, moe_p, x, R, N, K_top, g1, g2, eps):
    """Jamba layer pair with scalar Python loops only (no numpy arithmetic).

    RMSNorm -> Mamba mixer -> residual -> RMSNorm -> top-K softmax MoE of
    SwiGLU experts -> residual (summary page, section 2: pre-norm "standard"
    layers; RMSNorm on dt_low, B and C inside the mixer).  x: list of L
    token vectors; weights as nested lists.
    """
    dm = len(x[0])
    di = len(mp["conv_b"])
    K = len(mp["conv_w"][0])
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))

    def norm(v, w):
        r = math.sqrt(sum(a * a for a in v) / len(v) + eps)
        return [a / r * b for a, b in zip(v, w)]

    def mv(W, v):
        return [sum(W[i][j] * v[j] for j in range(len(v))) for i in range(len(W))]

    L = len(x)
    us = [norm(x[t], g1) for t in range(L)]
    xs, zs = [], []
    for t in range(L):
        xz = mv(mp["in_proj"], us[t])
        xs.append(xz[:di])
        zs.append(xz[di:])
    h = [[0.0] * N for _ in range(di)]
    hs = []
    for t in range(L):
        xc = []
        for c in range(di):
            acc = mp["conv_b"][c]
            for k in range(K):
                s = t - (K - 1) + k
                if s >= 0:
                    acc += mp["conv_w"][c][k] * xs[s][c]
            xc.append(acc * sig(acc))
        pr = mv(mp["x_proj"], xc)
        dtl = norm(pr[:R], mp["norm_dt"])
        Bv = norm(pr[R:R + N], mp["norm_B"])
        Cv = norm(pr[R + N:], mp["norm_C"])
        y = []
        for c in range(di):
            v = mp["dt_bias"][c] + sum(mp["dt_proj"][c][j] * dtl[j] for j in range(R))
            dt = math.log1p(math.exp(v))
            acc = mp["D"][c] * xc[c]
            for n in range(N):
                h[c][n] = math.exp(dt * mp["A"][c][n]) * h[c][n] + dt * Bv[n] * xc[c]
                acc += Cv[n] * h[c][n]
            y.append(acc * zs[t][c] * sig(zs[t][c]))
        mo = mv(mp["out_proj"], y)
        hs.append([x[t][i] + mo[i] for i in range(dm)])
    E = len(moe_p["router"])
    outs, idxs = [], []
    for t in range(L):
        v = norm(hs[t], g2)
        logits = mv(moe_p["router"], v)
        m = max(logits)
        ex = [math.exp(a - m) for a in logits]
        tot = sum(ex)
        order = sorted(range(E), key=lambda e: (-logits[e], e))[:K_top]
        o = list(hs[t])
        for e in order:
            gt = mv(moe_p["w_gate"][e], v)
            up = mv(moe_p["w_up"][e], v)
            act = [a * sig(a) * b for a, b in zip(gt, up)]
            dn = mv(moe_p["w_down"][e], act)
            o = [o[i] + ex[e] / tot * dn[i] for i in range(dm)]
        outs.append(o)
        idxs.append(order)
    return outs, hs, idxs


def test_layer_pair_vs_python_loops():
    """oracle.moe.layer_pair against the pair written with scalar loops (tiny case)."""
    sh = MambaShape(d_model=6, d_inner=8, d_state=3, d_conv=4, dt_rank=2, dtype="f32",
                    inner_norm=True)
    mp = om.params64(mamba_params(sh, seed=21, a_init="random", norm_init="random",
                                  d_init="random"))
    rng = np.random.default_rng(21)
    # larger weights than the init so every term moves the result
    for k in ("in_proj", "x_proj", "dt_proj", "out_proj", "conv_w", "conv_b"):
        mp[k] = mp[k] * 20.0
    E, dff = 16, 3
    moe_p = dict(router=rng.standard_normal((E, 6)), w_gate=rng.standard_normal((E, dff, 6)),
                 w_up=rng.standard_normal((E, dff, 6)), w_down=rng.standard_normal((E, 6, dff)))
    x = rng.standard_normal((1, 7, 6))
    g1 = 1.0 + 0.3 * rng.standard_normal(6)
    g2 = 1.0 + 0.3 * rng.standard_normal(6)
    r = omoe.layer_pair(mp, moe_p, x, sh, 2, g1, g2)
    tl = lambda a: np.asarray(a).tolist()
    outs, hs, idxs = _py_layer_pair({k: tl(v) for k, v in mp.items()},
                                    {k: tl(v) for k, v in moe_p.items()},
                                    tl(x[0]), sh.dt_rank, sh.d_state, 2, tl(g1), tl(g2), sh.eps)
    np.testing.assert_allclose(r["h"], np.array(hs), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r["out"], np.array(outs), rtol=1e-12, atol=1e-13)
    assert (r["idx"] == np.array(idxs)).all()
    # the Mamba half moved h away from x, and the MoE half moved out away from h
    assert np.abs(r["h"] - x[0]).max() > 1e-2 and np.abs(r["out"] - r["h"]).max() > 1e-2


def test_layer_pair_identical_experts_and_zero_mixer():
    """Closed forms of the pair: out_proj = 0 gives h = x; identical experts give
    out = h + (p_1 + p_2) f(RMSNorm(h)) with the two softmax weights of the router."""
    sh = MambaShape(d_model=6, d_inner=8, d_state=3, d_conv=4, dt_rank=2, dtype="f32")
    mp = om.params64(mamba_params(sh, seed=22))
    rng = np.random.default_rng(22)
    E, dff = 16, 5
    gt, up, dn = rng.standard_normal((dff, 6)), rng.standard_normal((dff, 6)), rng.standard_normal((6, dff))
    moe_p = dict(router=rng.standard_normal((E, 6)), w_gate=np.stack([gt] * E),
                 w_up=np.stack([up] * E), w_down=np.stack([dn] * E))
    x = rng.standard_normal((2, 5, 6))
    g1 = np.abs(rng.standard_normal(6)) + 0.5
    g2 = np.abs(rng.standard_normal(6)) + 0.5
    mp0 = dict(mp, out_proj=np.zeros_like(mp["out_proj"]))
    r = omoe.layer_pair(mp0, moe_p, x, sh, 2, g1, g2)
    xf = x.reshape(10, 6)
    np.testing.assert_allclose(r["h"], xf, rtol=0, atol=0)
    v = xf / np.sqrt((xf ** 2).mean(1, keepdims=True) + 1e-6) * g2
    f = (v @ gt.T) / (1 + np.exp(-(v @ gt.T))) * (v @ up.T) @ dn.T
    lg = v @ moe_p["router"].T
    pr = np.exp(lg - lg.max(1, keepdims=True))
    pr /= pr.sum(1, keepdims=True)
    top2 = np.sort(pr, axis=1)[:, -2:].sum(1)
    np.testing.assert_allclose(r["out"], xf + top2[:, None] * f, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------ MoE pins

def test_router_vs_bruteforce_sort():
    facts = _golden("page_facts.json")
    E, K = facts["n_experts"], facts["top_k"]
    rng = np.random.default_rng(14)
    v = rng.standard_normal((40, 6))
    W = rng.standard_normal((E, 6))
    idx, w, logits = omoe.router(v, W, K)
    for t in range(40):
        lg = [sum(v[t, j] * W[e, j] for j in range(6)) for e in range(E)]
        order = sorted(range(E), key=lambda e: (-lg[e], e))[:K]
        assert list(idx[t]) == order
        den = sum(math.exp(l) for l in lg)
        np.testing.assert_allclose(w[t], [math.exp(lg[e]) / den for e in order], rtol=1e-12)


def test_router_ties_go_to_lower_index():
    W = np.zeros((16, 4))
    W[3] = W[9] = W[12] = [1.0, 0, 0, 0]            # three equal winners
    v = np.array([[2.0, 0, 0, 0], [-1.0, 0, 0, 0]])
    idx, w, _ = omoe.router(v, W, 2)
    assert list(idx[0]) == [3, 9]
    # negative logit for the three: the 13 zero-logit experts win, lowest first
    assert list(idx[1]) == [0, 1]
    np.testing.assert_allclose(w[1], 1.0 / (13 + 3 * math.exp(-1.0)), rtol=1e-14)


def test_router_constructed_winners():
    E = 16
    W = np.eye(E)
    v = np.zeros((E, E))
    for t in range(E):
        v[t, t] = 5.0
        v[t, (t + 7) % E] = 3.0
    idx, _, _ = omoe.router(v, W, 2)
    np.testing.assert_array_equal(idx[:, 0], np.arange(E))
    np.testing.assert_array_equal(idx[:, 1], (np.arange(E) + 7) % E)


def test_permutation_invariants():
    rng = np.random.default_rng(15)
    T, E, K = 97, 16, 2
    idx = np.stack([rng.choice(E, 2, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm = omoe.permute(idx, E)
    assert counts.sum() == T * K
    assert sorted(perm.tolist()) == list(range(T * K))
    keys = [(idx.reshape(-1)[f], f // K, f % K) for f in perm]
    assert keys == sorted(keys)
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert all(idx.reshape(-1)[f] == e for f in seg)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(T * K)
    np.testing.assert_array_equal(perm[inv], np.arange(T * K))


def test_swiglu_expert_vs_loop():
    rng = np.random.default_rng(16)
    v = rng.standard_normal((2, 3))
    g, u, d = rng.standard_normal((4, 3)), rng.standard_normal((4, 3)), rng.standard_normal((3, 4))
    want = np.zeros((2, 3))
    for t in range(2):
        a = []
        for j in range(4):
            gv = sum(v[t, k] * g[j, k] for k in range(3))
            uv = sum(v[t, k] * u[j, k] for k in range(3))
            a.append(gv / (1 + math.exp(-gv)) * uv)
        for o in range(3):
            want[t, o] = sum(a[j] * d[o, j] for j in range(4))
    np.testing.assert_allclose(omoe.swiglu_expert(v, g, u, d), want, rtol=1e-13)


def test_moe_identical_experts():
    rng = np.random.default_rng(17)
    E, dm, dff = 16, 6, 5
    g, u, d = rng.standard_normal((dff, dm)), rng.standard_normal((dff, dm)), rng.standard_normal((dm, dff))
    p = dict(router=rng.standard_normal((E, dm)), w_gate=np.stack([g] * E),
             w_up=np.stack([u] * E), w_down=np.stack([d] * E))
    v = rng.standard_normal((11, dm))
    r = omoe.moe_forward(p, v, 2)
    want = r["w"].sum(1)[:, None] * omoe.swiglu_expert(v, g, u, d)
    np.testing.assert_allclose(r["out"], want, rtol=1e-12, atol=1e-13)
    # sampling tokens gives the same rows
    r2 = omoe.moe_forward(p, v, 2, tokens=[3, 7])
    np.testing.assert_allclose(r2["out"], r["out"][[3, 7]], rtol=1e-14)


def test_moe_single_expert_routing_by_hand():
    """Only experts 0 and 1 can win: out = p0 * f0(v) + p1 * f1(v)."""
    rng = np.random.default_rng(18)
    E, dm, dff = 16, 4, 3
    R = np.full((E, dm), 0.0)
    R[0, 0], R[1, 1] = 10.0, 9.0
    v = np.abs(rng.standard_normal((5, dm))) + 1.0
    v[:, 1] = v[:, 0]                                  # expert 0 logit > expert 1 logit
    p = dict(router=R, w_gate=rng.standard_normal((E, dff, dm)),
             w_up=rng.standard_normal((E, dff, dm)), w_down=rng.standard_normal((E, dm, dff)))
    r = omoe.moe_forward(p, v, 2)
    assert (r["idx"][:, 0] == 0).all() and (r["idx"][:, 1] == 1).all()
    f = lambda e: omoe.swiglu_expert(v, p["w_gate"][e], p["w_up"][e], p["w_down"][e])
    want = r["w"][:, :1] * f(0) + r["w"][:, 1:] * f(1)
    np.testing.assert_allclose(r["out"], want, rtol=1e-13)


# ------------------------------------------------------------------ ExpertsInt8 pins

def test_int8_rows_by_hand():
    """Rows whose maxima make s a power of two, so every w / s is exact.

    Row 0: max 127 -> s = 1; -63.5 and 2.5, 0.5, -1.5 are halves that round
    to the even neighbour.  Row 1: max 254 -> s = 2.  Row 2: all zero.
    """
    w = np.array([[127.0, -63.5, 2.5, 0.5, -1.5, 0.0, 1e-3],
                  [-254.0, -3.0, 5.0, 1.0, 7.0, 253.0, 3.0],
                  [0.0] * 7])
    q, s = omoe.quantize_int8_rows(w)
    assert q.dtype == np.int8 and s.dtype == np.float32
    assert s.tolist() == [1.0, 2.0, 0.0]
    assert q.tolist() == [[127, -64, 2, 0, -2, 0, 0],
                          [-127, -2, 2, 0, 4, 126, 2],
                          [0] * 7]


def test_int8_error_bound_and_extremes():
    rng = np.random.default_rng(19)
    w = (rng.standard_normal((3, 40, 33)) * 0.02).astype(np.float32)
    w[1, 5] *= 1000.0                              # one row far larger than the rest
    q, s = omoe.quantize_int8_rows(w)
    assert q.shape == w.shape and s.shape == w.shape[:2]
    deq = omoe.dequantize_int8_rows(q, s)
    err = np.abs(deq - w.astype(np.float64))
    # rint leaves at most half a step; the fp32 division adds one rounding of w / s
    assert (err <= s[..., None].astype(np.float64) * (0.5 + 2.0 ** -17)).all()
    # the row maximum is +-127, no code exceeds it, signs agree where q != 0
    amax_pos = np.abs(w).argmax(-1)
    np.testing.assert_array_equal(np.abs(np.take_along_axis(q, amax_pos[..., None], -1))[..., 0], 127)
    assert np.abs(q.astype(np.int32)).max() <= 127
    nz = q != 0
    assert (np.sign(q[nz]) == np.sign(w[nz])).all()
    # per-row: the large row does not change its neighbours' codes
    w2 = w.copy()
    w2[1, 5] = w[1, 5] / 1000.0
    q2, _ = omoe.quantize_int8_rows(w2)
    np.testing.assert_array_equal(np.delete(q2[1], 5, 0), np.delete(q[1], 5, 0))


def test_int8_power_of_two_scaling():
    rng = np.random.default_rng(20)
    w = (rng.standard_normal((8, 64)) * 0.02).astype(np.float32)
    q, s = omoe.quantize_int8_rows(w)
    for k in (-3, 1, 5):
        qk, sk = omoe.quantize_int8_rows(w * np.float32(2.0 ** k))
        np.testing.assert_array_equal(qk, q)
        np.testing.assert_array_equal(sk, s * np.float32(2.0 ** k))


def test_int8_moe_lossless_on_representable_weights():
    """Weights q * 2^-e with the row maximum at |q| = 127 come back exactly,
    so the MoE on the int8 codes equals the MoE on the original weights."""
    rng = np.random.default_rng(21)
    E, dm, dff = 16, 8, 6

    def grid(shape):
        q = rng.integers(-127, 128, size=shape)
        q[..., 0] = 127 * np.where(rng.random(shape[:-1]) < 0.5, -1, 1)
        e = rng.integers(5, 9, size=shape[:-1])[..., None]
        return q * 2.0 ** (-e)

    p = dict(router=rng.standard_normal((E, dm)), w_gate=grid((E, dff, dm)),
             w_up=grid((E, dff, dm)), w_down=grid((E, dm, dff)))
    pq = omoe.experts_int8(p)
    back = omoe.dequantized(pq)
    for k in ("w_gate", "w_up", "w_down"):
        np.testing.assert_array_equal(back[k], p[k])
    v = rng.standard_normal((13, dm))
    np.testing.assert_array_equal(omoe.moe_forward(back, v, 2)["out"], omoe.moe_forward(p, v, 2)["out"])


# ------------------------------------------------------------------ attention pins

from oracle import attention as oatt  # noqa: E402
from synthetic import AttnShape  # noqa: E402


def _attn_rand(rng, shape, B, L):
    H, G, D, dm = shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.d_model
    p = dict(wq=rng.standard_normal((H * D, dm)) * 0.5, wk=rng.standard_normal((G * D, dm)) * 0.5,
             wv=rng.standard_normal((G * D, dm)), wo=rng.standard_normal((dm, H * D)))
    return p, rng.standard_normal((B, L, dm))


def test_attention_vs_python_loop():
    sh = AttnShape(d_model=5, n_heads=4, n_kv_heads=2, head_dim=3)
    rng = np.random.default_rng(30)
    p, x = _attn_rand(rng, sh, 2, 4)
    H, G, D = 4, 2, 3
    want = np.zeros((2, 4, 5))
    for b in range(2):
        for t in range(4):
            o = []
            for h in range(H):
                g = h // (H // G)
                q = [sum(p["wq"][h * D + d, i] * x[b, t, i] for i in range(5)) for d in range(D)]
                ks = [[sum(p["wk"][g * D + d, i] * x[b, j, i] for i in range(5)) for d in range(D)] for j in range(t + 1)]
                vs = [[sum(p["wv"][g * D + d, i] * x[b, j, i] for i in range(5)) for d in range(D)] for j in range(t + 1)]
                sc = [sum(q[d] * ks[j][d] for d in range(D)) / math.sqrt(D) for j in range(t + 1)]
                mx = max(sc)
                e = [math.exp(v - mx) for v in sc]
                z = sum(e)
                o += [sum(e[j] / z * vs[j][d] for j in range(t + 1)) for d in range(D)]
            for i in range(5):
                want[b, t, i] = sum(p["wo"][i, c] * o[c] for c in range(H * D))
    np.testing.assert_allclose(oatt.attention_prefill(p, x, sh)["out"], want, rtol=1e-12, atol=1e-12)


def test_attention_zero_query_is_running_mean():
    sh = AttnShape(d_model=6, n_heads=2, n_kv_heads=1, head_dim=4)
    rng = np.random.default_rng(31)
    p, x = _attn_rand(rng, sh, 1, 7)
    p["wq"][:] = 0.0
    r = oatt.attention_prefill(p, x, sh)
    v = r["v"][0, :, 0]                                     # [L, D]
    want = np.cumsum(v, axis=0) / np.arange(1, 8)[:, None]
    for h in range(2):
        np.testing.assert_allclose(r["o"][0, :, h], want, rtol=1e-13)
    # the first token sees only itself
    np.testing.assert_allclose(r["o"][0, 0, 0], v[0], rtol=1e-14)


def test_attention_gqa_equals_repeated_mha():
    sh = AttnShape(d_model=8, n_heads=6, n_kv_heads=2, head_dim=3)
    rng = np.random.default_rng(32)
    p, x = _attn_rand(rng, sh, 2, 5)
    rep = dict(p)
    for k in ("wk", "wv"):
        w = p[k].reshape(2, 3, 8)
        rep[k] = np.repeat(w, 3, axis=0).reshape(18, 8)      # KV head g serves query heads 3g..3g+2
    mha = AttnShape(d_model=8, n_heads=6, n_kv_heads=6, head_dim=3)
    np.testing.assert_allclose(oatt.attention_prefill(p, x, sh)["out"],
                               oatt.attention_prefill(rep, x, mha)["out"], rtol=1e-13, atol=1e-13)


def test_attention_key_shift_and_causality():
    sh = AttnShape(d_model=6, n_heads=4, n_kv_heads=2, head_dim=4)
    rng = np.random.default_rng(33)
    p, x = _attn_rand(rng, sh, 1, 9)
    q, k, v = oatt.project(p, x, sh)
    o = oatt.attend(q, k, v)
    # a vector common to every key adds the same amount to a query's logits
    o2 = oatt.attend(q, k + rng.standard_normal((1, 1, 2, 4)), v)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-12)
    # changing token 5 leaves tokens 0..4 unchanged and moves token 5
    x2 = x.copy()
    x2[0, 5] += 1.0
    a = oatt.attention_prefill(p, x, sh)["out"]
    b = oatt.attention_prefill(p, x2, sh)["out"]
    np.testing.assert_array_equal(a[0, :5], b[0, :5])
    assert np.abs(a[0, 5:] - b[0, 5:]).min() > 0


def test_attention_two_keys_closed_form():
    """Query (s, 0) against one-hot keys e0, e1: weights e^{s/sqrt(2)} : 1."""
    q = np.zeros((1, 1, 1, 2))
    q[0, 0, 0, 0] = 3.0
    k = np.array([[[[1.0, 0.0]], [[0.0, 1.0]]]])            # [1, 2, 1, 2]
    v = np.array([[[[10.0, 0.0]], [[0.0, 20.0]]]])
    o = oatt.attend(q, k, v, q_pos0=1)
    w0 = math.exp(3.0 / math.sqrt(2)) / (math.exp(3.0 / math.sqrt(2)) + 1.0)
    np.testing.assert_allclose(o[0, 0, 0], [10.0 * w0, 20.0 * (1 - w0)], rtol=1e-14)


def test_attention_step_equals_prefill_last_row():
    sh = AttnShape(d_model=8, n_heads=4, n_kv_heads=2, head_dim=4)
    rng = np.random.default_rng(34)
    p, x = _attn_rand(rng, sh, 3, 7)
    full = oatt.attention_prefill(p, x, sh)
    pre = oatt.attention_prefill(p, x[:, :6], sh)
    st = oatt.attention_step(p, x[:, 6], pre["k"], pre["v"], 6, sh)
    np.testing.assert_allclose(st["out"], full["out"][:, 6], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(st["k_new"], full["k"][:, 6], rtol=1e-13)
