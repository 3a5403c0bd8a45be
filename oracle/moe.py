"""fp64 oracle of the top-K MoE with SwiGLU experts, and of the Jamba layer pair.

TEST INFRASTRUCTURE: see the package header for who may import this.

"Jamba: A Hybrid Transformer-Mamba Language Model" (summary page), section 2:
some MLPs are replaced by MoE layers with n experts of which the router picks
the top K per token; the MLPs are SwiGLU; section 3.1 fixes n = 16, K = 2.
Readings where the page is silent: the router is a linear map d_model -> n
followed by a softmax over all n; the K largest logits win, ties going to the
lower expert index; each token's output is sum_k p_k * expert_k(v) with the
raw (not renormalised) softmax probabilities, slot 0 first; a SwiGLU expert
computes down(SiLU(gate v) * (up v)); routed rows are ordered by (expert,
token, slot).  The layer pair is pre-norm residual: h = x + Mamba(RMSNorm(x)),
out = h + MoE(RMSNorm(h)).

ExpertsInt8 ("Jamba-1.5" article, section on ExpertsInt8; "Jamba-1.5"
abstract): only the expert (MoE/MLP) weights are stored as INT8 and are
dequantised inside the MoE kernel at run time; activations stay BF16; no
calibration data is used.  The pages do not give the scheme.  Reading: each
output row of each expert matrix (a row of w_gate / w_up over d_model, a row
of w_down over d_ff) gets one symmetric scale s = max|w| / 127, taken in
fp32; q = round-half-even(w / s) in fp32, an integer in [-127, 127]; an
all-zero row has s = 0 and q = 0.  The dequantised weight is q * s, formed
here in fp64, so the int8 MoE is the MoE above on the weights q * s.

Parity pins (tests/test_oracle_pins.py): top-K vs a brute-force sort with
Python's sorted(); forced ties; constructed winning rows; the permutation
invariants (a permutation, sorted by (expert, token, slot), counts sum to
T*K, inverse composes to identity); identical experts give
(w_0 + w_1) * expert(v); SwiGLU vs a pure-Python loop on a tiny case.
Int8: hand-worked rows with exact halves (ties to even); the error bound
|q s - w| <= s / 2; the row maximum maps to +-127; per-row independence;
power-of-two scaling of a row scales s alone; weights that are already
q * s with s a power of two quantise losslessly, so the int8 MoE equals the
plain MoE exactly.
Layer pair: the whole pair against the same pair written with scalar Python
loops on a tiny case (router indices equal, outputs to 1e-12), and two
closed forms: out_proj = 0 gives h = x exactly, and identical experts give
out = h + (p_1 + p_2) f(RMSNorm(h)).
"""
import numpy as np

from .mamba import linear, rmsnorm, silu, mamba_prefill, to64


def router(v, W_r, top_k):
    """Returns (idx [T, K] int32, w [T, K] float64, logits [T, E])."""
    logits = linear(v, W_r)
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    p = e / e.sum(axis=1, keepdims=True)
    E = logits.shape[1]
    # stable sort on -logit keeps the lower index first among equal logits
    order = np.argsort(-logits, axis=1, kind="stable")[:, :top_k]
    idx = order.astype(np.int32)
    w = np.take_along_axis(p, order, axis=1)
    assert idx.max() < E
    return idx, w, logits


def permute(idx, n_experts):
    """Counting sort of the (token, slot) pairs by (expert, token, slot).

    Returns (counts [E], offsets [E+1], perm [T*K]) where perm[p] = t*K + k of
    the pair stored at routed row p.
    """
    T, K = idx.shape
    flat = idx.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=n_experts).astype(np.int32)
    offsets = np.zeros(n_experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    # key (expert, flat position): flat position already orders (token, slot)
    perm = np.argsort(flat * (T * K) + np.arange(T * K), kind="stable").astype(np.int32)
    return counts, offsets, perm


def swiglu_expert(v, w_gate, w_up, w_down):
    return linear(silu(linear(v, w_gate)) * linear(v, w_up), w_down)


def quantize_int8_rows(w):
    """Per-row symmetric INT8 codes of w [..., k] (any float array).

    Returns (q int8 [..., k], s float32 [...]).  Every decision is taken in
    fp32: s = fp32(max|w|) / 127, q = rint(fp32(w) / s) (numpy rounds halves
    to even); rows of zeros give s = 0, q = 0.
    """
    w32 = to64(w).astype(np.float32)   # bf16 and fp32 inputs are exact in both
    amax = np.max(np.abs(w32), axis=-1)
    s = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    q = np.rint(w32 / safe[..., None])
    q = np.where(s[..., None] > 0, q, 0.0)
    assert np.abs(q).max(initial=0) <= 127
    return q.astype(np.int8), s


def dequantize_int8_rows(q, s):
    """fp64 weights q * s (s broadcast over the last axis)."""
    return np.asarray(q, dtype=np.float64) * np.asarray(s, dtype=np.float64)[..., None]


def experts_int8(p):
    """INT8 codes and scales of the expert matrices of a MoE parameter dict."""
    out = dict(router=to64(p["router"]))
    for k in ("w_gate", "w_up", "w_down"):
        out["q_" + k[2:]], out["s_" + k[2:]] = quantize_int8_rows(p[k])
    return out


def dequantized(pq):
    """fp64 MoE parameter dict from the output of experts_int8."""
    out = dict(router=np.asarray(pq["router"], dtype=np.float64))
    for k in ("gate", "up", "down"):
        out["w_" + k] = dequantize_int8_rows(pq["q_" + k], pq["s_" + k])
    return out


def moe_forward(p, v, top_k, tokens=None):
    """MoE output for every token (or only the listed tokens, for sampling).

    p: dict of float64 arrays router [E, dm], w_gate/w_up [E, dff, dm],
    w_down [E, dm, dff].  Returns dict(out, idx, w, counts, offsets, perm).
    """
    E = p["router"].shape[0]
    idx, w, logits = router(v, p["router"], top_k)
    counts, offsets, perm = permute(idx, E)
    sel = np.arange(v.shape[0]) if tokens is None else np.asarray(tokens)
    out = np.zeros((len(sel), v.shape[1]))
    for e in range(E):
        rows, slots = np.nonzero(idx[sel] == e)
        if len(rows) == 0:
            continue
        ye = swiglu_expert(v[sel[rows]], p["w_gate"][e], p["w_up"][e], p["w_down"][e])
        # accumulate slot 0 before slot 1 (same order as the sum over k)
        for k in range(top_k):
            m = slots == k
            out[rows[m]] += w[sel[rows[m]], k][:, None] * ye[m]
    return dict(out=out, idx=idx, w=w, logits=logits, counts=counts,
                offsets=offsets, perm=perm, tokens=sel)


def layer_pair(mp, moe_p, x, mshape, top_k, g1, g2, eps=1e-6, tokens=None, scan="numpy"):
    """x [B, L, dm] -> (out, h, ...) of RMSNorm->Mamba->residual->RMSNorm->MoE->residual.

    tokens: flat token indices (b*L + t) at which to evaluate the MoE (all
    when None); the Mamba half is always evaluated in full.
    """
    Bsz, L, dm = x.shape
    u = rmsnorm(x, g1, eps)
    h = x + mamba_prefill(mp, u, mshape, scan=scan)["out"]
    hf = h.reshape(Bsz * L, dm)
    v = rmsnorm(hf, g2, eps)
    r = moe_forward(moe_p, v, top_k, tokens)
    sel = r["tokens"]
    out = hf[sel] + r["out"]
    return dict(out=out, h=hf, v=v, **{k: r[k] for k in ("idx", "w", "logits", "counts",
                                                         "offsets", "perm", "tokens")})
