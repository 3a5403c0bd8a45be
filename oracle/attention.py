"""fp64 oracle of the Jamba attention layer (grouped-query attention).

TEST INFRASTRUCTURE: see the package header for who may import this.

"Jamba: A Hybrid Transformer-Mamba Language Model" (summary page), section 2:
one layer in eight of a Jamba block is an attention layer (1:7 with Mamba);
its other details are the standard ones, grouped-query attention (GQA) among
them; no explicit positional information (no positional embedding, no RoPE)
is used.  Readings where the page is silent: n_heads query heads and
n_kv_heads key/value heads of width head_dim (4096 = 32 x 128 with 8 KV
heads at Jamba width); query head h reads KV head h // (n_heads /
n_kv_heads); causal softmax over keys 0..t of q_t . k_j / sqrt(head_dim);
projections without bias; out = o W_o^T (+ residual).  Decoding appends the
new token's key and value to the cache and attends over positions 0..pos.

Parity pins (tests/test_oracle_pins.py): a pure-Python loop on a tiny case;
q = 0 gives the running mean of the values; one token attends to itself
only; GQA equals multi-head attention with the KV heads repeated; a common
vector added to every key changes nothing; outputs before t do not depend on
inputs at t; two one-hot keys give the closed-form two-way softmax; a decode
step equals the last row of the prefill of L + 1 tokens.
"""
import numpy as np

from .mamba import linear


def heads(shape):
    H, G, D = shape.n_heads, shape.n_kv_heads, shape.head_dim
    assert H % G == 0
    return H, G, D


def project(p, x, shape):
    """x [B, L, d_model] -> q [B, L, H, D], k, v [B, L, G, D]."""
    H, G, D = heads(shape)
    Bsz, L, _ = x.shape
    q = linear(x, p["wq"]).reshape(Bsz, L, H, D)
    k = linear(x, p["wk"]).reshape(Bsz, L, G, D)
    v = linear(x, p["wv"]).reshape(Bsz, L, G, D)
    return q, k, v


def attend(q, k, v, q_pos0=0):
    """Causal GQA attention core.

    q [B, Lq, H, D] at positions q_pos0 .. q_pos0 + Lq - 1; k, v [B, Lk, G, D]
    at positions 0 .. Lk - 1.  Query t sees keys 0 .. q_pos0 + t.
    """
    Bsz, Lq, H, D = q.shape
    G = k.shape[2]
    rep = H // G
    o = np.zeros_like(q)
    for b in range(Bsz):
        for h in range(H):
            g = h // rep
            s = q[b, :, h] @ k[b, :, g].T / np.sqrt(D)            # [Lq, Lk]
            t = np.arange(Lq)[:, None] + q_pos0
            j = np.arange(k.shape[1])[None, :]
            s = np.where(j <= t, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            e = np.exp(s)
            o[b, :, h] = (e / e.sum(axis=1, keepdims=True)) @ v[b, :, g]
    return o


def attention_prefill(p, x, shape, residual=None):
    """x [B, L, d_model] -> dict(out [B, L, d_model], k, v [B, L, G, D], o)."""
    q, k, v = project(p, x, shape)
    o = attend(q, k, v)
    Bsz, L = x.shape[:2]
    out = linear(o.reshape(Bsz, L, -1), p["wo"])
    if residual is not None:
        out = out + residual
    return dict(out=out, k=k, v=v, o=o)


def attention_step(p, x_t, k_cache, v_cache, pos, shape, residual=None):
    """One token per sequence at position pos (0-based) after pos cached tokens.

    x_t [B, d_model]; k_cache, v_cache [B, >= pos, G, D] (positions 0..pos-1
    used).  Returns dict(out [B, d_model], k_new, v_new [B, G, D]).
    """
    q, k, v = project(p, x_t[:, None], shape)
    kk = np.concatenate([k_cache[:, :pos], k], axis=1)
    vv = np.concatenate([v_cache[:, :pos], v], axis=1)
    o = attend(q, kk, vv, q_pos0=pos)
    out = linear(o.reshape(x_t.shape[0], -1), p["wo"])
    if residual is not None:
        out = out + residual
    return dict(out=out, k_new=k[:, 0], v_new=v[:, 0])
