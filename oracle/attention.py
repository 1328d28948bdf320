"""Oracle for the head-group-masked attention half and the whole layer (fp64, CPU).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the CUDA path.

Source: "WIDE: Boosting Adaptive LLM Inference via Token-level Dynamic Width
Pruning" -- technical summary section 2.A: attention prunes groups of heads
aligned with the grouped-query-attention structure (a group = the query heads
that share one KV head), chosen per token.  The pages fix nothing else about
the layer, so the readings below are the plain Llama-3 pre-norm block:

* RMSNorm(x) = x / sqrt(mean(x^2) + eps) * gamma, eps = 1e-5.
* RoPE in the rotate-half pairing (i, i + hd/2), inverse frequency
  theta^(-2i/hd), theta = 5e5, applied to q and k at the token's position.
* A skipped head group masks queries only: every token's K and V are computed
  and cached for every group (later queries need them); a token that skips
  group j gets a zero output for the query heads of j, so those heads'
  attention and their o_proj columns contribute nothing.
* Softmax scale 1/sqrt(hd); decode appends the new token's K/V at position
  cache_len and attends over cache_len + 1 keys; prefill is causal within
  each sequence from position 0.
* Layer: h1 = x + attn_out; out = h1 + FFN(RMSNorm(h1) * gamma2) with the
  token's FFN group mask.
"""
from __future__ import annotations

import numpy as np

from .ffn import widen, mask_bool, ffn_masked_f64


def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * gamma over the last axis (float64)."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * gamma


def rope(v: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE.  v[..., T, hd] with positions pos[T]."""
    hd = v.shape[-1]
    half = hd // 2
    inv = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]      # [T][half]
    c, s = np.cos(ang), np.sin(ang)
    a, b = v[..., :half], v[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def softmax_rows(s: np.ndarray) -> np.ndarray:
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention_masked(case, ret_parts: bool = False):
    """Masked GQA attention half of the layer, for an ``AttnCase``.

    Returns attn_out[T][H] (float64, before the residual) and, with
    ``ret_parts``, a dict with xn, q, k, v (after RoPE) and the per-head
    outputs o[T][n_q][hd] (after the head-group mask).
    """
    c = case
    T, H, nq, nkv, hd = c.T, c.H, c.n_q, c.n_kv, c.hd
    rep = nq // nkv
    x = widen(c.x, "bf16")
    xn = rmsnorm(x, widen(c.gamma1, "bf16"), c.eps)
    q = (xn @ widen(c.wq, "bf16").T).reshape(T, nq, hd)
    k = (xn @ widen(c.wk, "bf16").T).reshape(T, nkv, hd)
    v = (xn @ widen(c.wv, "bf16").T).reshape(T, nkv, hd)
    pos = c.positions
    q = rope(q.transpose(1, 0, 2), pos, c.theta).transpose(1, 0, 2)
    k = rope(k.transpose(1, 0, 2), pos, c.theta).transpose(1, 0, 2)
    m = mask_bool(c.mask_words, nkv)                                   # [T][nkv]
    o = np.zeros((T, nq, hd), dtype=np.float64)
    scale = 1.0 / np.sqrt(hd)
    S = c.seq_len
    for b in range(c.n_seq):
        rows = slice(b * S, (b + 1) * S)
        for j in range(nkv):
            if c.mode == "decode":
                Kp = widen(c.k_cache[b, j], "bf16") if c.cache_len > 0 else np.zeros((0, hd))
                Vp = widen(c.v_cache[b, j], "bf16") if c.cache_len > 0 else np.zeros((0, hd))
                K = np.concatenate([Kp, k[rows, j]], axis=0)           # [L + S][hd]
                V = np.concatenate([Vp, v[rows, j]], axis=0)
            else:
                K, V = k[rows, j], v[rows, j]
            L0 = K.shape[0] - S                                        # keys before the block
            causal = np.arange(K.shape[0])[None, :] <= (L0 + np.arange(S))[:, None]
            for hh in range(rep):
                h = j * rep + hh
                s = (q[rows, h] @ K.T) * scale
                s = np.where(causal, s, -np.inf)
                o[rows, h] = softmax_rows(s) @ V
        o[rows] *= np.repeat(m[rows], rep, axis=1)[:, :, None]
    attn_out = o.reshape(T, nq * hd) @ widen(c.wo, "bf16").T
    if ret_parts:
        return attn_out, {"xn": xn, "q": q, "k": k, "v": v, "o": o}
    return attn_out


def layer_masked(lc, ret_parts: bool = False):
    """The whole masked layer for a ``LayerCase`` (pre-norm Llama block)."""
    a = lc.attn
    attn_out, parts = attention_masked(a, ret_parts=True)
    h1 = widen(a.x, "bf16") + attn_out
    xn2 = rmsnorm(h1, widen(lc.gamma2, "bf16"), a.eps)
    f = lc.ffn
    ffn_out = ffn_masked_f64(xn2, widen(f.w_gate, "bf16"), widen(f.w_up, "bf16"),
                             widen(f.w_down, "bf16"), mask_bool(f.mask_words, f.I // f.gs), f.gs)
    out = h1 + ffn_out
    if ret_parts:
        parts.update({"attn_out": attn_out, "h1": h1, "xn2": xn2, "ffn_out": ffn_out})
        return out, parts
    return out


def layer_masked_rows(lc, rows):
    """The layer's outputs for the token rows ``rows`` only: the same
    definition as ``layer_masked``, evaluated row by row (K and V are still
    computed for every token a selected query can see).  Returns (out[rows],
    parts) with attn_out, ffn_out, h1 for those rows and k, v (after RoPE)
    for all tokens."""
    a = lc.attn
    T, nq, nkv, hd = a.T, a.n_q, a.n_kv, a.hd
    rep = nq // nkv
    rows = np.asarray(rows)
    x = widen(a.x, "bf16")
    xn = rmsnorm(x, widen(a.gamma1, "bf16"), a.eps)
    pos = a.positions
    k = rope((xn @ widen(a.wk, "bf16").T).reshape(T, nkv, hd).transpose(1, 0, 2), pos,
             a.theta).transpose(1, 0, 2)
    v = (xn @ widen(a.wv, "bf16").T).reshape(T, nkv, hd)
    q = (xn[rows] @ widen(a.wq, "bf16").T).reshape(len(rows), nq, hd)
    q = rope(q.transpose(1, 0, 2), pos[rows], a.theta).transpose(1, 0, 2)
    m = mask_bool(a.mask_words, nkv)
    S = a.seq_len
    o = np.zeros((len(rows), nq, hd))
    for n, t in enumerate(rows):
        b, i = divmod(int(t), S)
        for j in range(nkv):
            if not m[t, j]:
                continue
            Kn, Vn = k[b * S:b * S + i + 1, j], v[b * S:b * S + i + 1, j]
            if a.mode == "decode" and a.cache_len > 0:
                Kn = np.concatenate([widen(a.k_cache[b, j], "bf16"), Kn], axis=0)
                Vn = np.concatenate([widen(a.v_cache[b, j], "bf16"), Vn], axis=0)
            for hh in range(rep):
                h = j * rep + hh
                s = (Kn @ q[n, h]) / np.sqrt(hd)
                p = np.exp(s - s.max())
                o[n, h] = (p / p.sum()) @ Vn
    attn_out = o.reshape(len(rows), nq * hd) @ widen(a.wo, "bf16").T
    h1 = x[rows] + attn_out
    xn2 = rmsnorm(h1, widen(lc.gamma2, "bf16"), a.eps)
    f = lc.ffn
    ffn_out = ffn_masked_f64(xn2, widen(f.w_gate, "bf16"), widen(f.w_up, "bf16"),
                             widen(f.w_down, "bf16"), mask_bool(f.mask_words, f.I // f.gs)[rows],
                             f.gs)
    out = h1 + ffn_out
    return out, {"attn_out": attn_out, "ffn_out": ffn_out, "h1": h1, "k": k, "v": v}


__all__ = ["rmsnorm", "rope", "softmax_rows", "attention_masked", "layer_masked",
           "layer_masked_rows"]
