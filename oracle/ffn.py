"""Oracle for the masked SwiGLU FFN and for mask reordering (fp64, CPU).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the CUDA path.

Source: "WIDE: Boosting Adaptive LLM Inference via Token-level Dynamic Width
Pruning" -- technical summary section 2.A (pruning units: contiguous channel
groups of the FFN intermediate dimension D'; a per-token binary execute/skip
decision per group) and section 2.B (unified mask reordering: per routing
group, sort the binary mask along the token dimension M so that the active
tokens form a contiguous prefix).

The method only skips work whose result is multiplied by zero, so the value it
must reach is the dense layer with the per-token group mask applied
elementwise to the intermediate activations; ``ffn_masked`` is that
definition.  ``ffn_token_loop`` is a second, independent form (the per-token
loop that visits only kept groups, in C) used as a cross-check and as the
timed CPU baseline.  ``reorder`` is the canonical form of section 2.B.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _clib


def widen(a: np.ndarray, dtype: str) -> np.ndarray:
    """bf16 bit patterns (uint16) or fp32 values -> float64, exactly."""
    if dtype == "bf16":
        u = np.ascontiguousarray(a, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
        return u.view(np.float32).astype(np.float64)
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    raise ValueError(dtype)


def mask_bool(words: np.ndarray, G: int) -> np.ndarray:
    """Packed words[T][ceil(G/32)] -> bool[T][G] (bit g%32 of word g//32)."""
    words = np.asarray(words, dtype=np.uint32)
    T, W = words.shape
    out = np.zeros((T, G), dtype=bool)
    for g in range(G):
        out[:, g] = (words[:, g // 32] >> np.uint32(g % 32)) & np.uint32(1) == 1
    return out


def silu(a: np.ndarray) -> np.ndarray:
    """SiLU(a) = a * sigmoid(a) = a / (1 + exp(-a))."""
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-a))


def ffn_masked(x, w_gate, w_up, w_down, mask_words, gs: int, dtype: str = "bf16") -> np.ndarray:
    """Masked SwiGLU FFN, definition form (section 2.A).

    h = silu(x W_gate^T) * (x W_up^T)           [T][I]
    h[t, c] = 0 where token t skips group c // gs
    out = h W_down^T                             [T][H]

    x[T][H], W_gate/W_up[I][H], W_down[H][I] (nn.Linear layout); returns
    float64 [T][H].  The matrix products are numpy float64 matmuls.
    """
    Wg = widen(w_gate, dtype)
    return ffn_masked_f64(widen(x, dtype), Wg, widen(w_up, dtype), widen(w_down, dtype),
                          mask_bool(mask_words, Wg.shape[0] // gs), gs)


def ffn_masked_f64(X, Wg, Wu, Wd, m, gs: int) -> np.ndarray:
    """The same definition on float64 operands and a bool[T][G] mask."""
    h = silu(X @ Wg.T) * (X @ Wu.T)
    h *= np.repeat(m, gs, axis=1)
    return h @ Wd.T


def ffn_dense(x, w_gate, w_up, w_down, dtype: str = "bf16") -> np.ndarray:
    """The unmasked SwiGLU FFN (the all-ones special case)."""
    X = widen(x, dtype)
    return (silu(X @ widen(w_gate, dtype).T) * (X @ widen(w_up, dtype).T)) @ widen(w_down, dtype).T


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    return ctypes.c_void_p(a.ctypes.data)


def ffn_token_loop(x, w_gate, w_up, w_down, mask_words, gs: int, dtype: str = "bf16") -> np.ndarray:
    """Per-token loop over kept groups only (C, fp64, OpenMP over tokens)."""
    dt = {"bf16": 0, "f32": 1}[dtype]
    cast = np.uint16 if dt == 0 else np.float32
    x = np.ascontiguousarray(x, dtype=cast)
    w_gate = np.ascontiguousarray(w_gate, dtype=cast)
    w_up = np.ascontiguousarray(w_up, dtype=cast)
    w_down = np.ascontiguousarray(w_down, dtype=cast)
    mask_words = np.ascontiguousarray(mask_words, dtype=np.uint32)
    T, H = x.shape
    I = w_gate.shape[0]
    out = np.zeros((T, H), dtype=np.float64)
    rc = _clib.lib().oracle_ffn_token_loop(_ptr(x), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                                           _ptr(mask_words), T, H, I, gs, dt, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_ffn_token_loop failed: {rc}")
    return out


def check_mask(mask_words, G: int) -> int:
    """0 when no bit at or above G is set, else a negative code."""
    mw = np.ascontiguousarray(mask_words, dtype=np.uint32)
    return _clib.lib().oracle_check_mask(_ptr(mw), mw.shape[0], G)


def reorder(mask_words, G: int, tile_m: int) -> dict:
    """Canonical mask reordering (section 2.B) -- see wide_oracle.c.

    Returns count[G], perm[G][T], items[n][2] (group, tile), sig_perm[T],
    tile_union[ceil(T/tile_m)][W].
    """
    mw = np.ascontiguousarray(mask_words, dtype=np.uint32)
    T, W = mw.shape
    nt = (T + tile_m - 1) // tile_m
    count = np.zeros(G, dtype=np.int32)
    perm = np.zeros((G, T), dtype=np.int32)
    items = np.zeros((G * nt + 1, 2), dtype=np.int32)
    n_items = np.zeros(1, dtype=np.int64)
    sig = np.zeros(T, dtype=np.int32)
    tu = np.zeros((nt, W), dtype=np.uint32)
    rc = _clib.lib().oracle_reorder(_ptr(mw), T, G, tile_m, _ptr(count), _ptr(perm), _ptr(items),
                                    _ptr(n_items), _ptr(sig), _ptr(tu))
    if rc != 0:
        raise ValueError(f"oracle_reorder failed: {rc}")
    n = int(n_items[0])
    return {"count": count, "perm": perm, "items": items[:n].copy(), "sig_perm": sig,
            "tile_union": tu}
