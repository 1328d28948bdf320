"""Oracle for the bottleneck router that produces the group masks (fp64, CPU).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the CUDA path.

Source: "WIDE: Boosting Adaptive LLM Inference via Token-level Dynamic Width
Pruning", technical summary section 2.A, "router architecture": a light
bottleneck router maps the input activations of a block to one binary
decision per group (execute or skip); the Gumbel-Softmax relaxation is used
only while training.

The pages give no equation.  Reading taken here (the plainest one):
  z      = act(u W1^T)              W1 [R][H], R the bottleneck width
  logit  = z W2^T + b               W2 [G][R], b [G] (zero when absent)
  keep   = logit > 0                one difference logit per group; at
                                    inference the execute/skip choice is the
                                    argmax of the two, i.e. the sign
act is ReLU or SiLU (the pages name none).  A logit of exactly 0 skips.
The mask is returned bit-packed token-major, group g in bit g % 32 of word
g // 32, bits at or above G zero: the layout every masked kernel reads.

``route_logits`` is the definition with numpy float64 matmuls on operands
widened exactly from bf16; ``route_logits_loop`` is a second form written as
plain per-(token, group) scalar loops, for tiny sizes only.
"""
from __future__ import annotations

import numpy as np

from .ffn import silu, widen


def _act(a: np.ndarray, act: str) -> np.ndarray:
    if act == "relu":
        return np.maximum(a, 0.0)
    if act == "silu":
        return silu(a)
    raise ValueError(act)


def route_logits(x, w_r1, w_r2, b_r2=None, act: str = "relu") -> np.ndarray:
    """Router logits [T][G] in float64 (section 2.A, reading above).

    x [T][H], w_r1 [R][H], w_r2 [G][R] as bf16 bit patterns (uint16);
    b_r2 fp32 [G] or None.
    """
    X = widen(x, "bf16")
    z = _act(X @ widen(w_r1, "bf16").T, act)
    logit = z @ widen(w_r2, "bf16").T
    if b_r2 is not None:
        logit = logit + np.asarray(b_r2, dtype=np.float32).astype(np.float64)[None, :]
    return logit


def decide(logits: np.ndarray) -> np.ndarray:
    """Execute/skip decision per (token, group): bool[T][G], True = execute."""
    return np.asarray(logits) > 0.0


def pack(keep: np.ndarray) -> np.ndarray:
    """bool[T][G] -> uint32 words[T][ceil(G/32)], group g in bit g%32 of word g//32."""
    keep = np.asarray(keep, dtype=bool)
    T, G = keep.shape
    W = (G + 31) // 32
    out = np.zeros((T, W), dtype=np.uint32)
    for g in range(G):
        out[:, g // 32] |= keep[:, g].astype(np.uint32) << np.uint32(g % 32)
    return out


def route_mask(x, w_r1, w_r2, b_r2=None, act: str = "relu") -> np.ndarray:
    """The router's packed group mask, uint32[T][ceil(G/32)]."""
    return pack(decide(route_logits(x, w_r1, w_r2, b_r2, act)))


def route_logits_loop(x, w_r1, w_r2, b_r2=None, act: str = "relu") -> np.ndarray:
    """The same logits as plain scalar loops (tiny sizes only)."""
    X = widen(x, "bf16")
    W1 = widen(w_r1, "bf16")
    W2 = widen(w_r2, "bf16")
    T, H = X.shape
    R, G = W1.shape[0], W2.shape[0]
    out = np.zeros((T, G))
    for t in range(T):
        z = [0.0] * R
        for r in range(R):
            s = 0.0
            for k in range(H):
                s += float(X[t, k]) * float(W1[r, k])
            if act == "relu":
                z[r] = s if s > 0.0 else 0.0
            else:
                z[r] = s / (1.0 + float(np.exp(-s)))
        for g in range(G):
            s = 0.0 if b_r2 is None else float(np.float32(b_r2[g]))
            for r in range(R):
                s += z[r] * float(W2[g, r])
            out[t, g] = s
    return out
