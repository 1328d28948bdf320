"""Seeded synthetic workloads shaped like the pages' Llama-3.1-8B / 3.2-3B layers.

Every tensor is drawn from its own PCG64 stream, ``default_rng([seed, stream,
*extra])``, so that one tensor can be regenerated without the others and the
weights of a model are the same whatever batch size is drawn with them.
Floating-point draws are fp32 and, for the bf16 workloads, rounded to bf16 by
round-to-nearest-even on the bit pattern; bf16 tensors are returned as
``uint16`` bit patterns (numpy has no bf16 type).

Masks are ``bool[T][G]`` (True = the token executes the group) and are also
returned bit-packed, token-major: ``uint32[T][ceil(G/32)]``, group g in bit
``g % 32`` of word ``g // 32``; bits at or above G are zero.

Workload shapes (WIDE: Boosting Adaptive LLM Inference via Token-level Dynamic
Width Pruning, technical summary section 4: Llama3.1-8B and Llama3.2-3B;
section 2.A: GQA-aligned head groups and contiguous FFN channel groups):

* tiny:   fp32, T=64, H=256, I=1024, 16 groups of 64, Bernoulli(0.5) with at
          least one kept group per token (a row drawn all-zero is redrawn from
          the same stream until it is not).
* decode_ffn: H=3072, I=8192, 64 groups of 128, batch 1/8/32, Bernoulli(0.5).
* prefill_ffn: T=4096, H=4096, I=14336, 112 groups of 128, 8 prototypes each
          keeping exactly 56 groups, each bit then flipped with p=0.1.
* decode_layer: B=16 sequences with a 2048-entry KV cache ~ N(0,1), head-group
          mask Bernoulli(0.34) over 8 KV groups, FFN mask Bernoulli(0.72).
* prefill_layer: 4 sequences x 2048 tokens, 16 prototypes over (8 head groups,
          112 FFN groups) at keep k (0.25/0.5/0.75/1.0), flips p=0.1 (none at
          k=1.0).
* router: a bottleneck router (section 2.A) with random weights: x ~ N(0,1)
          bf16 [T][H] stands for the normalised sublayer input, W_r1 [R][H]
          and W_r2 [G][R] ~ N(0, 0.02) bf16, optional bias ~ N(0, bias_std)
          fp32 [G].

x ~ N(0,1); weights ~ N(0, 0.02) (0.02 is the standard deviation) in the
nn.Linear layout [out_features][in_features]; RMSNorm gains are
1 + 0.02 N(0,1) so that the gain multiply is exercised.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

# One stream id per drawn tensor.  Extra key parts (batch size, keep rate)
# follow the id.
_STREAM = {
    "x": 1, "w_gate": 2, "w_up": 3, "w_down": 4,
    "wq": 5, "wk": 6, "wv": 7, "wo": 8, "gamma1": 9, "gamma2": 10,
    "k_cache": 11, "v_cache": 12,
    "mask_f": 20, "mask_a": 21, "proto_f": 22, "proto_a": 23,
    "proto_pick": 24, "flip_f": 25, "flip_a": 26,
    "w_r1": 30, "w_r2": 31, "b_r2": 32,
}


def _rng(seed: int, name: str, *extra: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), _STREAM[name], *[int(e) for e in extra]])


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); uint16 bits."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (b >> np.uint32(16)) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += b
    r >>= np.uint32(16)
    return r.astype(np.uint16)


def f32_from_bf16_bits(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32 (test convenience)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(seed, name, shape, std=1.0, bf16=True, *extra):
    a = _rng(seed, name, *extra).standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return bf16_bits_from_f32(a) if bf16 else a


def pack_mask(mask: np.ndarray) -> np.ndarray:
    """bool[T][G] -> uint32[T][ceil(G/32)], group g in bit g%32 of word g//32."""
    mask = np.asarray(mask, dtype=bool)
    T, G = mask.shape
    W = (G + 31) // 32
    padded = np.zeros((T, W * 32), dtype=np.uint64)
    padded[:, :G] = mask
    padded = padded.reshape(T, W, 32)
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (padded * weights).sum(axis=2).astype(np.uint32)


def unpack_mask(words: np.ndarray, G: int) -> np.ndarray:
    words = np.asarray(words, dtype=np.uint32)
    T, W = words.shape
    bits = (words[:, :, None] >> np.arange(32, dtype=np.uint32)) & np.uint32(1)
    return bits.reshape(T, W * 32)[:, :G].astype(bool)


def bernoulli_mask(rng: np.random.Generator, T: int, G: int, p: float,
                   min_one: bool = False) -> np.ndarray:
    m = rng.random((T, G), dtype=np.float32) < np.float32(p)
    if min_one:
        for t in range(T):
            while not m[t].any():
                m[t] = rng.random(G, dtype=np.float32) < np.float32(p)
    return m


def prototype_masks(seed: int, T: int, groups: list[tuple[str, int]],
                    n_proto: int, keep: float, flip: float,
                    extra: tuple = ()) -> dict[str, np.ndarray]:
    """Masks drawn around ``n_proto`` prototypes.

    Each prototype keeps exactly round(keep*G) groups of every group set
    (chosen uniformly without replacement); each token picks one prototype
    uniformly (the same index for all group sets); each bit is then flipped
    independently with probability ``flip`` (no flips when keep == 1.0).
    """
    pick = _rng(seed, "proto_pick", *extra).integers(0, n_proto, size=T)
    out = {}
    for name, G in groups:
        kind = name[-1]  # "f" or "a"
        prng = _rng(seed, "proto_" + kind, *extra)
        nk = int(round(keep * G))
        protos = np.zeros((n_proto, G), dtype=bool)
        for p in range(n_proto):
            protos[p, prng.choice(G, size=nk, replace=False)] = True
        m = protos[pick].copy()
        if keep < 1.0 and flip > 0.0:
            fl = _rng(seed, "flip_" + kind, *extra).random((T, G), dtype=np.float32) < np.float32(flip)
            m ^= fl
        out[name] = m
    out["pick"] = pick
    return out


@dataclasses.dataclass
class FFNCase:
    """Masked SwiGLU FFN inputs.  bf16 tensors are uint16 bit arrays."""
    name: str
    T: int
    H: int
    I: int
    gs: int
    dtype: str                 # "bf16" or "f32"
    x: np.ndarray              # [T][H]
    w_gate: np.ndarray         # [I][H]
    w_up: np.ndarray           # [I][H]
    w_down: np.ndarray         # [H][I]
    mask: np.ndarray           # bool [T][G]

    @property
    def G(self) -> int:
        return self.I // self.gs

    @property
    def mask_words(self) -> np.ndarray:
        return pack_mask(self.mask)


@dataclasses.dataclass
class AttnCase:
    """Masked GQA attention inputs (one layer's attention half)."""
    name: str
    mode: str                  # "decode" or "prefill"
    n_seq: int
    seq_len: int               # new tokens per sequence (1 for decode)
    cache_len: int             # past positions already in the cache
    H: int
    n_q: int
    n_kv: int
    hd: int
    theta: float
    eps: float
    x: np.ndarray              # [T][H] bf16 bits (layer input, before RMSNorm)
    gamma1: np.ndarray         # [H] bf16 bits
    wq: np.ndarray             # [n_q*hd][H]
    wk: np.ndarray             # [n_kv*hd][H]
    wv: np.ndarray             # [n_kv*hd][H]
    wo: np.ndarray             # [H][n_q*hd]
    k_cache: Optional[np.ndarray]  # [n_seq][n_kv][cache_len][hd] or None
    v_cache: Optional[np.ndarray]
    mask: np.ndarray           # bool [T][n_kv]

    @property
    def T(self) -> int:
        return self.n_seq * self.seq_len

    @property
    def mask_words(self) -> np.ndarray:
        return pack_mask(self.mask)

    @property
    def positions(self) -> np.ndarray:
        """Position of every new token inside its sequence (int32 [T])."""
        p = np.arange(self.seq_len, dtype=np.int32) + np.int32(self.cache_len)
        return np.tile(p, self.n_seq)


@dataclasses.dataclass
class LayerCase:
    attn: AttnCase
    ffn: FFNCase               # ffn.x is unused (the FFN input is computed)
    gamma2: np.ndarray         # [H] bf16 bits

    @property
    def T(self) -> int:
        return self.attn.T


def tiny_ffn(seed: int = 0) -> FFNCase:
    T, H, I, gs = 64, 256, 1024, 64
    return FFNCase(
        "tiny_ffn_f32", T, H, I, gs, "f32",
        x=_normal(seed, "x", (T, H), 1.0, False),
        w_gate=_normal(seed, "w_gate", (I, H), 0.02, False),
        w_up=_normal(seed, "w_up", (I, H), 0.02, False),
        w_down=_normal(seed, "w_down", (H, I), 0.02, False),
        mask=bernoulli_mask(_rng(seed, "mask_f"), T, I // gs, 0.5, min_one=True),
    )


def ffn_case(T: int, H: int, I: int, gs: int, seed: int = 0, keep: float = 0.5,
             dtype: str = "bf16", mask_kind: str = "bernoulli",
             n_proto: int = 8, flip: float = 0.1, name: str = "ffn") -> FFNCase:
    """A generic masked-FFN case (any size), used by parity tests."""
    bf = dtype == "bf16"
    G = I // gs
    if mask_kind == "bernoulli":
        mask = bernoulli_mask(_rng(seed, "mask_f", T, G), T, G, keep)
    elif mask_kind == "prototype":
        mask = prototype_masks(seed, T, [("mask_f", G)], n_proto, keep, flip, extra=(T, G))["mask_f"]
    elif mask_kind == "ones":
        mask = np.ones((T, G), dtype=bool)
    elif mask_kind == "zeros":
        mask = np.zeros((T, G), dtype=bool)
    else:
        raise ValueError(mask_kind)
    return FFNCase(
        name, T, H, I, gs, dtype,
        x=_normal(seed, "x", (T, H), 1.0, bf, T, H),
        w_gate=_normal(seed, "w_gate", (I, H), 0.02, bf, I, H),
        w_up=_normal(seed, "w_up", (I, H), 0.02, bf, I, H),
        w_down=_normal(seed, "w_down", (H, I), 0.02, bf, H, I),
        mask=mask,
    )


def decode_ffn(batch: int, seed: int = 0, weights: bool = True) -> FFNCase:
    """Llama-3.2-3B-shaped decode FFN; weights independent of the batch size
    (``weights=False`` leaves them as None, for a batch that reuses them)."""
    H, I, gs = 3072, 8192, 128
    return FFNCase(
        f"decode_ffn_3b_b{batch}", batch, H, I, gs, "bf16",
        x=_normal(seed, "x", (batch, H), 1.0, True, batch),
        w_gate=_normal(seed, "w_gate", (I, H), 0.02) if weights else None,
        w_up=_normal(seed, "w_up", (I, H), 0.02) if weights else None,
        w_down=_normal(seed, "w_down", (H, I), 0.02) if weights else None,
        mask=bernoulli_mask(_rng(seed, "mask_f", batch), batch, I // gs, 0.5),
    )


def _ffn_8b_weights(seed):
    H, I = 4096, 14336
    return (_normal(seed, "w_gate", (I, H), 0.02),
            _normal(seed, "w_up", (I, H), 0.02),
            _normal(seed, "w_down", (H, I), 0.02))


def prefill_ffn(seed: int = 0, T: int = 4096) -> FFNCase:
    """Llama-3.1-8B-shaped prefill FFN with 8 prototype masks (56 of 112 kept)."""
    H, I, gs = 4096, 14336, 128
    wg, wu, wd = _ffn_8b_weights(seed)
    m = prototype_masks(seed, T, [("mask_f", I // gs)], 8, 0.5, 0.1, extra=(T,))["mask_f"]
    return FFNCase("prefill_ffn_8b", T, H, I, gs, "bf16",
                   x=_normal(seed, "x", (T, H), 1.0, True, T),
                   w_gate=wg, w_up=wu, w_down=wd, mask=m)


def _attn_weights(seed, H=4096, n_q=32, n_kv=8, hd=128):
    return dict(
        wq=_normal(seed, "wq", (n_q * hd, H), 0.02),
        wk=_normal(seed, "wk", (n_kv * hd, H), 0.02),
        wv=_normal(seed, "wv", (n_kv * hd, H), 0.02),
        wo=_normal(seed, "wo", (H, n_q * hd), 0.02),
    )


def _gamma(seed, name, H):
    g = np.float32(1.0) + np.float32(0.02) * _rng(seed, name).standard_normal(H, dtype=np.float32)
    return bf16_bits_from_f32(g)


def decode_layer(seed: int = 0, batch: int = 16, cache_len: int = 2048,
                 keep_a: float = 0.34, keep_f: float = 0.72) -> LayerCase:
    H, n_q, n_kv, hd = 4096, 32, 8, 128
    I, gs = 14336, 128
    x = _normal(seed, "x", (batch, H), 1.0, True, batch, 1)
    attn = AttnCase(
        "decode_layer_8b", "decode", batch, 1, cache_len, H, n_q, n_kv, hd, 5e5, 1e-5,
        x=x, gamma1=_gamma(seed, "gamma1", H), **_attn_weights(seed),
        k_cache=_normal(seed, "k_cache", (batch, n_kv, cache_len, hd), 1.0, True, batch, cache_len),
        v_cache=_normal(seed, "v_cache", (batch, n_kv, cache_len, hd), 1.0, True, batch, cache_len),
        mask=bernoulli_mask(_rng(seed, "mask_a", batch), batch, n_kv, keep_a),
    )
    wg, wu, wd = _ffn_8b_weights(seed)
    ffn = FFNCase("decode_layer_8b_ffn", batch, H, I, gs, "bf16", x=x,
                  w_gate=wg, w_up=wu, w_down=wd,
                  mask=bernoulli_mask(_rng(seed, "mask_f", batch, 1), batch, I // gs, keep_f))
    return LayerCase(attn, ffn, _gamma(seed, "gamma2", H))


def prefill_layer(seed: int = 0, keep: float = 0.5, n_seq: int = 4,
                  seq_len: int = 2048) -> LayerCase:
    H, n_q, n_kv, hd = 4096, 32, 8, 128
    I, gs = 14336, 128
    T = n_seq * seq_len
    kcode = int(round(keep * 100))
    x = _normal(seed, "x", (T, H), 1.0, True, T, 2)
    m = prototype_masks(seed, T, [("mask_a", n_kv), ("mask_f", I // gs)], 16, keep, 0.1,
                        extra=(T, kcode))
    attn = AttnCase(
        f"prefill_layer_8b_k{kcode}", "prefill", n_seq, seq_len, 0, H, n_q, n_kv, hd, 5e5, 1e-5,
        x=x, gamma1=_gamma(seed, "gamma1", H), **_attn_weights(seed),
        k_cache=None, v_cache=None, mask=m["mask_a"],
    )
    wg, wu, wd = _ffn_8b_weights(seed)
    ffn = FFNCase(f"prefill_layer_8b_k{kcode}_ffn", T, H, I, gs, "bf16", x=x,
                  w_gate=wg, w_up=wu, w_down=wd, mask=m["mask_f"])
    return LayerCase(attn, ffn, _gamma(seed, "gamma2", H))


def small_layer(mode: str, seed: int = 0, n_seq: int = 2, seq_len: int = 1,
                cache_len: int = 64, H: int = 256, n_q: int = 8, n_kv: int = 2,
                hd: int = 32, I: int = 512, gs: int = 64, keep_a: float = 0.5,
                keep_f: float = 0.5) -> LayerCase:
    """A reduced layer of the same structure, for fast oracle/parity tests."""
    T = n_seq * seq_len
    x = _normal(seed, "x", (T, H), 1.0, True, T, H, 3)
    wq = _normal(seed, "wq", (n_q * hd, H), 0.02, True, H, 1)
    wk = _normal(seed, "wk", (n_kv * hd, H), 0.02, True, H, 1)
    wv = _normal(seed, "wv", (n_kv * hd, H), 0.02, True, H, 1)
    wo = _normal(seed, "wo", (H, n_q * hd), 0.02, True, H, 1)
    kc = vc = None
    if mode == "decode" and cache_len > 0:
        kc = _normal(seed, "k_cache", (n_seq, n_kv, cache_len, hd), 1.0, True, n_seq, cache_len, 1)
        vc = _normal(seed, "v_cache", (n_seq, n_kv, cache_len, hd), 1.0, True, n_seq, cache_len, 1)
    attn = AttnCase(f"small_{mode}", mode, n_seq, seq_len, cache_len if mode == "decode" else 0,
                    H, n_q, n_kv, hd, 5e5, 1e-5, x=x, gamma1=_gamma(seed, "gamma1", H),
                    wq=wq, wk=wk, wv=wv, wo=wo, k_cache=kc, v_cache=vc,
                    mask=bernoulli_mask(_rng(seed, "mask_a", T, 7), T, n_kv, keep_a))
    ffn = FFNCase(f"small_{mode}_ffn", T, H, I, gs, "bf16", x=x,
                  w_gate=_normal(seed, "w_gate", (I, H), 0.02, True, I, H, 3),
                  w_up=_normal(seed, "w_up", (I, H), 0.02, True, I, H, 3),
                  w_down=_normal(seed, "w_down", (H, I), 0.02, True, H, I, 3),
                  mask=bernoulli_mask(_rng(seed, "mask_f", T, 7), T, I // gs, keep_f))
    g2 = _gamma(seed, "gamma2", H)
    return LayerCase(attn, ffn, g2)


CONFIGS = {
    "tiny_ffn_f32": "fp32 masked SwiGLU FFN, T=64 H=256 I=1024, 16 groups of 64, Bernoulli(0.5), >=1 kept group/token",
    "decode_ffn_3b": "bf16 decode FFN, H=3072 I=8192, 64 groups of 128, batch 1/8/32, Bernoulli(0.5)",
    "prefill_ffn_8b": "bf16 prefill FFN, T=4096 H=4096 I=14336, 112 groups of 128, 8 prototypes (56 kept) + 0.1 flips",
    "decode_layer_8b": "bf16 decode layer, B=16, cache 2048, head groups Bernoulli(0.34), FFN groups Bernoulli(0.72)",
    "prefill_layer_8b": "bf16 prefill layer, 4 x 2048 tokens, 16 prototypes (8 head / 112 FFN groups), keep 0.25-1.0 + 0.1 flips",
}


@dataclasses.dataclass
class RouterCase:
    """Bottleneck router inputs.  bf16 tensors are uint16 bit arrays."""
    name: str
    T: int
    H: int
    R: int
    G: int
    act: str                   # "relu" or "silu"
    x: np.ndarray              # [T][H] bf16
    w_r1: np.ndarray           # [R][H] bf16
    w_r2: np.ndarray           # [G][R] bf16
    b_r2: Optional[np.ndarray]  # [G] fp32 or None


def router_case(T: int, H: int, R: int, G: int, seed: int = 0, act: str = "relu",
                bias_std: float = 0.0, name: str = "router") -> RouterCase:
    """Router weights depend on (seed, H, R, G) only, so decode and prefill
    batches of one model share them."""
    b = None
    if bias_std > 0.0:
        b = _rng(seed, "b_r2", G).standard_normal(G, dtype=np.float32) * np.float32(bias_std)
    return RouterCase(
        name, T, H, R, G, act,
        x=_normal(seed, "x", (T, H), 1.0, True, T, H),
        w_r1=_normal(seed, "w_r1", (R, H), 0.02, True, R, H),
        w_r2=_normal(seed, "w_r2", (G, R), 0.02, True, G, R),
        b_r2=b,
    )
