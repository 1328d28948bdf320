"""Pins for the attention / layer oracle (CPU only).

WIDE, technical summary section 2.A: attention prunes per-token groups of
query heads aligned with GQA.  The oracle's RMSNorm, RoPE and attention are
checked against closed forms (tests/golden), torch's scaled_dot_product_attention
(a library routine, float64), and invariants: decode must agree with prefill
on the same sequence, a skipped group removes exactly its o_proj term, and
masks of all zeros leave the residual stream untouched.
"""
import copy
import json
import os

import numpy as np
import pytest

import synth
from oracle.attention import rmsnorm, rope, attention_masked, layer_masked, layer_masked_rows
from oracle.ffn import widen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden():
    with open(os.path.join(GOLDEN, "rope_rmsnorm_closed_forms.json")) as f:
        return json.load(f)


def test_rmsnorm_closed_form():
    g = _golden()["rmsnorm"]
    y = rmsnorm(np.array(g["x"]), np.array(g["gamma"]), g["eps"])
    np.testing.assert_allclose(y, g["y"], rtol=0, atol=1e-15)


def test_rope_closed_forms_and_identity_at_zero():
    g = _golden()["rope"]
    for c in g["cases"]:
        out = rope(np.array([c["v"]], dtype=np.float64), np.array([g["pos"]]), g["theta"])
        np.testing.assert_allclose(out[0], c["out"], rtol=0, atol=1e-15)
    v = np.random.default_rng(0).standard_normal((3, 128))
    np.testing.assert_array_equal(rope(v, np.zeros(3), 5e5), v)


def test_rope_is_a_rotation_with_relative_phase():
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal((1, 128)), rng.standard_normal((1, 128))
    m, n = 1234, 777
    qm, kn = rope(q, np.array([m]), 5e5), rope(k, np.array([n]), 5e5)
    np.testing.assert_allclose(np.linalg.norm(qm), np.linalg.norm(q), rtol=1e-13)
    rel = rope(q, np.array([m - n]), 5e5)
    np.testing.assert_allclose(qm @ kn.T, rel @ k.T, rtol=1e-9)


def _sdpa_reference(case):
    """Dense (all groups kept) attention via torch SDPA in float64."""
    import torch
    c = case
    _, parts = attention_masked(c, ret_parts=True)
    q, k, v = (torch.from_numpy(parts[n]) for n in ("q", "k", "v"))
    S, rep = c.seq_len, c.n_q // c.n_kv
    outs = []
    for b in range(c.n_seq):
        rows = slice(b * S, (b + 1) * S)
        qb = q[rows].transpose(0, 1)                                   # [nq][S][hd]
        kb, vb = k[rows].transpose(0, 1), v[rows].transpose(0, 1)
        if c.mode == "decode":
            kb = torch.cat([torch.from_numpy(widen(c.k_cache[b], "bf16")), kb], dim=1)
            vb = torch.cat([torch.from_numpy(widen(c.v_cache[b], "bf16")), vb], dim=1)
        kb = kb.repeat_interleave(rep, dim=0)
        vb = vb.repeat_interleave(rep, dim=0)
        o = torch.nn.functional.scaled_dot_product_attention(
            qb[None], kb[None], vb[None], is_causal=(c.mode == "prefill"))[0]
        outs.append(o.transpose(0, 1))
    o = torch.cat(outs, 0).reshape(c.T, -1)
    return (o @ torch.from_numpy(widen(c.wo, "bf16")).T).numpy()


@pytest.mark.parametrize("mode,kw", [("decode", dict(n_seq=3, cache_len=40)),
                                     ("prefill", dict(n_seq=2, seq_len=24))])
def test_all_groups_kept_equals_library_attention(mode, kw):
    lc = synth.small_layer(mode, seed=4, keep_a=1.0, **kw)
    lc.attn.mask[:] = True
    ours = attention_masked(lc.attn)
    np.testing.assert_allclose(ours, _sdpa_reference(lc.attn), rtol=1e-10, atol=1e-12)


def test_zero_queries_average_visible_values():
    """q = 0 makes every score equal, so each head returns the mean of the V
    rows it may see (closed form)."""
    lc = synth.small_layer("prefill", seed=2, n_seq=1, seq_len=10, keep_a=1.0)
    a = lc.attn
    a.mask[:] = True
    a.wq = np.zeros_like(a.wq)
    _, parts = attention_masked(a, ret_parts=True)
    v = parts["v"]                                                     # [T][nkv][hd]
    rep = a.n_q // a.n_kv
    for t in range(a.T):
        for h in range(a.n_q):
            np.testing.assert_allclose(parts["o"][t, h], v[:t + 1, h // rep].mean(axis=0),
                                       rtol=1e-12, atol=1e-14)


def test_skipped_group_removes_exactly_its_oproj_term():
    lc = synth.small_layer("decode", seed=6, n_seq=2, cache_len=16, keep_a=1.0)
    a = lc.attn
    a.mask[:] = True
    full, parts = attention_masked(a, ret_parts=True)
    b = copy.deepcopy(a)
    t, j = 1, 1
    b.mask[t, j] = False
    part = attention_masked(b)
    rep, hd = a.n_q // a.n_kv, a.hd
    cols = slice(j * rep * hd, (j + 1) * rep * hd)
    term = parts["o"][t].reshape(-1)[cols] @ widen(a.wo, "bf16")[:, cols].T
    np.testing.assert_array_equal(full[0], part[0])
    np.testing.assert_allclose(full[t] - part[t], term, rtol=1e-9, atol=1e-13)


def test_decode_agrees_with_prefill_on_the_same_sequence():
    """Prefill over L+1 tokens, then decode the last token against the
    prefill's own (post-RoPE) K/V of the first L tokens: same output."""
    L = 12
    lp = synth.small_layer("prefill", seed=8, n_seq=1, seq_len=L + 1, keep_a=0.6, keep_f=0.6)
    out_p, parts = layer_masked(lp, ret_parts=True)
    a = lp.attn
    kc = synth.bf16_bits_from_f32(parts["k"][:L].transpose(1, 0, 2)[None].astype(np.float32))
    vc = synth.bf16_bits_from_f32(parts["v"][:L].transpose(1, 0, 2)[None].astype(np.float32))
    dec = copy.deepcopy(lp)
    d = dec.attn
    d.mode, d.seq_len, d.cache_len = "decode", 1, L
    d.x = a.x[L:L + 1]
    d.mask = a.mask[L:L + 1]
    d.k_cache, d.v_cache = kc, vc
    dec.ffn.mask = lp.ffn.mask[L:L + 1]
    dec.ffn.T = 1
    out_d = layer_masked(dec)
    # the cache went through bf16, so agreement is to bf16 rounding of K/V
    np.testing.assert_allclose(out_d[0], out_p[L], rtol=0, atol=2e-2 * np.abs(out_p[L]).max())
    # and exactly when the prefill K/V are themselves representable in bf16
    assert np.linalg.norm(out_d[0] - out_p[L]) / np.linalg.norm(out_p[L]) < 5e-3


def test_all_masks_zero_leave_residual():
    lc = synth.small_layer("decode", seed=3, n_seq=4, cache_len=8)
    lc.attn.mask[:] = False
    lc.ffn.mask[:] = False
    out = layer_masked(lc)
    np.testing.assert_array_equal(out, widen(lc.attn.x, "bf16"))


def test_sequence_permutation_in_decode():
    lc = synth.small_layer("decode", seed=5, n_seq=4, cache_len=8)
    p = np.array([2, 0, 3, 1])
    out = layer_masked(lc)
    q = copy.deepcopy(lc)
    q.attn.x, q.attn.mask = lc.attn.x[p], lc.attn.mask[p]
    q.attn.k_cache, q.attn.v_cache = lc.attn.k_cache[p], lc.attn.v_cache[p]
    q.ffn.mask = lc.ffn.mask[p]
    np.testing.assert_array_equal(layer_masked(q), out[p])


@pytest.mark.parametrize("mode,kw", [("prefill", dict(n_seq=3, seq_len=20)),
                                     ("decode", dict(n_seq=5, cache_len=30))])
def test_row_form_equals_full_layer(mode, kw):
    """The per-row form (used for full-size sampled checks) is the same
    definition: it matches the full layer on every row."""
    lc = synth.small_layer(mode, seed=21, **kw)
    full, parts = layer_masked(lc, ret_parts=True)
    rows = np.arange(lc.attn.T)[::2]
    out, rp = layer_masked_rows(lc, rows)
    np.testing.assert_allclose(out, full[rows], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(rp["attn_out"], parts["attn_out"][rows], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(rp["k"], parts["k"], rtol=1e-12, atol=1e-13)
