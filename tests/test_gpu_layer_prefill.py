"""Prefill masked layer (tcgen05 Q/KV projections, causal attention on
compacted queries, tile-union o_proj, masked FFN) against the fp64 oracle.

WIDE, technical summary sections 2.A-2.C: per-token GQA head groups and FFN
channel groups; reordered so that each group's queries are one contiguous
range; skipped pairs computed nowhere."""
import numpy as np
import pytest

import synth
from oracle.attention import layer_masked, layer_masked_rows
from tests._util import rel_l2, from_dev
from tests._layer_util import layer_to_dev, layer_dims

pytestmark = pytest.mark.gpu

TOL = 5e-3


def _run(lc):
    import torch
    import token_level_dynamic_b200 as w
    x, wts, kc, vc, hm, fm, cap = layer_to_dev(lc)
    d = layer_dims(lc, cap)
    w.wide_clear_device_status()
    attn = torch.empty_like(x)
    ffn = torch.empty_like(x)
    out = w.wide_layer_masked(x, wts, kc, vc, hm, fm, d, attn_out=attn, ffn_out=ffn)
    torch.cuda.synchronize()
    assert w.wide_get_device_status() == 0
    return {"attn_out": from_dev(attn), "ffn_out": from_dev(ffn), "out": from_dev(out),
            "k": from_dev(kc), "v": from_dev(vc)}


def _kv_check(lc, got, k_ref, v_ref, tokens):
    a = lc.attn
    for t in tokens:
        b, i = divmod(int(t), a.seq_len)
        assert rel_l2(got["k"][b, :, i], k_ref[t]) <= TOL
        assert rel_l2(got["v"][b, :, i], v_ref[t]) <= TOL


def _check_full(lc, got, parts=("attn_out", "ffn_out", "out")):
    ref, p = layer_masked(lc, ret_parts=True)
    p["out"] = ref
    for name in parts:
        e = rel_l2(got[name], p[name])
        assert e <= TOL, (name, e)
    _kv_check(lc, got, p["k"], p["v"], range(lc.attn.T))


@pytest.mark.parametrize("n_q,n_kv,seq_len,n_seq", [(8, 2, 256, 2), (4, 2, 200, 3),
                                                    (8, 4, 130, 2)])
def test_prefill_layer_small(n_q, n_kv, seq_len, n_seq):
    lc = synth.small_layer("prefill", seed=seq_len + n_q, n_seq=n_seq, seq_len=seq_len, H=512,
                           n_q=n_q, n_kv=n_kv, hd=128, I=1024, gs=128, keep_a=0.5, keep_f=0.5)
    _check_full(lc, _run(lc))


def test_prefill_layer_prototype_masks():
    lc = synth.small_layer("prefill", seed=7, n_seq=2, seq_len=384, H=768, n_q=8, n_kv=2,
                           hd=128, I=1536, gs=128)
    m = synth.prototype_masks(7, lc.attn.T, [("mask_a", 2), ("mask_f", 12)], 4, 0.5, 0.1)
    lc.attn.mask, lc.ffn.mask = m["mask_a"], m["mask_f"]
    _check_full(lc, _run(lc))


def test_prefill_all_head_groups_skipped():
    lc = synth.small_layer("prefill", seed=8, n_seq=2, seq_len=150, H=512, n_q=8, n_kv=2,
                           hd=128, I=1024, gs=128)
    lc.attn.mask[:] = False
    got = _run(lc)
    assert not np.any(got["attn_out"])
    _check_full(lc, got, parts=("ffn_out", "out"))


def test_prefill_all_groups_kept():
    lc = synth.small_layer("prefill", seed=9, n_seq=2, seq_len=256, H=512, n_q=8, n_kv=2,
                           hd=128, I=1024, gs=128)
    lc.attn.mask[:] = True
    lc.ffn.mask[:] = True
    _check_full(lc, _run(lc))


def test_prefill_layer_ffn_group_size_32():
    """The prefill layer with 32-channel FFN groups (the down projection
    takes them in pairs)."""
    lc = synth.small_layer("prefill", seed=41, n_seq=2, seq_len=200, H=512, n_q=8, n_kv=2,
                           hd=128, I=1024, gs=32, keep_a=0.5, keep_f=0.5)
    _check_full(lc, _run(lc))


@pytest.mark.parametrize("keep", [0.25, 0.5, 0.75, 1.0])
def test_prefill_layer_8b_full_size_sampled(keep):
    """The Llama-3.1-8B-shaped prefill layer (4 sequences x 2048 tokens,
    16 prototypes + 0.1 flips) at every keep rate the benchmark sweeps
    (1.0: every group kept, no flips), checked on 24 sampled tokens (first,
    last and random positions of every sequence) and on the K/V the layer
    wrote for them."""
    lc = synth.prefill_layer(keep=keep)
    got = _run(lc)
    S = lc.attn.seq_len
    rng = np.random.default_rng(1)
    rows = []
    for b in range(lc.attn.n_seq):
        rows += [b * S, b * S + S - 1] + list(b * S + rng.choice(S, 4, replace=False))
    rows = np.array(sorted(set(rows)))
    ref, p = layer_masked_rows(lc, rows)
    assert rel_l2(got["out"][rows], ref) <= TOL
    assert rel_l2(got["attn_out"][rows], p["attn_out"]) <= TOL
    assert rel_l2(got["ffn_out"][rows], p["ffn_out"]) <= TOL
    _kv_check(lc, got, p["k"], p["v"], rows)
    assert np.isfinite(got["out"]).all()


def test_prefill_layer_ffn_group_size_64():
    """The layer with 64-channel FFN groups (gate/up tiles N = 128)."""
    lc = synth.small_layer("prefill", seed=31, n_seq=2, seq_len=256, H=512, n_q=8, n_kv=2,
                           hd=128, I=1024, gs=64, keep_a=0.5, keep_f=0.5)
    _check_full(lc, _run(lc))
