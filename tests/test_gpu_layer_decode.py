"""Decode masked layer (attention half + FFN) against the fp64 oracle.

WIDE, technical summary section 2.A: per-token GQA head groups and FFN
channel groups; a skipped head group computes no query heads, reads no K/V
and its o_proj columns; K/V are appended for every token."""
import numpy as np
import pytest

import synth
from oracle.attention import layer_masked
from tests._util import rel_l2, from_dev
from tests._layer_util import layer_to_dev, layer_dims

pytestmark = pytest.mark.gpu

TOL = 5e-3


def _run(lc, attn_only=False):
    import torch
    import token_level_dynamic_b200 as w
    x, wts, kc, vc, hm, fm, cap = layer_to_dev(lc)
    d = layer_dims(lc, cap)
    w.wide_clear_device_status()
    attn = torch.empty_like(x)
    ffn = torch.empty_like(x)
    if attn_only:
        w.wide_attn_masked(x, wts, kc, vc, hm, d, attn_out=attn)
        out = None
    else:
        out = w.wide_layer_masked(x, wts, kc, vc, hm, fm, d, attn_out=attn, ffn_out=ffn)
    torch.cuda.synchronize()
    assert w.wide_get_device_status() == 0
    res = {"attn_out": from_dev(attn), "k": from_dev(kc), "v": from_dev(vc)}
    if not attn_only:
        res.update({"out": from_dev(out), "ffn_out": from_dev(ffn)})
    return res


def _check(lc, got, parts=("attn_out", "ffn_out", "out")):
    ref, p = layer_masked(lc, ret_parts=True)
    p["out"] = ref
    for name in parts:
        e = rel_l2(got[name], p[name])
        assert e <= TOL, (name, e)
    a = lc.attn
    # the appended K/V at position cache_len (k after RoPE)
    pos = a.cache_len
    k_new = got["k"][:, :, pos, :]
    v_new = got["v"][:, :, pos, :]
    assert rel_l2(k_new, p["k"]) <= TOL
    assert rel_l2(v_new, p["v"]) <= TOL
    # the old cache entries are untouched
    if a.cache_len:
        np.testing.assert_array_equal(
            got["k"][:, :, :pos], synth.f32_from_bf16_bits(a.k_cache).astype(np.float64))


@pytest.mark.parametrize("n_q,n_kv", [(8, 2), (4, 2), (4, 4)])
def test_decode_layer_small(n_q, n_kv):
    lc = synth.small_layer("decode", seed=n_q + n_kv, n_seq=5, cache_len=100, H=512, n_q=n_q,
                           n_kv=n_kv, hd=128, I=1024, gs=128, keep_a=0.5, keep_f=0.5)
    _check(lc, _run(lc))


def test_decode_layer_ragged_cache_and_batch():
    lc = synth.small_layer("decode", seed=11, n_seq=17, cache_len=37, H=1024, n_q=8, n_kv=2,
                           hd=128, I=2048, gs=64, keep_a=0.34, keep_f=0.72)
    _check(lc, _run(lc))


@pytest.mark.parametrize("cache_len,n_q,n_kv", [(127, 8, 2), (128, 4, 4), (300, 4, 2), (1000, 8, 2)])
def test_decode_layer_key_slices(cache_len, n_q, n_kv):
    """Caches that span several 128-key attention slices, with a ragged last
    slice (cache_len + 1 keys), for 4, 1 and 2 query heads per group."""
    lc = synth.small_layer("decode", seed=cache_len, n_seq=6, cache_len=cache_len, H=512,
                           n_q=n_q, n_kv=n_kv, hd=128, I=1024, gs=128, keep_a=0.5, keep_f=0.5)
    _check(lc, _run(lc))


def test_decode_attention_long_cache_many_slices():
    """A 70000-entry cache: hundreds of key slices merged by the last one."""
    lc = synth.small_layer("decode", seed=23, n_seq=2, cache_len=70000, H=512, n_q=4, n_kv=1,
                           hd=128, I=1024, gs=128, keep_a=1.0, keep_f=0.5)
    _check(lc, _run(lc, attn_only=True), parts=("attn_out",))


def test_decode_layer_repeated_calls_reuse_workspace():
    """Two calls in a row on one workspace give the same attention output
    (the slice counters are reset between calls)."""
    import torch
    import token_level_dynamic_b200 as w
    lc = synth.small_layer("decode", seed=21, n_seq=4, cache_len=400, H=512, n_q=8, n_kv=2,
                           hd=128, I=1024, gs=128, keep_a=0.7, keep_f=0.5)
    x, wts, kc, vc, hm, fm, cap = layer_to_dev(lc)
    d = layer_dims(lc, cap)
    ws = torch.full((w.wide_layer_workspace_bytes(d),), 0xAB, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(2):
        attn = torch.empty_like(x)
        w.wide_attn_masked(x, wts, kc, vc, hm, d, attn_out=attn, workspace=ws)
        outs.append(from_dev(attn))
    torch.cuda.synchronize()
    assert w.wide_get_device_status() == 0
    np.testing.assert_array_equal(outs[0], outs[1])
    ref, p = layer_masked(lc, ret_parts=True)
    assert rel_l2(outs[0], p["attn_out"]) <= TOL


def test_decode_layer_empty_cache():
    lc = synth.small_layer("decode", seed=12, n_seq=3, cache_len=0, H=512, n_q=8, n_kv=2,
                           hd=128, I=1024, gs=128)
    _check(lc, _run(lc))


def test_all_head_groups_skipped_gives_zero_attention_but_appends_kv():
    lc = synth.small_layer("decode", seed=13, n_seq=4, cache_len=20, H=512, n_q=8, n_kv=2,
                           hd=128, I=1024, gs=128)
    lc.attn.mask[:] = False
    got = _run(lc)
    assert not np.any(got["attn_out"])
    _check(lc, got, parts=("ffn_out", "out"))


def test_attention_only_entry_point_matches_layer():
    lc = synth.small_layer("decode", seed=14, n_seq=6, cache_len=64, H=512, n_q=8, n_kv=2,
                           hd=128, I=1024, gs=128)
    a = _run(lc, attn_only=True)
    b = _run(lc)
    np.testing.assert_array_equal(a["attn_out"], b["attn_out"])
    _check(lc, a, parts=("attn_out",))


def test_decode_layer_8b_full_config():
    """The Llama-3.1-8B-shaped decode layer: batch 16, cache 2048, head
    groups Bernoulli(0.34), FFN groups Bernoulli(0.72)."""
    lc = synth.decode_layer()
    _check(lc, _run(lc))


@pytest.mark.parametrize("mode", ["gemv", "fused"])
def test_decode_layer_on_cuda_core_kernels(mode):
    """The 8B decode layer with the decode mode forcing CUDA-core kernels
    (o_proj on the GEMV, the FFN on the GEMVs or the channel-split kernel):
    the same oracle outputs as the default tensor-core path."""
    import token_level_dynamic_b200 as w
    prev = w.wide_set_decode_ffn_path(w.WIDE_DECODE_GEMV if mode == "gemv" else w.WIDE_DECODE_FUSED)
    try:
        lc = synth.decode_layer()
        _check(lc, _run(lc))
    finally:
        w.wide_set_decode_ffn_path(prev)
