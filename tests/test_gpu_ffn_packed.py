"""The decode FFN on the packed weight layout (wide_ffn_pack +
wide_ffn_masked_packed) and the decode layer reading it, against the fp64
oracle.  WIDE, technical summary section 2.A: a token's skipped channel
groups contribute nothing; only the batch's union of groups is streamed.

The packing itself is a pure permutation, so it is checked bit for bit
against the layout the header states, written out with numpy."""
import numpy as np
import pytest

import synth
from oracle.ffn import ffn_masked, ffn_dense
from tests._util import rel_l2, ffn_to_dev, from_dev

pytestmark = pytest.mark.gpu

TOL = 5e-3   # relative L2: bf16 weights and h, fp32 accumulation


def _packed_run(c, pk=None):
    import torch
    import token_level_dynamic_b200 as w
    x, wg, wu, wd, m = ffn_to_dev(c)
    if pk is None:
        pk = w.wide_ffn_pack(wg, wu, wd)
    w.wide_clear_device_status()
    out = w.wide_ffn_masked_packed(x, pk, m, c.gs, c.I)
    torch.cuda.synchronize()
    assert w.wide_get_device_status() == 0
    return from_dev(out)


def _ref(c):
    return ffn_masked(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, c.gs, c.dtype)


def test_pack_is_the_stated_permutation():
    """W_gate / W_up interleaved: element [p][k][q][s][r][e] = (W_gate if
    s == 0 else W_up)[64p + 16q + r][64k + e]; W_down: element [c][n][e] =
    W_down[n][16c + e]; bitwise."""
    import torch
    import token_level_dynamic_b200 as w
    c = synth.ffn_case(4, 384, 640, 64, seed=1)
    H, I = c.H, c.I
    x, wg, wu, wd, m = ffn_to_dev(c)
    pk = w.wide_ffn_pack(wg, wu, wd)
    torch.cuda.synchronize()
    got = pk.cpu().numpy().view(np.uint16)
    g, u, d = (np.asarray(a, dtype=np.uint16) for a in (c.w_gate, c.w_up, c.w_down))
    mat = H * I
    gu = np.stack([g, u])                                     # [s][I][H]
    want_gu = gu.reshape(2, I // 64, 4, 16, H // 64, 64).transpose(1, 4, 2, 0, 3, 5).reshape(-1)
    want_d = d.reshape(H, I // 16, 16).transpose(1, 0, 2).reshape(-1)
    np.testing.assert_array_equal(got[:2 * mat], want_gu)
    np.testing.assert_array_equal(got[2 * mat:3 * mat], want_d)


@pytest.mark.parametrize("batch", [1, 8, 32])
def test_decode_ffn_3b_config(batch):
    c = synth.decode_ffn(batch)
    assert rel_l2(_packed_run(c), _ref(c)) <= TOL


def test_decode_layer_ffn_shape():
    c = synth.ffn_case(16, 4096, 14336, 128, seed=4, keep=0.72)
    assert rel_l2(_packed_run(c), _ref(c)) <= TOL


@pytest.mark.parametrize("T,H,I,gs", [
    (1, 128, 256, 64),        # one K step block, two output blocks short of a stage
    (3, 1152, 1024, 128),     # 18 K steps: the last 4-step stage is half out of range
    (7, 1280, 3072, 64),      # 10 output blocks: a partial W_down stage
    (17, 512, 2048, 32),      # group size 32, 17 tokens (TP = 32)
    (33, 256, 1024, 128),     # 33 tokens: a second launch of 1
    (70, 384, 768, 64),       # three launches (32 + 32 + 6)
    (16, 512, 8192, 256),     # group size 256
    (13, 256, 32768, 32),     # 1024 groups: several windows per CTA
])
def test_packed_shapes_and_token_counts(T, H, I, gs):
    c = synth.ffn_case(T, H, I, gs, seed=T + H, keep=0.5)
    assert rel_l2(_packed_run(c), _ref(c)) <= TOL


def test_all_zero_mask_gives_exact_zero():
    c = synth.ffn_case(8, 512, 1024, 128, seed=1, mask_kind="zeros")
    assert not np.any(_packed_run(c))


def test_all_ones_mask_equals_dense():
    c = synth.ffn_case(8, 512, 1024, 128, seed=2, mask_kind="ones")
    assert rel_l2(_packed_run(c), ffn_dense(c.x, c.w_gate, c.w_up, c.w_down)) <= TOL


def test_one_token_keeps_one_group():
    """Only token 19 keeps anything (group 3): every other row is exactly
    zero and the kept group is right."""
    c = synth.ffn_case(20, 512, 2048, 128, seed=9)
    c.mask[:] = False
    c.mask[19, 3] = True
    out = _packed_run(c)
    assert not np.any(out[:19])
    assert rel_l2(out, _ref(c)) <= TOL


def test_packed_matches_nn_linear_tensor_core_path():
    """The same kernel on the nn.Linear weights and on the packed copy: the
    sums are the same up to fp32 order (atomics), so the outputs agree to a
    bf16 step."""
    import torch
    import token_level_dynamic_b200 as w
    c = synth.decode_ffn(32)
    x, wg, wu, wd, m = ffn_to_dev(c)
    prev = w.wide_set_decode_ffn_path(w.WIDE_DECODE_TC)
    try:
        a = from_dev(w.wide_ffn_masked(x, wg, wu, wd, m, c.gs, path=w.WIDE_PATH_DECODE))
    finally:
        w.wide_set_decode_ffn_path(prev)
    b = from_dev(w.wide_ffn_masked_packed(x, w.wide_ffn_pack(wg, wu, wd), m, c.gs, c.I))
    torch.cuda.synchronize()
    assert rel_l2(a, b) <= 1e-3


def test_bad_mask_bit_sets_device_status():
    import torch
    import token_level_dynamic_b200 as w
    c = synth.ffn_case(2, 256, 1024, 128, seed=5)           # G = 8
    x, wg, wu, wd, m = ffn_to_dev(c)
    pk = w.wide_ffn_pack(wg, wu, wd)
    m[1, 0] |= 1 << 9
    w.wide_clear_device_status()
    w.wide_ffn_masked_packed(x, pk, m, c.gs, c.I)
    torch.cuda.synchronize()
    assert w.wide_get_device_status() & w.WIDE_DEV_BAD_MASK
    w.wide_clear_device_status()


def test_decode_layer_reads_the_packed_copy():
    """The 8B decode layer with ffn_packed given: same outputs as the
    oracle, and the tensor-core kernel is the one that ran."""
    import torch
    import token_level_dynamic_b200 as w
    from oracle.attention import layer_masked
    from tests._layer_util import layer_to_dev, layer_dims
    lc = synth.decode_layer()
    x, wts, kc, vc, hm, fm, cap = layer_to_dev(lc)
    wts = dict(wts)
    wts["ffn_packed"] = w.wide_ffn_pack(wts["w_gate"], wts["w_up"], wts["w_down"])
    d = layer_dims(lc, cap)
    w.wide_clear_device_status()
    ffn = torch.empty_like(x)
    w.wide_profile_start(1024)
    out = w.wide_layer_masked(x, wts, kc, vc, hm, fm, d, ffn_out=ffn)
    w.wide_profile_stop()
    names = {n for n, _ in w.wide_profile_read()}
    torch.cuda.synchronize()
    assert w.wide_get_device_status() == 0
    assert "decode_ffn_tcgen05" in names, names
    ref, p = layer_masked(lc, ret_parts=True)
    assert rel_l2(from_dev(ffn), p["ffn_out"]) <= TOL
    assert rel_l2(from_dev(out), ref) <= TOL


@pytest.mark.parametrize("T,kernel", [(1, "decode_ffn_split_gemv"), (8, "decode_ffn_split_gemv"),
                                      (16, "decode_ffn_tcgen05"), (32, "decode_ffn_tcgen05"),
                                      (40, None)])
def test_packed_with_linear_weights_picks_per_launch(T, kernel):
    """Given the nn.Linear weights too, the call runs the channel-split
    kernel for up to 8 tokens per launch and the tensor-core kernel on the
    packed copy above (40 tokens: one launch of each); the result is the
    oracle's either way."""
    import torch
    import token_level_dynamic_b200 as w
    c = synth.ffn_case(T, 3072, 8192, 128, seed=70 + T, keep=0.5)
    x, wg, wu, wd, m = ffn_to_dev(c)
    pk = w.wide_ffn_pack(wg, wu, wd)
    w.wide_clear_device_status()
    w.wide_profile_start(64)
    out = w.wide_ffn_masked_packed(x, pk, m, c.gs, c.I, weights=(wg, wu, wd))
    w.wide_profile_stop()
    names = [n for n, _ in w.wide_profile_read()]
    torch.cuda.synchronize()
    assert w.wide_get_device_status() == 0
    if kernel is None:
        assert names.count("decode_ffn_tcgen05") == 1 and names.count("decode_ffn_split_gemv") == 1
    else:
        assert names == [kernel], names
    assert rel_l2(from_dev(out), _ref(c)) <= TOL
