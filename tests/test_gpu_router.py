"""Bottleneck router (WIDE, technical summary section 2.A, router
architecture) on the GPU against the fp64 oracle, through the C ABI.  Both
kernels are covered: the cluster kernel on CUDA cores (up to 32 tokens) and
the tcgen05 kernel (more tokens).

The logits are floating point: relative L2 <= 1e-4 against the oracle (the
kernel keeps every intermediate in fp32; bf16 appears only in the stored
inputs).  The execute bits are an integer decision taken on floating point,
so they are checked in the kernel's own precision -- every bit equals
(kernel logit > 0) exactly -- and against the oracle wherever the oracle's
logit is further from 0 than a margin of 1e-3 x the logits' RMS, far above
the fp32 error of either side; the test also checks that such near-zero
logits are rare, so the comparison is not vacuous.
"""
import numpy as np
import pytest

import synth
from oracle.ffn import ffn_masked, mask_bool
from oracle.router import pack, route_logits
from tests._util import from_dev, rel_l2, to_dev

pytestmark = pytest.mark.gpu

TOL_LOGITS = 1e-4
MARGIN = 1e-3


def _dev(rc):
    x = to_dev(rc.x, "bf16")
    w1 = to_dev(rc.w_r1, "bf16")
    w2 = to_dev(rc.w_r2, "bf16")
    b = None if rc.b_r2 is None else to_dev(rc.b_r2, "f32")
    return x, w1, w2, b


def _route(rc, with_logits=True):
    import torch
    import token_level_dynamic_b200 as w
    x, w1, w2, b = _dev(rc)
    act = w.WIDE_ACT_RELU if rc.act == "relu" else w.WIDE_ACT_SILU
    # poison the outputs so that an unwritten word or logit shows
    words = torch.full((rc.T, (rc.G + 31) // 32), -1, dtype=torch.int32, device="cuda")
    lg = None
    if with_logits:
        lg = torch.full((rc.T, rc.G), float("nan"), dtype=torch.float32, device="cuda")
    w.wide_clear_device_status()
    w.wide_route(x, w1, w2, b, act, mask_words=words, logits=lg)
    torch.cuda.synchronize()
    assert w.wide_get_device_status() == 0
    m = words.cpu().numpy().view(np.uint32)
    return m, (None if lg is None else lg.cpu().numpy().astype(np.float64))


def _check(rc, m, lg):
    ref = route_logits(rc.x, rc.w_r1, rc.w_r2, rc.b_r2, rc.act)
    assert np.all(np.isfinite(lg))
    err = rel_l2(lg, ref)
    assert err <= TOL_LOGITS, err
    # decisions in the kernel's precision: bit-exact against its own logits
    np.testing.assert_array_equal(m, pack(lg > 0.0))
    # bits at or above G are zero
    if rc.G % 32:
        assert np.all(m[:, -1] >> np.uint32(rc.G % 32) == 0)
    # against the oracle away from the decision boundary
    rms = float(np.sqrt(np.mean(ref * ref)))
    clear = np.abs(ref) > MARGIN * rms
    assert clear.mean() > 0.99, clear.mean()
    got = mask_bool(m, rc.G)
    np.testing.assert_array_equal(got[clear], (ref > 0)[clear])
    return ref


@pytest.mark.parametrize("T,H,R,G,act,bias", [
    # up to 32 tokens: the cluster kernel (CUDA cores)
    (1, 256, 32, 8, "silu", 0.0),          # one token, one word
    (5, 1024, 256, 1024, "silu", 0.05),    # partial cluster, widest shapes
    (16, 4096, 128, 8, "relu", 0.0),       # decode batch, head-group router
    (32, 4096, 128, 112, "relu", 0.02),    # largest batch of the cluster kernel
    # more than 32 tokens: tcgen05
    (33, 4096, 128, 112, "relu", 0.02),    # one partial tile
    (127, 512, 64, 33, "relu", 0.05),      # one partial tile, two words
    (300, 256, 64, 40, "relu", 0.05),      # three tiles, ragged tail
    (384, 192, 96, 200, "silu", 0.02),     # three full tiles, 7 words
    (129, 128, 256, 1024, "relu", 0.0),    # widest bottleneck, most groups
    (257, 64, 32, 1, "silu", 0.1),         # narrowest shapes, one group
])
def test_router_matches_oracle(T, H, R, G, act, bias):
    rc = synth.router_case(T, H, R, G, seed=11, act=act, bias_std=bias)
    m, lg = _route(rc)
    _check(rc, m, lg)


def test_router_paths_agree_at_the_boundary():
    """Tokens 0..31 routed as a batch of 32 (cluster kernel) and as the first
    rows of a batch of 33 (tcgen05 kernel): same decisions away from the
    margin, logits within the tolerance of each other."""
    rc33 = synth.router_case(33, 2048, 64, 40, seed=14, bias_std=0.02)
    rc32 = synth.RouterCase(**{**rc33.__dict__})
    rc32.x, rc32.T = rc33.x[:32], 32
    m33, lg33 = _route(rc33)
    m32, lg32 = _route(rc32)
    assert rel_l2(lg32, lg33[:32]) <= TOL_LOGITS
    rms = float(np.sqrt(np.mean(lg33 * lg33)))
    clear = np.abs(lg33[:32]) > MARGIN * rms
    np.testing.assert_array_equal(mask_bool(m32, 40)[clear], mask_bool(m33[:32], 40)[clear])


def test_router_without_logits_output():
    rc = synth.router_case(200, 256, 64, 40, seed=12, bias_std=0.05)
    m1, lg = _route(rc, with_logits=True)
    m2, _ = _route(rc, with_logits=False)
    np.testing.assert_array_equal(m1, m2)


def test_router_empty_batch():
    import torch
    import token_level_dynamic_b200 as w
    rc = synth.router_case(1, 256, 32, 8, seed=1)
    x, w1, w2, b = _dev(rc)
    words = torch.empty((0, 1), dtype=torch.int32, device="cuda")
    w.wide_route(x[:0], w1, w2, b, mask_words=words)
    torch.cuda.synchronize()


@pytest.mark.parametrize("T", [16, 8192])
def test_router_8b_ffn_full_size(T):
    """The FFN router at the 8B prefill-layer (T = 8192) and decode (T = 16)
    sizes: hidden 4096, bottleneck 128, 112 groups; every output compared."""
    rc = synth.router_case(T, 4096, 128, 112, seed=0)
    m, lg = _route(rc)
    ref = _check(rc, m, lg)
    keep = float((ref > 0).mean())
    assert 0.3 < keep < 0.7, keep


def test_router_feeds_masked_ffn():
    """Router -> packed mask -> masked FFN, both on the GPU, against oracle
    router -> oracle FFN.  Tokens with a logit inside the decision margin are
    left out of the comparison (their masks may legitimately differ)."""
    import torch
    import token_level_dynamic_b200 as w
    T, H, I, gs = 256, 512, 2048, 128
    G = I // gs
    rc = synth.router_case(T, H, 64, G, seed=13, bias_std=0.02)
    fc = synth.ffn_case(T, H, I, gs, seed=13)
    x, w1, w2, b = _dev(rc)
    words = w.wide_route(x, w1, w2, b)
    out = w.wide_ffn_masked(x, to_dev(fc.w_gate, "bf16"), to_dev(fc.w_up, "bf16"),
                            to_dev(fc.w_down, "bf16"), words, gs)
    torch.cuda.synchronize()
    ref_lg = route_logits(rc.x, rc.w_r1, rc.w_r2, rc.b_r2)
    ref = ffn_masked(rc.x, fc.w_gate, fc.w_up, fc.w_down, pack(ref_lg > 0), gs)
    rms = float(np.sqrt(np.mean(ref_lg * ref_lg)))
    ok_rows = np.all(np.abs(ref_lg) > MARGIN * rms, axis=1)
    assert ok_rows.mean() > 0.9
    got = from_dev(out)
    assert rel_l2(got[ok_rows], ref[ok_rows]) <= 5e-3
    np.testing.assert_array_equal(words.cpu().numpy().view(np.uint32)[ok_rows],
                                  pack(ref_lg > 0)[ok_rows])
