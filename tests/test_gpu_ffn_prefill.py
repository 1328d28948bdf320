"""Prefill (tcgen05) masked FFN against the fp64 oracle, through the C ABI.

WIDE, technical summary sections 2.B/2.C: groups run as dense tensor-core
tiles over their reordered active-token prefixes; tiles with no active token
are never issued; the down projection visits only the groups some token of a
signature tile keeps."""
import numpy as np
import pytest

import synth
from oracle.ffn import ffn_masked, ffn_dense
from tests._util import rel_l2, ffn_to_dev, from_dev

pytestmark = pytest.mark.gpu

TOL = 5e-3


def _run(c, x=None):
    import torch
    import token_level_dynamic_b200 as w
    x_, wg, wu, wd, m = ffn_to_dev(c)
    w.wide_clear_device_status()
    out = w.wide_ffn_masked(x_ if x is None else x, wg, wu, wd, m, c.gs,
                            path=w.WIDE_PATH_PREFILL)
    torch.cuda.synchronize()
    assert w.wide_get_device_status() == 0
    return from_dev(out)


def _ref(c):
    return ffn_masked(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, c.gs)


@pytest.mark.parametrize("T,H,I,kind,keep", [
    (128, 256, 256, "bernoulli", 0.5),        # one full tile per group
    (300, 256, 512, "bernoulli", 0.5),        # ragged tails, 4 groups
    (1000, 512, 1024, "prototype", 0.5),      # prototype masks, several tiles
    (777, 768, 1408, "bernoulli", 0.3),       # 11 groups (one partial word)
    (513, 1024, 4352, "prototype", 0.25),     # 34 groups over two mask words
])
def test_prefill_parity_small(T, H, I, kind, keep):
    c = synth.ffn_case(T, H, I, 128, seed=T, keep=keep, mask_kind=kind)
    assert rel_l2(_run(c), _ref(c)) <= TOL


def test_prefill_single_token_and_tiny():
    for T in (1, 3, 5):
        c = synth.ffn_case(T, 256, 512, 128, seed=10 + T)
        assert rel_l2(_run(c), _ref(c)) <= TOL


def test_prefill_all_zero_mask_is_exact_zero():
    c = synth.ffn_case(200, 256, 512, 128, seed=3, mask_kind="zeros")
    assert not np.any(_run(c))


def test_prefill_all_ones_equals_dense():
    c = synth.ffn_case(260, 512, 1024, 128, seed=4, mask_kind="ones")
    assert rel_l2(_run(c), ffn_dense(c.x, c.w_gate, c.w_up, c.w_down)) <= TOL


def test_prefill_one_group_per_token():
    c = synth.ffn_case(333, 256, 1024, 128, seed=5)
    c.mask[:] = False
    c.mask[np.arange(c.T), np.arange(c.T) % c.G] = True
    assert rel_l2(_run(c), _ref(c)) <= TOL


def test_prefill_matches_decode_path():
    """Both paths compute the same masked FFN (different kernels)."""
    import torch
    import token_level_dynamic_b200 as w
    c = synth.ffn_case(32, 512, 1024, 128, seed=6)
    x, wg, wu, wd, m = ffn_to_dev(c)
    a = from_dev(w.wide_ffn_masked(x, wg, wu, wd, m, 128, path=w.WIDE_PATH_PREFILL))
    b = from_dev(w.wide_ffn_masked(x, wg, wu, wd, m, 128, path=w.WIDE_PATH_DECODE))
    torch.cuda.synchronize()
    assert rel_l2(a, b) <= TOL


def test_prefill_repeatable_bitwise():
    c = synth.ffn_case(400, 512, 1024, 128, seed=7, mask_kind="prototype")
    np.testing.assert_array_equal(_run(c), _run(c))


def test_prefill_ffn_8b_full_size_sampled():
    """The full Llama-3.1-8B-shaped prefill FFN (T=4096, H=4096, I=14336,
    8 prototypes + 0.1 flips), checked on 48 sampled tokens whose outputs
    the oracle computes one by one (tokens are independent)."""
    c = synth.prefill_ffn()
    out = _run(c)
    rows = np.random.default_rng(0).choice(c.T, 48, replace=False)
    sub = synth.FFNCase("s", len(rows), c.H, c.I, c.gs, "bf16", c.x[rows], c.w_gate, c.w_up,
                        c.w_down, c.mask[rows])
    assert rel_l2(out[rows], _ref(sub)) <= TOL
    assert np.isfinite(out).all()


@pytest.mark.parametrize("T,H,I,kind,keep", [
    (300, 256, 512, "bernoulli", 0.5),        # 8 groups of 64, ragged tails
    (1000, 512, 2048, "prototype", 0.5),      # 32 groups of 64, prototypes
    (513, 1024, 4352, "prototype", 0.25),     # 68 groups of 64 over three mask words
])
def test_prefill_group_size_64(T, H, I, kind, keep):
    """64-channel groups: the gate/up tiles are N = 128 (gate + up rows of
    one group) and the down projection visits one 64-column K stage per
    union group."""
    c = synth.ffn_case(T, H, I, 64, seed=T + 7, keep=keep, mask_kind=kind)
    assert rel_l2(_run(c), _ref(c)) <= TOL


def test_prefill_group_size_64_all_zero_and_dense():
    c = synth.ffn_case(200, 256, 512, 64, seed=13, mask_kind="zeros")
    assert not np.any(_run(c))
    c = synth.ffn_case(260, 512, 1024, 64, seed=14, mask_kind="ones")
    assert rel_l2(_run(c), ffn_dense(c.x, c.w_gate, c.w_up, c.w_down)) <= TOL


@pytest.mark.parametrize("T,H,I,kind,keep", [
    (300, 256, 512, "bernoulli", 0.5),        # 16 groups of 32, ragged tails
    (1000, 512, 2048, "prototype", 0.5),      # 64 groups of 32: two mask words
    (513, 1024, 4352, "prototype", 0.25),     # 136 groups of 32 over five mask words
    (1024, 2048, 8192, "bernoulli", 0.5),     # 256 groups of 32, wider hidden
])
def test_prefill_group_size_32(T, H, I, kind, keep):
    """32-channel groups: gate/up tiles are N = 64, and the down projection
    takes the groups in pairs (one 64-column stage per pair that some token
    of the tile keeps), zeroing each 32-channel half for the tokens that
    skip that half's group."""
    c = synth.ffn_case(T, H, I, 32, seed=T + 11, keep=keep, mask_kind=kind)
    assert rel_l2(_run(c), _ref(c)) <= TOL


def test_prefill_group_size_32_halves_of_a_pair():
    """Tokens keep only odd groups, or only even ones, or one half of a
    pair each: every pair's stage is loaded and the half a token skips is
    zeroed for it (an all-zero or a both-halves mistake shows here)."""
    c = synth.ffn_case(384, 512, 1024, 32, seed=21)         # 32 groups
    G = c.I // c.gs
    c.mask[:] = False
    c.mask[:128, 1::2] = True                  # odd groups only
    c.mask[128:256, 0::2] = True               # even groups only
    c.mask[256:, 5] = True                     # one half of pair 2
    c.mask[300:, 10] = True                    # the other tokens: pair 5's first half
    assert rel_l2(_run(c), _ref(c)) <= TOL
    assert G == 32


def test_prefill_group_size_32_all_zero_and_dense():
    c = synth.ffn_case(200, 256, 512, 32, seed=15, mask_kind="zeros")
    assert not np.any(_run(c))
    c = synth.ffn_case(260, 512, 1024, 32, seed=16, mask_kind="ones")
    assert rel_l2(_run(c), ffn_dense(c.x, c.w_gate, c.w_up, c.w_down)) <= TOL


@pytest.mark.parametrize("path", ["decode", "prefill"])
def test_empty_batch_is_a_no_op(path):
    """Zero tokens: the call succeeds, launches nothing that fails, and
    leaves the device status clear, on either path."""
    import torch
    import token_level_dynamic_b200 as w
    c = synth.ffn_case(4, 256, 512, 128, seed=3)
    _, wg, wu, wd, _ = ffn_to_dev(c)
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    m = torch.empty((0, 1), dtype=torch.int32, device="cuda")
    w.wide_clear_device_status()
    p = w.WIDE_PATH_DECODE if path == "decode" else w.WIDE_PATH_PREFILL
    out = w.wide_ffn_masked(x, wg, wu, wd, m, 128, path=p)
    torch.cuda.synchronize()
    assert out.shape == (0, 256)
    assert w.wide_get_device_status() == 0


def test_prefill_caller_worklist_reused():
    """A work list built once by wide_reorder from the mask and passed to
    wide_ffn_masked twice (and for a second input x) gives the oracle's
    result each time; the call does not reorder again."""
    import torch
    import token_level_dynamic_b200 as w
    c = synth.ffn_case(700, 512, 1024, 128, seed=21, mask_kind="prototype")
    x, wg, wu, wd, m = ffn_to_dev(c)
    wl = w.wide_reorder(m, c.G, 128)
    w.wide_clear_device_status()
    n0 = w.wide_launch_count()
    a = from_dev(w.wide_ffn_masked(x, wg, wu, wd, m, c.gs, path=w.WIDE_PATH_PREFILL,
                                   worklist=wl))
    per_call = w.wide_launch_count() - n0
    b = from_dev(w.wide_ffn_masked(x, wg, wu, wd, m, c.gs, path=w.WIDE_PATH_PREFILL,
                                   worklist=wl))
    x2 = torch.flip(x, dims=[1]).contiguous()
    c2 = synth.FFNCase("flipped", c.T, c.H, c.I, c.gs, "bf16", c.x[:, ::-1].copy(), c.w_gate,
                       c.w_up, c.w_down, c.mask)
    d = from_dev(w.wide_ffn_masked(x2, wg, wu, wd, m, c.gs, path=w.WIDE_PATH_PREFILL,
                                   worklist=wl))
    torch.cuda.synchronize()
    assert w.wide_get_device_status() == 0
    ref = _ref(c)
    assert rel_l2(a, ref) <= TOL
    np.testing.assert_array_equal(a, b)
    assert rel_l2(d, _ref(c2)) <= TOL
    # the internal path launches the reorder kernels on top of the GEMMs
    n1 = w.wide_launch_count()
    w.wide_ffn_masked(x, wg, wu, wd, m, c.gs, path=w.WIDE_PATH_PREFILL)
    assert w.wide_launch_count() - n1 > per_call
    # a work list for another shape is refused before any launch
    wl_other = w.wide_reorder(m[:-1].contiguous(), c.G, 128)
    with pytest.raises(ValueError, match="worklist was built for"):
        w.wide_ffn_masked(x, wg, wu, wd, m, c.gs, path=w.WIDE_PATH_PREFILL, worklist=wl_other)
