"""Pins for the FFN oracle (CPU only).

The oracle is checked against things it does not compute itself: a worked
closed-form example (tests/golden), an independent library implementation of
the dense layer (torch CPU, float64), the brute-force per-token loop, and the
invariants the method implies (WIDE, technical summary section 2.A: a skipped
channel group contributes nothing; section 2.B: reordering tokens must not
change any result).
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth
from oracle.ffn import ffn_masked, ffn_token_loop, widen, check_mask

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _worked():
    with open(os.path.join(GOLDEN, "ffn_worked_example.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("form", ["definition", "token_loop"])
def test_worked_example(form):
    ex = _worked()
    x = np.array([ex["x"]], dtype=np.float32)
    wg = np.array(ex["w_gate"], dtype=np.float32)
    wu = np.array(ex["w_up"], dtype=np.float32)
    wd = np.array(ex["w_down"], dtype=np.float32)
    for case in ex["cases"]:
        m = synth.pack_mask(np.array([case["mask"]], dtype=bool))
        f = ffn_masked if form == "definition" else ffn_token_loop
        out = f(x, wg, wu, wd, m, ex["gs"], "f32")
        np.testing.assert_allclose(out[0], case["out"], rtol=0, atol=1e-15)


def test_widen_bf16_exact():
    bits = np.array([0x3F80, 0xC020, 0x0001, 0x7F7F, 0x8000], dtype=np.uint16)
    v = widen(bits, "bf16")
    assert v[0] == 1.0 and v[1] == -2.5
    assert v[2] == 2.0 ** -133                      # smallest bf16 subnormal
    assert v[3] == (2 - 2.0 ** -7) * 2.0 ** 127      # largest finite bf16
    assert v[4] == 0.0 and np.signbit(v[4])


def _case(T=9, H=48, I=160, gs=16, seed=3, dtype="bf16", keep=0.5):
    return synth.ffn_case(T, H, I, gs, seed=seed, keep=keep, dtype=dtype)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(1, 16, 32, 16), (7, 64, 256, 32), (5, 40, 40 * 33, 40)])
def test_definition_equals_token_loop(dtype, shape):
    """Brute force on tiny inputs: the per-token loop over kept groups (C)
    equals the dense-then-mask definition (numpy) to fp64 rounding.  The last
    shape has G = 33 groups, so the mask spans two words."""
    T, H, I, gs = shape
    c = synth.ffn_case(T, H, I, gs, seed=11, dtype=dtype)
    a = ffn_masked(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, gs, dtype)
    b = ffn_token_loop(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, gs, dtype)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


def test_all_ones_equals_library_dense():
    """All-ones mask = the dense SwiGLU FFN computed by torch (float64)."""
    import torch
    c = _case(keep=1.0)
    c.mask[:] = True
    out = ffn_masked(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, c.gs)
    X = torch.from_numpy(widen(c.x, "bf16"))
    lin = torch.nn.functional.linear
    ref = lin(torch.nn.functional.silu(lin(X, torch.from_numpy(widen(c.w_gate, "bf16")))) *
              lin(X, torch.from_numpy(widen(c.w_up, "bf16"))),
              torch.from_numpy(widen(c.w_down, "bf16"))).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-15)


def test_all_zero_mask_is_exactly_zero():
    c = _case()
    c.mask[:] = False
    assert not np.any(ffn_masked(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, c.gs))
    assert not np.any(ffn_token_loop(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, c.gs))


def test_removing_one_group_removes_exactly_its_term():
    """Zeroing (t, g) changes only token t's output, by exactly
    -h[t, g-slab] W_down[:, g-slab]^T, with h = silu(gate) * up."""
    import torch
    c = _case(T=6, H=32, I=128, gs=16, seed=5, keep=0.6)
    t, g = 2, int(np.flatnonzero(c.mask[2])[0])
    full = ffn_masked(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, c.gs)
    m2 = c.mask.copy()
    m2[t, g] = False
    part = ffn_masked(c.x, c.w_gate, c.w_up, c.w_down, synth.pack_mask(m2), c.gs)
    others = [i for i in range(c.T) if i != t]
    np.testing.assert_array_equal(full[others], part[others])
    sl = slice(g * c.gs, (g + 1) * c.gs)
    X = torch.from_numpy(widen(c.x[t:t + 1], "bf16"))
    a = X @ torch.from_numpy(widen(c.w_gate[sl], "bf16")).T
    b = X @ torch.from_numpy(widen(c.w_up[sl], "bf16")).T
    term = (torch.nn.functional.silu(a) * b) @ torch.from_numpy(widen(c.w_down[:, sl], "bf16")).T
    np.testing.assert_allclose(full[t] - part[t], term.numpy()[0], rtol=1e-9, atol=1e-15)


def test_token_permutation_permutes_output():
    c = _case(T=12, seed=7)
    p = np.random.default_rng(1).permutation(c.T)
    a = ffn_masked(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, c.gs)
    b = ffn_masked(c.x[p], c.w_gate, c.w_up, c.w_down, c.mask_words[p], c.gs)
    np.testing.assert_array_equal(a[p], b)


def test_group_permutation_with_weight_slabs_is_invariant():
    """Relabelling groups (moving gate/up row slabs, down column slabs and
    mask columns together) leaves every output unchanged up to rounding."""
    c = _case(T=8, H=32, I=160, gs=16, seed=9)
    G = c.G
    q = np.random.default_rng(2).permutation(G)
    ch = (q[:, None] * c.gs + np.arange(c.gs)[None, :]).reshape(-1)
    a = ffn_masked(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, c.gs)
    b = ffn_masked(c.x, c.w_gate[ch], c.w_up[ch], c.w_down[:, ch],
                   synth.pack_mask(c.mask[:, q]), c.gs)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-15)


def test_mask_bits_beyond_G_rejected():
    m = np.zeros((3, 1), dtype=np.uint32)
    assert check_mask(m, 20) == 0
    m[1, 0] = 1 << 20
    assert check_mask(m, 20) != 0
    assert check_mask(m, 21) == 0
    with pytest.raises(ValueError):
        ffn_token_loop(np.zeros((3, 8), np.float32), np.zeros((20, 8), np.float32),
                       np.zeros((20, 8), np.float32), np.zeros((8, 20), np.float32), m, 1, "f32")


def test_tiny_config_shape_and_mask_rule():
    c = synth.tiny_ffn()
    assert (c.T, c.H, c.I, c.gs, c.G) == (64, 256, 1024, 64, 16)
    assert c.mask.any(axis=1).all()
    assert 0.4 < c.mask.mean() < 0.6
    assert oracle.ffn.mask_bool(c.mask_words, c.G).tolist() == c.mask.tolist()
