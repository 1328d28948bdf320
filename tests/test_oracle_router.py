"""Pins for the router oracle (CPU only).

The router oracle (WIDE, technical summary section 2.A, router architecture)
is checked against things it does not compute itself: a hand-derived worked
example (tests/golden/router_worked_example.json), an independent library
form of the same network (torch CPU float64 Linear / ReLU / SiLU layers), a
scalar brute-force loop on tiny inputs, and invariants of the definition
(token permutation, permutation of bottleneck units, sign flips, bit
packing).
"""
import json
import os

import numpy as np
import pytest

import synth
from oracle.router import decide, pack, route_logits, route_logits_loop, route_mask

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(a):
    return synth.bf16_bits_from_f32(np.asarray(a, dtype=np.float32))


def _worked():
    with open(os.path.join(GOLDEN, "router_worked_example.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("with_bias", [True, False])
@pytest.mark.parametrize("form", ["definition", "loop"])
def test_worked_example(form, with_bias):
    ex = _worked()
    x, w1, w2 = _bits(ex["x"]), _bits(ex["w_r1"]), _bits(ex["w_r2"])
    b = np.array(ex["b_r2"], dtype=np.float32) if with_bias else None
    f = route_logits if form == "definition" else route_logits_loop
    lg = f(x, w1, w2, b, "relu")
    key = "with_bias" if with_bias else "no_bias"
    np.testing.assert_array_equal(lg, np.array(ex["logits_" + key]))
    np.testing.assert_array_equal(pack(decide(lg)), np.array(ex["words_" + key], dtype=np.uint32))
    np.testing.assert_array_equal(route_mask(x, w1, w2, b, "relu"),
                                  np.array(ex["words_" + key], dtype=np.uint32))


def test_zero_logit_skips():
    """The worked example's token 0, group 2 has a logit of exactly 0: skipped."""
    ex = _worked()
    lg = route_logits(_bits(ex["x"]), _bits(ex["w_r1"]), _bits(ex["w_r2"]),
                      np.array(ex["b_r2"], dtype=np.float32))
    assert lg[0, 2] == 0.0 and not decide(lg)[0, 2]


@pytest.mark.parametrize("act", ["relu", "silu"])
@pytest.mark.parametrize("bias", [0.0, 0.05])
def test_equals_torch_layers(act, bias):
    """Library cross-check: torch's Linear -> ReLU/SiLU -> Linear in float64."""
    import torch
    rc = synth.router_case(T=11, H=96, R=32, G=40, seed=5, act=act, bias_std=bias)
    X = torch.from_numpy(synth.f32_from_bf16_bits(rc.x).astype(np.float64))
    l1 = torch.nn.Linear(rc.H, rc.R, bias=False, dtype=torch.float64)
    l2 = torch.nn.Linear(rc.R, rc.G, bias=rc.b_r2 is not None, dtype=torch.float64)
    with torch.no_grad():
        l1.weight.copy_(torch.from_numpy(synth.f32_from_bf16_bits(rc.w_r1).astype(np.float64)))
        l2.weight.copy_(torch.from_numpy(synth.f32_from_bf16_bits(rc.w_r2).astype(np.float64)))
        if rc.b_r2 is not None:
            l2.bias.copy_(torch.from_numpy(rc.b_r2.astype(np.float64)))
        a = torch.nn.ReLU() if act == "relu" else torch.nn.SiLU()
        ref = l2(a(l1(X))).numpy()
    got = route_logits(rc.x, rc.w_r1, rc.w_r2, rc.b_r2, act)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("act", ["relu", "silu"])
def test_definition_equals_loop(act):
    """Brute force on tiny inputs: scalar loops equal the matmul form."""
    rc = synth.router_case(T=5, H=24, R=8, G=35, seed=2, act=act, bias_std=0.01)
    a = route_logits(rc.x, rc.w_r1, rc.w_r2, rc.b_r2, act)
    b = route_logits_loop(rc.x, rc.w_r1, rc.w_r2, rc.b_r2, act)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-15)


def test_token_permutation():
    rc = synth.router_case(T=17, H=64, R=16, G=12, seed=7)
    p = np.random.default_rng(1).permutation(rc.T)
    a = route_mask(rc.x, rc.w_r1, rc.w_r2)
    b = route_mask(rc.x[p], rc.w_r1, rc.w_r2)
    np.testing.assert_array_equal(a[p], b)


@pytest.mark.parametrize("act", ["relu", "silu"])
def test_bottleneck_unit_permutation(act):
    """Reordering the bottleneck units (rows of W1 with the columns of W2)
    leaves every logit unchanged up to summation order."""
    rc = synth.router_case(T=9, H=64, R=24, G=10, seed=8, act=act, bias_std=0.02)
    p = np.random.default_rng(3).permutation(rc.R)
    a = route_logits(rc.x, rc.w_r1, rc.w_r2, rc.b_r2, act)
    b = route_logits(rc.x, rc.w_r1[p], rc.w_r2[:, p], rc.b_r2, act)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-15)


def test_sign_flip_inverts_decisions():
    """Negating W2 and b negates every logit, so every group with a nonzero
    logit flips between execute and skip."""
    rc = synth.router_case(T=13, H=64, R=16, G=20, seed=9, bias_std=0.02)
    w2n = rc.w_r2 ^ np.uint16(0x8000)            # bf16 sign bit
    a = route_logits(rc.x, rc.w_r1, rc.w_r2, rc.b_r2)
    b = route_logits(rc.x, rc.w_r1, w2n, -rc.b_r2)
    np.testing.assert_array_equal(a, -b)
    nz = a != 0
    assert np.all(decide(a)[nz] != decide(b)[nz])


def test_group_forced_by_bias():
    """A group whose W2 row is zero is decided by its bias alone."""
    rc = synth.router_case(T=8, H=32, R=8, G=6, seed=4)
    w2 = rc.w_r2.copy()
    w2[2] = 0
    w2[4] = 0
    b = np.zeros(rc.G, dtype=np.float32)
    b[2], b[4] = -1e-3, 1e-3
    keep = synth.unpack_mask(route_mask(rc.x, rc.w_r1, w2, b), rc.G)
    assert not keep[:, 2].any() and keep[:, 4].all()


def test_packing_layout():
    """Group g in bit g % 32 of word g // 32; bits at or above G stay zero."""
    keep = np.zeros((3, 40), dtype=bool)
    keep[0, 33] = True
    keep[1, 0] = keep[1, 31] = keep[1, 39] = True
    w = pack(keep)
    np.testing.assert_array_equal(w, np.array([[0, 2], [0x80000001, 0x80], [0, 0]], dtype=np.uint32))
    rc = synth.router_case(T=21, H=32, R=8, G=45, seed=6, bias_std=0.05)
    m = route_mask(rc.x, rc.w_r1, rc.w_r2, rc.b_r2)
    assert np.all(m[:, 1] >> np.uint32(45 - 32) == 0)
    np.testing.assert_array_equal(m, synth.pack_mask(synth.unpack_mask(m, rc.G)))


def test_router_case_weights_independent_of_batch():
    """The seeded router weights depend on (seed, H, R, G) only, so a decode
    batch and a prefill batch of one model share them; x depends on T."""
    a = synth.router_case(T=3, H=64, R=32, G=10, seed=4, bias_std=0.1)
    b = synth.router_case(T=9, H=64, R=32, G=10, seed=4, bias_std=0.1)
    np.testing.assert_array_equal(a.w_r1, b.w_r1)
    np.testing.assert_array_equal(a.w_r2, b.w_r2)
    np.testing.assert_array_equal(a.b_r2, b.b_r2)
    assert a.x.shape == (3, 64) and b.x.shape == (9, 64)
    c = synth.router_case(T=3, H=64, R=32, G=10, seed=5, bias_std=0.1)
    assert not np.array_equal(a.w_r1, c.w_r1)
