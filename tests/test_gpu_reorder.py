"""GPU mask reordering is bit-exact against the oracle's canonical reorder
(WIDE, technical summary section 2.B).  Runs through the C ABI."""
import numpy as np
import pytest

import synth
from oracle.ffn import reorder as oracle_reorder
from tests._util import to_dev

pytestmark = pytest.mark.gpu


def _gpu(mask_words, G, tile_m):
    import torch
    import token_level_dynamic_b200 as w
    w.wide_clear_device_status()
    r = w.wide_reorder(to_dev(mask_words, "mask"), G, tile_m)
    torch.cuda.synchronize()
    out = {k: v.cpu().numpy() for k, v in r.items() if not k.startswith("_")}
    out["status"] = w.wide_get_device_status()
    return out


def _compare(mask_words, G, tile_m):
    ref = oracle_reorder(mask_words, G, tile_m)
    got = _gpu(mask_words, G, tile_m)
    assert got["status"] == 0
    np.testing.assert_array_equal(got["count"], ref["count"])
    np.testing.assert_array_equal(got["perm"], ref["perm"])
    n = int(got["n_items"][0])
    assert n == len(ref["items"])
    np.testing.assert_array_equal(got["items"][:n], ref["items"])
    np.testing.assert_array_equal(got["sig_perm"], ref["sig_perm"])
    inv = np.empty_like(ref["sig_perm"])
    inv[ref["sig_perm"]] = np.arange(len(inv), dtype=inv.dtype)
    np.testing.assert_array_equal(got["sig_pos"], inv)
    np.testing.assert_array_equal(got["tile_union"].astype(np.uint32), ref["tile_union"])


@pytest.mark.parametrize("T,G,tile_m,p", [
    (1, 1, 128, 1.0), (5, 3, 64, 0.5), (37, 33, 64, 0.3), (300, 112, 128, 0.5),
    (257, 64, 128, 0.0), (257, 64, 128, 1.0), (1000, 1024, 128, 0.5), (129, 40, 64, 0.9),
    (2049, 8, 128, 0.34), (9000, 40, 128, 0.5), (20000, 5, 64, 0.5), (8192, 112, 128, 0.02),
])
def test_reorder_bit_exact_random(T, G, tile_m, p):
    m = np.random.default_rng(T + G).random((T, G)) < p
    _compare(synth.pack_mask(m), G, tile_m)


def test_reorder_prefill_ffn_full_size():
    c = synth.prefill_ffn()
    _compare(c.mask_words, c.G, 128)


@pytest.mark.parametrize("keep", [0.25, 0.5, 1.0])
def test_reorder_prefill_layer_masks_full_size(keep):
    m = synth.prototype_masks(0, 8192, [("mask_a", 8), ("mask_f", 112)], 16, keep,
                              0.1, extra=(8192, int(keep * 100)))
    _compare(synth.pack_mask(m["mask_f"]), 112, 128)
    _compare(synth.pack_mask(m["mask_a"]), 8, 128)


def test_reorder_empty_and_deterministic():
    import torch
    import token_level_dynamic_b200 as w
    r = w.wide_reorder(torch.zeros((0, 4), dtype=torch.int32, device="cuda"), 112, 128)
    torch.cuda.synchronize()
    assert int(r["n_items"][0]) == 0 and int(r["count"].sum()) == 0
    m = synth.pack_mask(np.random.default_rng(3).random((777, 50)) < 0.5)
    a, b = _gpu(m, 50, 128), _gpu(m, 50, 128)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])


def test_bad_mask_bit_sets_device_status():
    """A bit at or above G is reported through the status word (no fault)."""
    m = synth.pack_mask(np.random.default_rng(0).random((100, 20)) < 0.5)
    m[17, 0] |= np.uint32(1 << 25)
    got = _gpu(m, 20, 128)
    assert got["status"] & 0x1
    import token_level_dynamic_b200 as w
    w.wide_clear_device_status()
    assert w.wide_get_device_status() == 0
