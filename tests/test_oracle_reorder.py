"""Pins for the oracle's canonical mask reordering (CPU only).

WIDE, technical summary section 2.B: per routing group the binary mask is
sorted along the token dimension M so that the active tokens form a
contiguous prefix; a tile of that order is dense up to a known active prefix.
Every output is checked against Python's own stable sort and plain loops.
"""
import numpy as np
import pytest

import synth
from oracle.ffn import reorder


def _expected(mask: np.ndarray, tile_m: int):
    T, G = mask.shape
    words = synth.pack_mask(mask)
    count = mask.sum(axis=0).astype(np.int32)
    perm = np.array([sorted(range(T), key=lambda t: (not mask[t, g], t)) for g in range(G)],
                    dtype=np.int32).reshape(G, T)
    items = [(g, i) for g in range(G) for i in range(-(-int(count[g]) // tile_m))]
    # big-endian key: last word first, then as unsigned ints
    sig = sorted(range(T), key=lambda t: (tuple(int(w) for w in words[t][::-1]), t))
    nt = -(-T // tile_m)
    tu = np.zeros((nt, words.shape[1]), dtype=np.uint32)
    for s in range(nt):
        for r in range(s * tile_m, min(T, (s + 1) * tile_m)):
            tu[s] |= words[sig[r]]
    return count, perm, np.array(items, dtype=np.int32).reshape(-1, 2), np.array(sig, np.int32), tu


CASES = [
    (1, 1, 1, 0.5), (5, 3, 2, 0.5), (37, 33, 8, 0.3), (130, 64, 128, 0.5), (300, 112, 128, 0.5),
    (64, 16, 16, 1.0), (64, 16, 16, 0.0), (200, 8, 64, 0.34), (129, 40, 32, 0.9),
]


@pytest.mark.parametrize("T,G,tile_m,p", CASES)
def test_reorder_matches_library_sort(T, G, tile_m, p):
    mask = np.random.default_rng(T * 1000 + G).random((T, G)) < p
    r = reorder(synth.pack_mask(mask), G, tile_m)
    count, perm, items, sig, tu = _expected(mask, tile_m)
    np.testing.assert_array_equal(r["count"], count)
    np.testing.assert_array_equal(r["perm"], perm)
    np.testing.assert_array_equal(r["items"], items)
    np.testing.assert_array_equal(r["sig_perm"], sig)
    np.testing.assert_array_equal(r["tile_union"], tu)


def test_active_prefix_is_contiguous_and_a_permutation():
    mask = np.random.default_rng(0).random((257, 50)) < 0.5
    r = reorder(synth.pack_mask(mask), 50, 64)
    for g in range(50):
        row = r["perm"][g]
        assert sorted(row.tolist()) == list(range(257))
        k = r["count"][g]
        assert mask[row[:k], g].all() and not mask[row[k:], g].any()
        assert (np.diff(row[:k]) > 0).all() and (np.diff(row[k:]) > 0).all()


def test_prototype_masks_cluster_in_signature_order():
    """Tokens drawn from few prototypes with no noise: the signature order
    puts equal rows together, so each sig tile's union is one prototype when
    the tile lies inside one run."""
    m = synth.prototype_masks(4, 512, [("mask_f", 112)], 4, 0.5, 0.0)["mask_f"]
    r = reorder(synth.pack_mask(m), 112, 128)
    rows = m[r["sig_perm"]]
    changes = np.flatnonzero((rows[1:] != rows[:-1]).any(axis=1))
    assert len(changes) <= 3
    assert r["count"].sum() == m.sum()


def test_empty_token_set():
    r = reorder(np.zeros((0, 2), np.uint32), 40, 128)
    assert r["count"].tolist() == [0] * 40 and len(r["items"]) == 0 and len(r["sig_perm"]) == 0


def test_bad_mask_bit_rejected():
    w = np.zeros((4, 1), np.uint32)
    w[3, 0] = 1 << 9
    with pytest.raises(ValueError):
        reorder(w, 9, 16)
