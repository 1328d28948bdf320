"""The benchmark's comparators against the fp64 oracle: the naive masked FFN
the pages compare WIDE with (gather each group's tokens, three matmuls,
scatter-add back; WIDE, technical summary section 2) and the dense torch
FFN.  A speed-up is quoted against them, so they must compute the same
function as the masked kernels.

Both run torch bf16 matmuls: the naive one rounds each group's h and its
partial output to bf16 before the fp32 scatter-add, so its tolerance is
wider than the kernels' (one bf16 step, 2^-8, per partial sum)."""
import os
import sys
from types import SimpleNamespace

import numpy as np
import pytest

import synth
from oracle.ffn import ffn_masked, ffn_dense
from tests._util import rel_l2, from_dev

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TOL_NAIVE = 1e-2
TOL_DENSE = 1e-2


def _device(cases):
    import torch
    sys.path.insert(0, ROOT)
    import bench
    wl = SimpleNamespace(path_name="WIDE_PATH_DECODE")
    dev = torch.device("cuda", torch.cuda.current_device())
    return bench.FFNDevice(wl, cases, dev, torch.cuda.current_stream(dev))


@pytest.mark.parametrize("T,H,I,gs,keep", [
    (8, 512, 2048, 128, 0.5),       # a decode batch
    (37, 256, 1024, 64, 0.3),       # ragged token count, sparse
    (64, 384, 768, 32, 0.9),        # dense-ish, small groups
])
def test_naive_gather_scatter_matches_oracle(T, H, I, gs, keep):
    import torch
    c = synth.ffn_case(T, H, I, gs, seed=100 + T, keep=keep)
    D = _device([c])
    D.naive_gather_scatter(0)
    torch.cuda.synchronize()
    got = from_dev(D.outs[0])
    ref = ffn_masked(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, c.gs, c.dtype)
    assert np.isfinite(got).all()
    assert rel_l2(got, ref) <= TOL_NAIVE


def test_naive_gather_scatter_all_zero_mask_is_zero():
    import torch
    c = synth.ffn_case(5, 256, 512, 64, seed=3, mask_kind="zeros")
    D = _device([c])
    D.outs[0].fill_(1.0)
    D.naive_gather_scatter(0)
    torch.cuda.synchronize()
    assert not np.any(from_dev(D.outs[0]))


def test_dense_torch_matches_dense_oracle():
    import torch
    c = synth.ffn_case(16, 512, 1024, 128, seed=5)
    D = _device([c])
    D.dense_torch(0)
    torch.cuda.synchronize()
    ref = ffn_dense(c.x, c.w_gate, c.w_up, c.w_down)
    assert rel_l2(from_dev(D.outs[0]), ref) <= TOL_DENSE
