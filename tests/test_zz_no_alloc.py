"""wide_ffn_masked_noalloc: the decode FFN for callers that cannot allocate
device memory (a host framework that owns the whole device pool and hands
out no workspace, or a latency-critical loop where cudaMalloc/cudaFree would
synchronise the device).  Its scratch lives in a fixed device array inside
the library instead of a caller workspace.

The new entry point is called through the C ABI and compared with the
existing workspace entry point (wide_ffn_masked, decode path) on two calls in
a row, within the tolerance the decode parity tests use.  This file sorts
last so that a run stopping at the first failure has run everything else."""
import ctypes

import numpy as np
import pytest

import synth
from tests._util import rel_l2, ffn_to_dev, from_dev

pytestmark = pytest.mark.gpu

TOL_BF16 = 5e-3
TOL_F32 = 1e-5


def _noalloc_c_call(x, wg, wu, wd, m, out, gs, stream):
    from token_level_dynamic_b200 import _native
    L = _native.lib()
    T, H = x.shape
    d = _native.WideFFNDims(T, H, wg.shape[0], gs,
                            _native.WIDE_BF16 if x.dtype.is_floating_point and x.element_size() == 2
                            else _native.WIDE_F32, _native.WIDE_PATH_DECODE)
    return L.wide_ffn_masked_noalloc(x.data_ptr(), wg.data_ptr(), wu.data_ptr(), wd.data_ptr(),
                                     m.data_ptr(), out.data_ptr(), ctypes.byref(d), stream)


@pytest.mark.parametrize("make,tol", [
    (lambda: synth.decode_ffn(8), TOL_BF16),
    (lambda: synth.ffn_case(32, 4096, 14336, 128, seed=4, keep=0.72), TOL_BF16),
    (lambda: synth.tiny_ffn(), TOL_F32),
])
def test_noalloc_matches_workspace_entry_point_on_two_calls(make, tol):
    import torch
    import token_level_dynamic_b200 as w
    c = make()
    x, wg, wu, wd, m = ffn_to_dev(c)
    stream = torch.cuda.current_stream().cuda_stream
    w.wide_clear_device_status()
    ref = from_dev(w.wide_ffn_masked(x, wg, wu, wd, m, c.gs, path=w.WIDE_PATH_DECODE))
    outs = []
    for _ in range(2):
        out = torch.full_like(x, float("nan"))
        assert _noalloc_c_call(x, wg, wu, wd, m, out, c.gs, stream) == w.WIDE_OK
        torch.cuda.synchronize()
        outs.append(from_dev(out))
    assert w.wide_get_device_status() == 0
    from oracle.ffn import ffn_masked
    oracle = ffn_masked(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, c.gs, c.dtype)
    for o in outs:
        assert np.isfinite(o).all()
        assert rel_l2(o, ref) <= tol
        assert rel_l2(o, oracle) <= tol


def test_noalloc_token_counts_after_other_shapes():
    """Odd and multi-launch token counts (1, 33 = 32 + 1, 40 = 32 + 8) on the
    3B FFN shape, each called right after a call of another shape, so the
    fixed array holds an earlier call's unrelated data: the result equals
    the workspace entry point's and the oracle's, and is finite."""
    import torch
    import token_level_dynamic_b200 as w
    from oracle.ffn import ffn_masked
    stream = torch.cuda.current_stream().cuda_stream
    other = synth.ffn_case(24, 1024, 4096, 64, seed=77)       # a different shape
    ox, owg, owu, owd, om = ffn_to_dev(other)
    base = synth.decode_ffn(1)
    for T in (1, 33, 40):
        c = synth.decode_ffn(T, weights=False) if T > 1 else base
        c.w_gate, c.w_up, c.w_down = base.w_gate, base.w_up, base.w_down
        x, wg, wu, wd, m = ffn_to_dev(c)
        w.wide_clear_device_status()
        oo = torch.empty_like(ox)
        assert _noalloc_c_call(ox, owg, owu, owd, om, oo, other.gs, stream) == w.WIDE_OK
        out = torch.full_like(x, float("nan"))
        assert _noalloc_c_call(x, wg, wu, wd, m, out, c.gs, stream) == w.WIDE_OK
        ref = from_dev(w.wide_ffn_masked(x, wg, wu, wd, m, c.gs, path=w.WIDE_PATH_DECODE))
        torch.cuda.synchronize()
        assert w.wide_get_device_status() == 0
        got = from_dev(out)
        assert np.isfinite(got).all()
        assert rel_l2(got, ref) <= TOL_BF16
        assert rel_l2(got, ffn_masked(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, c.gs,
                                      c.dtype)) <= TOL_BF16


def test_noalloc_rejects_problems_beyond_its_scratch():
    import torch
    import token_level_dynamic_b200 as w
    from token_level_dynamic_b200 import _native
    # 32 tokens x 16384 channels x 4 bytes = the whole 2 MiB array: accepted
    # by the size check; one more group of channels is refused on the host.
    T, H, gs = 32, 128, 128
    for I, expect_ok in ((16384, True), (16384 + 128, False)):
        d = _native.WideFFNDims(T, H, I, gs, _native.WIDE_BF16, _native.WIDE_PATH_DECODE)
        if expect_ok:
            # the fixed array holds h (or a persistent kernel's accumulator)
            assert T * I * 4 <= w.WIDE_NOALLOC_SCRATCH_BYTES
            assert w.wide_ffn_workspace_bytes(T, H, I, gs) == T * I * 4 + 256
        else:
            p = ctypes.c_void_p(1 << 20)
            rc = _native.lib().wide_ffn_masked_noalloc(p, p, p, p, p, p, ctypes.byref(d), None)
            assert rc == w.WIDE_ETOOLARGE
    # the binding refuses too, with a clear message
    x = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    wg = torch.zeros((16384 + 128, H), dtype=torch.bfloat16, device="cuda")
    wd = torch.zeros((H, 16384 + 128), dtype=torch.bfloat16, device="cuda")
    m = torch.zeros((T, 5), dtype=torch.int32, device="cuda")
    with pytest.raises(w.WideError, match="fixed scratch"):
        w.wide_ffn_masked_noalloc(x, wg, wg, wd, m, gs, out=torch.empty_like(x))
