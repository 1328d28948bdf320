"""Decode (CUDA-core GEMV) masked FFN against the fp64 oracle, through the
C ABI.  WIDE, technical summary section 2.A: a token's skipped FFN channel
groups contribute nothing; the union of the batch's groups is streamed."""
import numpy as np
import pytest

import synth
from oracle.ffn import ffn_masked
from tests._util import rel_l2, ffn_to_dev, from_dev

pytestmark = pytest.mark.gpu

TOL_BF16 = 5e-3   # relative L2, bf16 storage / fp32 accumulation
TOL_F32 = 1e-5    # relative L2, fp32 tiny configuration


@pytest.fixture(params=["auto", "tc", "fused", "gemv"], autouse=True)
def decode_kernels(request):
    """Every case runs on the dispatcher's choice and on each bf16 decode
    implementation forced: the tensor-core kernel (launches of up to 32
    tokens, hidden % 128 == 0, group size a multiple of 16), the channel-
    split CUDA-core kernel (launches of up to 16 tokens, hidden % 256 ==
    0) and the two GEMV kernels, each wherever its limits allow (else the
    dispatcher's next choice).  bf16 group size 32 has no GEMV kernel and
    runs on a persistent kernel in every mode."""
    import token_level_dynamic_b200 as w
    mode = {"auto": w.WIDE_DECODE_AUTO, "tc": w.WIDE_DECODE_TC, "fused": w.WIDE_DECODE_FUSED,
            "gemv": w.WIDE_DECODE_GEMV}[request.param]
    prev = w.wide_set_decode_ffn_path(mode)
    yield request.param
    w.wide_set_decode_ffn_path(prev)


def _run(c, path=None):
    import torch
    import token_level_dynamic_b200 as w
    x, wg, wu, wd, m = ffn_to_dev(c)
    w.wide_clear_device_status()
    out = w.wide_ffn_masked(x, wg, wu, wd, m, c.gs,
                            path=w.WIDE_PATH_DECODE if path is None else path)
    torch.cuda.synchronize()
    assert w.wide_get_device_status() == 0
    return from_dev(out)


def _ref(c):
    return ffn_masked(c.x, c.w_gate, c.w_up, c.w_down, c.mask_words, c.gs, c.dtype)


def test_tiny_fp32_config():
    c = synth.tiny_ffn()
    assert rel_l2(_run(c), _ref(c)) <= TOL_F32


@pytest.mark.parametrize("batch", [1, 8, 32])
def test_decode_ffn_3b_config(batch):
    c = synth.decode_ffn(batch)
    assert rel_l2(_run(c), _ref(c)) <= TOL_BF16


def test_decode_layer_ffn_shape():
    """The FFN half of the 8B decode layer: B=16, H=4096, I=14336, keep 0.72."""
    c = synth.ffn_case(16, 4096, 14336, 128, seed=4, keep=0.72)
    assert rel_l2(_run(c), _ref(c)) <= TOL_BF16


@pytest.mark.parametrize("T,H,I,gs,dtype", [
    (1, 128, 256, 64, "bf16"), (3, 256, 1024, 128, "bf16"), (33, 384, 768, 64, "bf16"),
    (70, 256, 512, 32, "f32"), (5, 640, 1280, 128, "f32"), (32, 1024, 2048, 64, "bf16"),
])
def test_decode_shapes_and_ragged_token_counts(T, H, I, gs, dtype):
    c = synth.ffn_case(T, H, I, gs, seed=T, dtype=dtype)
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    assert rel_l2(_run(c), _ref(c)) <= tol


def test_all_zero_mask_gives_exact_zero():
    c = synth.ffn_case(8, 512, 1024, 128, seed=1, mask_kind="zeros")
    assert not np.any(_run(c))


def test_all_ones_mask_equals_dense():
    c = synth.ffn_case(8, 512, 1024, 128, seed=2, mask_kind="ones")
    from oracle.ffn import ffn_dense
    assert rel_l2(_run(c), ffn_dense(c.x, c.w_gate, c.w_up, c.w_down)) <= TOL_BF16


def test_single_token_single_group():
    c = synth.ffn_case(1, 256, 1024, 128, seed=3)
    c.mask[:] = False
    c.mask[0, 5] = True
    assert rel_l2(_run(c), _ref(c)) <= TOL_BF16


def test_repeatable(decode_kernels):
    """The GEMV kernels are bitwise repeatable.  The persistent kernels add
    their CTAs' fp32 partial sums with atomics, in an order that varies from
    call to call, so two calls agree to within one bf16 rounding step of the
    element plus the fp32 summation noise (an element whose terms nearly
    cancel can land on either side of a bf16 step of its own small size):
    1e-5 of the output's rms, far below any real error."""
    c = synth.decode_ffn(8)
    a, b = _run(c), _run(c)
    if decode_kernels == "gemv":
        np.testing.assert_array_equal(a, b)
    else:
        rms = float(np.sqrt(np.mean(a.astype(np.float64) ** 2)))
        lim = 2.0 ** -7 * np.maximum(np.abs(a), np.abs(b)) + 1e-5 * rms
        bad = np.abs(a - b) > lim
        i = np.unravel_index(np.argmax(np.abs(a - b) - lim), a.shape)
        assert not bad.any(), (int(bad.sum()), i, float(a[i]), float(b[i]), rms)


@pytest.mark.parametrize("T", [9, 17, 24, 31])
def test_odd_and_mid_token_counts(T):
    """Token counts between the kernel's pair templates, odd ones included
    (the last pair of a group then has one padding slot)."""
    c = synth.ffn_case(T, 1024, 4096, 128, seed=40 + T)
    assert rel_l2(_run(c), _ref(c)) <= TOL_BF16


@pytest.mark.parametrize("T,H,I,gs", [
    (2, 512, 2048, 128),       # one token pair
    (7, 768, 3072, 64),        # odd count, 48 groups of 64
    (32, 512, 4096, 32),       # bf16 group size 32, 128 groups
    (31, 512, 2048, 32),       # group size 32, odd count
    (8, 512, 16384, 64),       # ~256 live groups: more groups than CTAs
    (13, 256, 32768, 32),      # 1024 groups of 32: several whole groups per CTA
    (20, 1280, 2560, 128),     # hidden 1280: a partial last 1024-row block
])
def test_channel_split_shapes(T, H, I, gs):
    """Shapes that exercise the channel-split kernel's work split: items
    cut from one group over several CTAs, several whole groups per CTA, a
    W_down row block cut short by the hidden size, group sizes 32 to 128."""
    c = synth.ffn_case(T, H, I, gs, seed=T + H, keep=0.5)
    assert rel_l2(_run(c), _ref(c)) <= TOL_BF16


def test_union_of_one_group_with_a_full_batch():
    """Only token 19 keeps anything (group 3): every other token's output is
    exactly zero and the one kept group is right."""
    c = synth.ffn_case(20, 512, 2048, 128, seed=9)
    c.mask[:] = False
    c.mask[19, 3] = True
    out = _run(c)
    assert not np.any(out[:19])
    assert rel_l2(out, _ref(c)) <= TOL_BF16


def test_output_rows_split_unevenly_over_the_grid():
    """A hidden size whose output rows do not split evenly over the grid."""
    c = synth.ffn_case(5, 2816, 3072, 64, seed=11)
    assert rel_l2(_run(c), _ref(c)) <= TOL_BF16


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_bad_mask_bit_sets_device_status(dtype):
    """A bit at or above G in the decode mask sets WIDE_DEV_BAD_MASK."""
    import torch
    import token_level_dynamic_b200 as w
    c = synth.ffn_case(2, 256, 1024, 128, seed=5, dtype=dtype)          # G = 8
    x, wg, wu, wd, m = ffn_to_dev(c)
    m[1, 0] |= 1 << 9
    w.wide_clear_device_status()
    w.wide_ffn_masked(x, wg, wu, wd, m, c.gs, path=w.WIDE_PATH_DECODE)
    torch.cuda.synchronize()
    assert w.wide_get_device_status() & w.WIDE_DEV_BAD_MASK
    w.wide_clear_device_status()
