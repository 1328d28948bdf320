"""The C ABI library loads and exports every symbol include/wide.h declares;
host-side argument checks answer without touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "wide.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wide_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def native():
    from token_level_dynamic_b200 import _native
    return _native


def test_library_exports_every_declared_symbol(native):
    L = native.lib()
    declared = _header_functions()
    assert len(declared) >= 9
    for name in declared:
        assert hasattr(L, name), name
        assert name in native.SIGNATURES, f"binding lacks {name}"


def test_binding_names_match_c_names(native):
    import token_level_dynamic_b200 as w
    for name in _header_functions():
        if name in ("wide_worklist_carve",):
            continue
        assert hasattr(w, name), name


def test_constants_match_header(native):
    src = open(os.path.join(ROOT, "include", "wide.h")).read()
    for name, val in re.findall(r"#define (WIDE_[A-Z0-9_]+) (-?0x[0-9a-fA-F]+|-?\d+)", src):
        if hasattr(native, name):
            assert getattr(native, name) == int(val, 0), name


def test_version_and_status_strings(native):
    L = native.lib()
    assert L.wide_abi_version() == 3
    for code in (0, -1, -2, -3, -4, 1, 2, 4):
        assert L.wide_status_string(code)


def test_worklist_bytes_and_carve_validation(native):
    L = native.lib()
    assert L.wide_worklist_bytes(4096, 112, 128) > 4 * 112 * 4096
    assert L.wide_worklist_bytes(4096, 0, 128) == 0
    assert L.wide_worklist_bytes(4096, 1025, 128) == 0
    assert L.wide_worklist_bytes(-1, 8, 128) == 0
    assert L.wide_worklist_bytes(64, 8, 96) == 0
    wl = native.WideWorklist()
    # a misaligned base pointer is refused before anything is enqueued
    assert L.wide_worklist_carve(ctypes.c_void_p(16), 1 << 30, 64, 8, 128, ctypes.byref(wl)) \
        == native.WIDE_EUNSUPPORTED
    assert L.wide_worklist_carve(ctypes.c_void_p(256), 16, 64, 8, 128, ctypes.byref(wl)) \
        == native.WIDE_EWORKSPACE
    assert L.wide_worklist_carve(ctypes.c_void_p(1 << 20), 1 << 30, 64, 8, 128,
                                 ctypes.byref(wl)) == 0
    assert wl.tokens == 64 and wl.groups == 8 and wl.tile_m == 128
    assert wl.perm - wl.count >= 32 and (wl.perm % 256) == 0
    assert L.wide_reorder(None, 64, 8, 128, None, None) == native.WIDE_EINVAL
    assert L.wide_reorder(None, 64, 9, 128, ctypes.byref(wl), None) == native.WIDE_EINVAL


def test_ffn_argument_checks(native):
    L = native.lib()
    D = native.WideFFNDims
    ok = D(8, 3072, 8192, 128, native.WIDE_BF16, native.WIDE_PATH_DECODE)
    assert L.wide_ffn_workspace_bytes(ctypes.byref(ok)) >= 8 * 8192 * 4
    for bad in (D(-1, 3072, 8192, 128, 0, 1), D(8, 3072, 8192, 100, 0, 1),
                D(8, 3072, 8192, 128, 5, 1), D(8, 3072, 8192, 128, 0, 7),
                D(8, 3072, 128 * 2000, 128, 0, 1)):
        assert L.wide_ffn_workspace_bytes(ctypes.byref(bad)) == 0
        assert L.wide_ffn_masked(None, None, None, None, None, None, ctypes.byref(bad), None,
                                 None, 0, None) == native.WIDE_EINVAL
    # null pointers with valid dims
    assert L.wide_ffn_masked(None, None, None, None, None, None, ctypes.byref(ok), None, None, 0,
                             None) == native.WIDE_EINVAL
    # zero tokens is a no-op
    z = D(0, 3072, 8192, 128, 0, 1)
    assert L.wide_ffn_masked(None, None, None, None, None, None, ctypes.byref(z), None, None, 0,
                             None) == native.WIDE_OK
    # an unsupported shape is refused on the host (hidden not a multiple of 128)
    p = ctypes.c_void_p(1 << 20)
    odd = D(8, 3000, 8192, 128, 0, 1)
    assert L.wide_ffn_masked(p, p, p, p, p, p, ctypes.byref(odd), None, p, 1 << 30, None) \
        == native.WIDE_EUNSUPPORTED
    # group size 16 is not built on the bf16 decode path
    g16 = D(8, 3072, 8192, 16, 0, 1)
    assert L.wide_ffn_masked(p, p, p, p, p, p, ctypes.byref(g16), None, p, 1 << 30, None) \
        == native.WIDE_EUNSUPPORTED
    # misaligned pointer
    mis = ctypes.c_void_p((1 << 20) + 8)
    assert L.wide_ffn_masked(mis, p, p, p, p, p, ctypes.byref(ok), None, p, 1 << 30, None) \
        == native.WIDE_EUNSUPPORTED
    # workspace too small
    assert L.wide_ffn_masked(p, p, p, p, p, p, ctypes.byref(ok), None, p, 16, None) \
        == native.WIDE_EWORKSPACE


def test_ffn_worklist_argument_checks(native):
    """A caller work list must match the call's (T, G, tile_m = 128): a
    mismatch or a null array is refused on the host before anything runs."""
    L = native.lib()
    D = native.WideFFNDims
    T, H, I, gs = 300, 4096, 8192, 128
    G = I // gs
    base = ctypes.c_void_p(1 << 24)                     # never dereferenced
    p = ctypes.c_void_p(1 << 20)
    nbytes = L.wide_worklist_bytes(T, G, 128)
    wl = native.WideWorklist()
    assert L.wide_worklist_carve(base, nbytes, T, G, 128, ctypes.byref(wl)) == native.WIDE_OK
    d = D(T, H, I, gs, native.WIDE_BF16, native.WIDE_PATH_PREFILL)
    # a matching work list passes the check (the tiny workspace then stops the call)
    assert L.wide_ffn_masked(p, p, p, p, p, p, ctypes.byref(d), ctypes.byref(wl), p, 16,
                             None) == native.WIDE_EWORKSPACE
    for dims in (D(T + 1, H, I, gs, 0, 2), D(T, H, I, 64, 0, 2), D(T, H, I // 2, gs, 0, 2)):
        assert L.wide_ffn_masked(p, p, p, p, p, p, ctypes.byref(dims), ctypes.byref(wl), p,
                                 1 << 30, None) == native.WIDE_EINVAL
    wl64 = native.WideWorklist()
    assert L.wide_worklist_carve(base, L.wide_worklist_bytes(T, G, 64), T, G, 64,
                                 ctypes.byref(wl64)) == native.WIDE_OK
    assert L.wide_ffn_masked(p, p, p, p, p, p, ctypes.byref(d), ctypes.byref(wl64), p,
                             1 << 30, None) == native.WIDE_EINVAL
    wl.sig_pos = None
    assert L.wide_ffn_masked(p, p, p, p, p, p, ctypes.byref(d), ctypes.byref(wl), p, 1 << 30,
                             None) == native.WIDE_EINVAL


def test_packed_weight_entry_points_check_on_the_host(native):
    """The packed decode layout: its size, and the argument checks of
    wide_ffn_pack and wide_ffn_masked_packed, all answered before anything
    is enqueued (no GPU needed)."""
    L = native.lib()
    assert L.wide_ffn_packed_bytes(3072, 8192) == 3 * 3072 * 8192 * 2
    assert L.wide_ffn_packed_bytes(3072 + 64, 8192) == 0      # hidden % 128
    assert L.wide_ffn_packed_bytes(3072, 8192 + 32) == 0      # inter % 64
    assert L.wide_ffn_packed_bytes(0, 8192) == 0
    p = ctypes.c_void_p(1 << 20)
    need = L.wide_ffn_packed_bytes(256, 512)
    assert L.wide_ffn_pack(None, p, p, 256, 512, p, need, None) == native.WIDE_EINVAL
    assert L.wide_ffn_pack(p, p, p, 256, 512 + 32, p, need, None) == native.WIDE_EUNSUPPORTED
    assert L.wide_ffn_pack(p, p, p, 256, 512, p, need - 1, None) == native.WIDE_EWORKSPACE
    assert L.wide_ffn_pack(p, p, p, 256, 512, ctypes.c_void_p((1 << 20) + 16), need,
                           None) == native.WIDE_EUNSUPPORTED       # packed not 256-aligned
    D = native.WideFFNDims
    d = D(8, 256, 512, 128, native.WIDE_BF16, native.WIDE_PATH_DECODE)
    assert L.wide_ffn_masked_packed(None, p, None, None, None, p, p, ctypes.byref(d), p, 1 << 30,
                                    None) == native.WIDE_EINVAL
    # the nn.Linear weights come all three or none
    assert L.wide_ffn_masked_packed(p, p, p, None, p, p, p, ctypes.byref(d), p, 1 << 30,
                                    None) == native.WIDE_EINVAL
    for bad in (D(8, 256, 512, 128, native.WIDE_BF16, native.WIDE_PATH_PREFILL),
                D(8, 256, 512, 128, native.WIDE_F32, native.WIDE_PATH_DECODE),
                D(8, 256 + 64, 512, 128, native.WIDE_BF16, native.WIDE_PATH_DECODE)):
        assert L.wide_ffn_masked_packed(p, p, None, None, None, p, p, ctypes.byref(bad), p,
                                        1 << 30, None) == native.WIDE_EUNSUPPORTED
    z = D(0, 256, 512, 128, native.WIDE_BF16, native.WIDE_PATH_DECODE)
    assert L.wide_ffn_masked_packed(p, p, None, None, None, p, p, ctypes.byref(z), p, 0,
                                    None) == native.WIDE_OK


def test_binding_refuses_operands_on_two_devices():
    """The binding launches on the operands' device and refuses operands on
    different devices (or off the GPU) before any C call."""
    import types
    import torch
    pkg = pytest.importorskip("token_level_dynamic_b200")
    cuda0, cuda1 = torch.device("cuda", 0), torch.device("cuda", 1)

    def fake(dev):
        return types.SimpleNamespace(is_cuda=dev.type == "cuda", device=dev)

    assert pkg._one_device("f", x=fake(cuda1), w=fake(cuda1), out=None) == cuda1
    with pytest.raises(ValueError, match="every operand must be on one device"):
        pkg._one_device("f", x=fake(cuda0), w=fake(cuda1))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        pkg._one_device("f", x=fake(cuda0), mask=fake(torch.device("cpu")))
    with pytest.raises(ValueError, match="no tensor operand"):
        pkg._one_device("f", x=None)


def test_decode_path_switch_is_host_only(native):
    """wide_set_decode_ffn_path answers on the host: returns the previous
    mode and refuses unknown modes without changing the current one."""
    L = native.lib()
    prev = L.wide_set_decode_ffn_path(1)
    try:
        assert L.wide_set_decode_ffn_path(2) == 1
        assert L.wide_set_decode_ffn_path(3) == 2
        assert L.wide_set_decode_ffn_path(2) == 3
        assert L.wide_set_decode_ffn_path(7) == -1
        assert L.wide_set_decode_ffn_path(-1) == -1
        assert L.wide_set_decode_ffn_path(0) == 2
    finally:
        L.wide_set_decode_ffn_path(prev)


def test_route_argument_checks(native):
    """wide_route refuses bad dims, shapes and alignment on the host."""
    L = native.lib()
    D = native.WideRouterDims
    p = ctypes.c_void_p(1 << 20)
    mis = ctypes.c_void_p((1 << 20) + 8)
    for bad in (D(-1, 4096, 128, 112, 0), D(8, 0, 128, 112, 0), D(8, 4096, 0, 112, 0),
                D(8, 4096, 128, 0, 0), D(8, 4096, 128, 112, 2)):
        assert L.wide_route(p, p, p, None, p, None, ctypes.byref(bad), None) == native.WIDE_EINVAL
    assert L.wide_route(None, None, None, None, None, None, None, None) == native.WIDE_EINVAL
    ok = D(8, 4096, 128, 112, native.WIDE_ACT_RELU)
    assert L.wide_route(None, p, p, None, p, None, ctypes.byref(ok), None) == native.WIDE_EINVAL
    assert L.wide_route(p, p, p, None, None, None, ctypes.byref(ok), None) == native.WIDE_EINVAL
    # zero tokens is a no-op
    assert L.wide_route(None, None, None, None, None, None, ctypes.byref(D(0, 4096, 128, 112, 0)),
                        None) == native.WIDE_OK
    for unsup in (D(8, 4000, 128, 112, 0), D(8, 4096, 100, 112, 0), D(8, 4096, 288, 112, 0),
                  D(8, 4096, 128, 1025, 0), D(1 << 20, 4096, 128, 112, 0)):
        assert L.wide_route(p, p, p, None, p, None, ctypes.byref(unsup), None) \
            == native.WIDE_EUNSUPPORTED
    assert L.wide_route(mis, p, p, None, p, None, ctypes.byref(ok), None) \
        == native.WIDE_EUNSUPPORTED
    assert L.wide_route(p, p, mis, None, p, None, ctypes.byref(ok), None) \
        == native.WIDE_EUNSUPPORTED
    assert L.wide_route(p, p, p, ctypes.c_void_p((1 << 20) + 2), p, None, ctypes.byref(ok),
                        None) == native.WIDE_EUNSUPPORTED


def test_layer_argument_checks(native):
    """wide_layer_masked / wide_attn_masked / wide_layer_workspace_bytes
    answer on the host for bad dims, missing or misaligned pointers and a
    short workspace, before anything is enqueued."""
    L = native.lib()
    D, Wt = native.WideLayerDims, native.WideLayerWeights
    dec = D(16, 1, 2048, 2049, 4096, 14336, 128, 32, 8, 128, 5e5, 1e-5)
    pre = D(4, 2048, 0, 2048, 4096, 14336, 128, 32, 8, 128, 5e5, 1e-5)
    ws_dec = L.wide_layer_workspace_bytes(ctypes.byref(dec))
    ws_pre = L.wide_layer_workspace_bytes(ctypes.byref(pre))
    assert ws_dec > 16 * 14336 * 4
    assert ws_pre > 8192 * 14336 * 2
    for bad in (D(16, 1, 2048, 2049, 4096, 14336, 128, 32, 7, 128, 5e5, 1e-5),     # 32 % 7
                D(16, 1, 2048, 2048, 4096, 14336, 128, 32, 8, 128, 5e5, 1e-5),     # no room
                D(16, 1, 2048, 2049, 4096, 14336, 128, 32, 8, 128, 5e5, -1.0),     # eps < 0
                D(16, 1, 2048, 2049, 4096, 14336, 128, 32, 8, 128, 0.0, 1e-5),     # theta 0
                D(16, 1, 2048, 2049, 4096, 14336, 100, 32, 8, 128, 5e5, 1e-5),     # gs does not divide I
                D(16, 1, 2048, 2049, 4096, 14336, 128, 32, 8, 64, 5e5, 1e-5),      # head_dim 64
                D(16, 1, 131072, 131073, 4096, 14336, 128, 32, 8, 128, 5e5, 1e-5)):  # cache too long
        assert L.wide_layer_workspace_bytes(ctypes.byref(bad)) == 0
    p = ctypes.c_void_p(1 << 20)
    mis = ctypes.c_void_p((1 << 20) + 8)
    full = Wt(*([p] * 9))
    empty = Wt(*([None] * 9))
    args = lambda x, w, ws_bytes, d: (x, ctypes.byref(w), p, p, p, p, p, p, p, ctypes.byref(d),
                                      p, ws_bytes, None)
    assert L.wide_layer_masked(p, None, p, p, p, p, p, p, p, ctypes.byref(dec), p, ws_dec,
                               None) == native.WIDE_EINVAL
    assert L.wide_layer_masked(*args(p, empty, ws_dec, dec)) == native.WIDE_EINVAL
    assert L.wide_layer_masked(*args(mis, full, ws_dec, dec)) == native.WIDE_EUNSUPPORTED
    assert L.wide_layer_masked(*args(p, full, ws_dec - 1, dec)) == native.WIDE_EWORKSPACE
    assert L.wide_layer_masked(*args(p, full, ws_pre - 1, pre)) == native.WIDE_EWORKSPACE
    # the attention half alone needs its output pointer
    assert L.wide_attn_masked(p, ctypes.byref(full), p, p, p, None, ctypes.byref(dec), p,
                              ws_dec, None) == native.WIDE_EINVAL


def test_route_binding_checks_dtypes_and_shapes():
    """The Python binding refuses tensors the C ABI cannot check (dtype and
    shape) before touching the device."""
    import torch
    import token_level_dynamic_b200 as w
    bf = torch.bfloat16
    x, w1, w2 = torch.zeros(4, 64, dtype=bf), torch.zeros(32, 64, dtype=bf), torch.zeros(8, 32, dtype=bf)
    with pytest.raises(TypeError):
        w.wide_route(x.float(), w1, w2)
    with pytest.raises(ValueError):
        w.wide_route(x, torch.zeros(32, 32, dtype=bf), w2)          # W_r1 width != H
    with pytest.raises(ValueError):
        w.wide_route(x, w1, torch.zeros(8, 16, dtype=bf))           # W_r2 width != R
    with pytest.raises(ValueError):
        w.wide_route(x, w1, w2, b_r2=torch.zeros(8, dtype=torch.float64))
    with pytest.raises(ValueError):
        w.wide_route(x, w1, w2, mask_words=torch.zeros(4, 2, dtype=torch.int32))
    with pytest.raises(ValueError):
        w.wide_route(x, w1, w2, logits=torch.zeros(4, 9))
    # well-formed CPU tensors get past these checks and stop at the device check
    with pytest.raises(ValueError, match="CUDA tensor"):
        w.wide_route(x, w1, w2, mask_words=torch.zeros(4, 1, dtype=torch.int32))


def test_ffn_binding_checks_dtypes_and_shapes():
    """The FFN bindings refuse mismatched dtypes and shapes before the C call."""
    import torch
    import token_level_dynamic_b200 as w
    bf = torch.bfloat16
    x = torch.zeros(4, 64, dtype=bf)
    wg, wu, wd = torch.zeros(256, 64, dtype=bf), torch.zeros(256, 64, dtype=bf), torch.zeros(64, 256, dtype=bf)
    m = torch.zeros(4, 1, dtype=torch.int32)                     # G = 256 / 64 = 4
    for f in (lambda *a, **k: w.wide_ffn_masked(*a, **k),
              lambda *a, **k: w.wide_ffn_masked_noalloc(*a, out=k.pop("out", torch.zeros(4, 64, dtype=bf)), **k)):
        with pytest.raises(TypeError):
            f(x, wg.float(), wu, wd, m, 64)
        with pytest.raises(ValueError):
            f(x, wg, wu, wd.t().contiguous(), m, 64)             # W_down transposed
        with pytest.raises(ValueError):
            f(x, wg, wu, wd, torch.zeros(4, 2, dtype=torch.int32), 64)
        with pytest.raises(ValueError):
            f(x, wg, wu, wd, m.to(torch.int64), 64)
        with pytest.raises(ValueError):
            f(x, wg, wu, wd, m, 64, out=torch.zeros(4, 64))       # fp32 out for bf16 x
        # well-formed CPU tensors pass these checks and stop at the device check
        with pytest.raises(ValueError, match="CUDA tensor"):
            f(x, wg, wu, wd, m, 64)
