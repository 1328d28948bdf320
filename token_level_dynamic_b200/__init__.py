"""token_level_dynamic_b200 -- WIDE's masked transformer layer on B200 (sm_100a).

A thin Python binding over libwide.so (C ABI, include/wide.h).  Each function
here has the name of the C entry point it calls and only marshals arguments:
torch tensors supply device memory and the stream; every step of the layer
runs in the library's CUDA kernels.  Importing the package loads the library
and fails if it has not been built.

Method: "WIDE: Boosting Adaptive LLM Inference via Token-level Dynamic Width
Pruning" -- per-token FFN channel groups and GQA head groups (technical
summary section 2.A), mask reordering (2.B), block-level and intra-block
skipping (2.C).
"""
from __future__ import annotations

import ctypes

import torch

from . import _native
from ._native import (  # noqa: F401
    WIDE_OK, WIDE_EINVAL, WIDE_EUNSUPPORTED, WIDE_EWORKSPACE, WIDE_ECUDA, WIDE_ETOOLARGE,
    WIDE_NOALLOC_SCRATCH_BYTES,
    WIDE_DEV_BAD_MASK, WIDE_DEV_TIMEOUT, WIDE_DEV_BAD_ITEM, WIDE_DEV_LAYOUT,
    WIDE_BF16, WIDE_F32, WIDE_PATH_AUTO, WIDE_PATH_DECODE, WIDE_PATH_PREFILL,
    WIDE_ACT_RELU, WIDE_ACT_SILU,
    WideWorklist, WideFFNDims, WideLayerDims, WideLayerWeights, WideRouterDims,
)

_L = _native.lib()


class WideError(RuntimeError):
    def __init__(self, fn: str, code: int):
        msg = f"{fn}: {code} ({wide_status_string(code)})"
        if code == WIDE_ECUDA:
            msg += f" at {wide_last_error()}"
        super().__init__(msg)
        self.code = code


def _check(fn: str, rc: int) -> None:
    if rc != WIDE_OK:
        raise WideError(fn, rc)


def _stream(stream, device) -> int:
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return WIDE_BF16
    if t.dtype == torch.float32:
        return WIDE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev_ptr(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _one_device(fn: str, **tensors) -> torch.device:
    """The CUDA device every given tensor is on.  The library launches on the
    current device and takes raw pointers, so operands on another device
    would be handed to kernels that cannot address them: refuse that here
    (ValueError).  None entries are skipped."""
    dev = None
    first = None
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{fn}: {name} must be a CUDA tensor (is on {t.device})")
        if dev is None:
            dev, first = t.device, name
        elif t.device != dev:
            raise ValueError(f"{fn}: {name} is on {t.device} but {first} is on {dev}; "
                             "every operand must be on one device")
    if dev is None:
        raise ValueError(f"{fn}: no tensor operand")
    return dev


# ------------------------------------------------------------------ status

def wide_status_string(code: int) -> str:
    return _L.wide_status_string(int(code)).decode()


def wide_abi_version() -> int:
    return _L.wide_abi_version()


def wide_last_error() -> str:
    return _L.wide_last_error().decode()


def wide_get_device_status(stream=None, device=None) -> int:
    """Synchronises the stream and returns the device status word."""
    v = ctypes.c_int32(0)
    _check("wide_get_device_status",
           _L.wide_get_device_status(ctypes.byref(v), _stream(stream, device)))
    return v.value


def wide_clear_device_status(stream=None, device=None) -> None:
    _check("wide_clear_device_status", _L.wide_clear_device_status(_stream(stream, device)))


# ------------------------------------------------------------ measurement

def wide_profile_start(max_records: int = 4096) -> None:
    _check("wide_profile_start", _L.wide_profile_start(int(max_records)))


def wide_profile_stop() -> None:
    _check("wide_profile_stop", _L.wide_profile_stop())


def wide_profile_read(max_records: int = 65536) -> list:
    """[(kernel name, milliseconds)] for the launches recorded since start."""
    import numpy as np
    ids = np.zeros(max_records, dtype=np.int32)
    ms = np.zeros(max_records, dtype=np.float32)
    n = ctypes.c_int32(0)
    _check("wide_profile_read", _L.wide_profile_read(
        ids.ctypes.data, ms.ctypes.data, max_records, ctypes.byref(n)))
    return [(wide_kernel_name(int(ids[i])), float(ms[i])) for i in range(n.value)]


def wide_kernel_name(kernel_id: int) -> str:
    return _L.wide_kernel_name(int(kernel_id)).decode()


def wide_launch_count() -> int:
    return int(_L.wide_launch_count())


WIDE_DECODE_AUTO, WIDE_DECODE_FUSED, WIDE_DECODE_GEMV, WIDE_DECODE_TC = 0, 1, 2, 3


def wide_set_decode_ffn_path(mode: int) -> int:
    """Selects the kernels of the bf16 decode FFN; returns the previous mode."""
    rc = int(_L.wide_set_decode_ffn_path(int(mode)))
    if rc < 0:
        raise WideError("wide_set_decode_ffn_path", rc)
    return rc


# --------------------------------------------------------- mask reordering

def wide_worklist_bytes(T: int, G: int, tile_m: int = 128) -> int:
    return int(_L.wide_worklist_bytes(T, G, tile_m))


def wide_reorder(mask_words: torch.Tensor, G: int, tile_m: int = 128, buf: torch.Tensor = None,
                 stream=None) -> dict:
    """Device-side mask reordering (section 2.B) of an int32/uint32 [T][W]
    mask.  Returns tensor views into one device buffer: count, perm,
    items ([n_cap][2]), n_items ([1]), sig_perm, sig_pos, tile_union."""
    T, W = mask_words.shape
    if W != (G + 31) // 32:
        raise ValueError("mask has the wrong number of words per token")
    nbytes = wide_worklist_bytes(T, G, tile_m)
    if nbytes == 0:
        raise WideError("wide_worklist_bytes", WIDE_EINVAL)
    dev = _one_device("wide_reorder", mask_words=mask_words, buf=buf)
    if buf is None:
        buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    wl = WideWorklist()
    _check("wide_worklist_carve", _L.wide_worklist_carve(
        buf.data_ptr(), buf.numel(), T, G, tile_m, ctypes.byref(wl)))
    with torch.cuda.device(dev):
        _check("wide_reorder", _L.wide_reorder(
            _dev_ptr(mask_words, "mask_words"), T, G, tile_m, ctypes.byref(wl),
            _stream(stream, dev)))
    base = buf.data_ptr()
    nt = (T + tile_m - 1) // tile_m

    def view(ptr, n, dt=torch.int32):
        off = ptr - base
        return buf[off:off + 4 * n].view(dt)

    return {
        "count": view(wl.count, G),
        "perm": view(wl.perm, G * T).view(G, T),
        "items": view(wl.items, 2 * G * nt).view(G * nt, 2),
        "n_items": view(wl.n_items, 1),
        "sig_perm": view(wl.sig_perm, T),
        "sig_pos": view(wl.sig_pos, T),
        "tile_union": view(wl.tile_union, nt * W).view(nt, W),
        "_buf": buf,
        "_wl": wl,
        "_key": (T, G, tile_m),
    }


# -------------------------------------------------------------- masked FFN

def _check_ffn(x, w_gate, w_up, w_down, mask_words, group_size, out) -> None:
    """Dtypes and shapes the C ABI cannot see (it takes raw pointers)."""
    T, H = x.shape
    I = w_gate.shape[0]
    for name, t in (("w_gate", w_gate), ("w_up", w_up), ("w_down", w_down)):
        if t.dtype != x.dtype:
            raise TypeError(f"{name} is {t.dtype}, x is {x.dtype}")
    if tuple(w_gate.shape) != (I, H) or tuple(w_up.shape) != (I, H) or \
            tuple(w_down.shape) != (H, I):
        raise ValueError(f"weights {tuple(w_gate.shape)}, {tuple(w_up.shape)}, "
                         f"{tuple(w_down.shape)} do not fit x [{T}][{H}]: expected "
                         f"W_gate, W_up [I][{H}] and W_down [{H}][I]")
    if group_size > 0 and I % group_size == 0:
        W = (I // group_size + 31) // 32
        if mask_words.dtype != torch.int32 or tuple(mask_words.shape) != (T, W):
            raise ValueError(f"mask_words must be int32 [{T}][{W}], got {mask_words.dtype} "
                             f"{tuple(mask_words.shape)}")
    if out is not None and (out.dtype != x.dtype or tuple(out.shape) != (T, H)):
        raise ValueError(f"out must be {x.dtype} [{T}][{H}]")


def _ffn_dims(x, w_gate, group_size, path) -> WideFFNDims:
    T, H = x.shape
    I = w_gate.shape[0]
    return WideFFNDims(T, H, I, group_size, _dtype_code(x), path)


def wide_ffn_workspace_bytes(T: int, H: int, I: int, group_size: int, dtype=torch.bfloat16,
                             path: int = WIDE_PATH_AUTO) -> int:
    d = WideFFNDims(T, H, I, group_size, WIDE_BF16 if dtype == torch.bfloat16 else WIDE_F32, path)
    return int(_L.wide_ffn_workspace_bytes(ctypes.byref(d)))


def wide_ffn_masked(x: torch.Tensor, w_gate: torch.Tensor, w_up: torch.Tensor,
                    w_down: torch.Tensor, mask_words: torch.Tensor, group_size: int,
                    out: torch.Tensor = None, workspace: torch.Tensor = None,
                    path: int = WIDE_PATH_AUTO, stream=None, worklist: dict = None) -> torch.Tensor:
    """Masked SwiGLU FFN (section 2.A).  x[T][H]; W_gate/W_up[I][H];
    W_down[H][I]; mask_words int32 [T][ceil(G/32)]; returns out[T][H].
    ``worklist``: the dict wide_reorder returned for this same mask
    (tile_m 128), to reuse that reordering instead of reordering again."""
    _check_ffn(x, w_gate, w_up, w_down, mask_words, group_size, out)
    dev = _one_device("wide_ffn_masked", x=x, w_gate=w_gate, w_up=w_up, w_down=w_down,
                      mask_words=mask_words, out=out, workspace=workspace,
                      worklist=None if worklist is None else worklist["_buf"])
    d = _ffn_dims(x, w_gate, group_size, path)
    wl = None
    if worklist is not None:
        T, I = x.shape[0], w_gate.shape[0]
        if worklist["_key"] != (T, I // group_size if group_size > 0 else -1, 128):
            raise ValueError(f"worklist was built for (T, G, tile_m) = {worklist['_key']}, "
                             f"this call needs ({T}, {I // max(group_size, 1)}, 128)")
        wl = ctypes.byref(worklist["_wl"])
    if out is None:
        out = torch.empty_like(x)
    need = int(_L.wide_ffn_workspace_bytes(ctypes.byref(d)))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check("wide_ffn_masked", _L.wide_ffn_masked(
            _dev_ptr(x, "x"), _dev_ptr(w_gate, "w_gate"), _dev_ptr(w_up, "w_up"),
            _dev_ptr(w_down, "w_down"), _dev_ptr(mask_words, "mask_words"),
            _dev_ptr(out, "out"), ctypes.byref(d), wl, workspace.data_ptr(), workspace.numel(),
            _stream(stream, dev)))
    return out


def wide_ffn_masked_noalloc(x: torch.Tensor, w_gate: torch.Tensor, w_up: torch.Tensor,
                            w_down: torch.Tensor, mask_words: torch.Tensor, group_size: int,
                            out: torch.Tensor, stream=None) -> torch.Tensor:
    """The decode-path masked FFN for callers that cannot allocate device
    memory: no workspace argument, and `out` must be given (this wrapper
    allocates nothing either).  The library keeps the kernels' scratch in a
    fixed device array of WIDE_NOALLOC_SCRATCH_BYTES bytes shared by all
    calls on a device; calls that overlap on the GPU race on it.  Raises
    WideError (WIDE_ETOOLARGE) when min(T, 32) (rounded up to
    an even count) * I * 4 exceeds that size."""
    _check_ffn(x, w_gate, w_up, w_down, mask_words, group_size, out)
    dev = _one_device("wide_ffn_masked_noalloc", x=x, w_gate=w_gate, w_up=w_up, w_down=w_down,
                      mask_words=mask_words, out=out)
    d = _ffn_dims(x, w_gate, group_size, WIDE_PATH_DECODE)
    with torch.cuda.device(dev):
        _check("wide_ffn_masked_noalloc", _L.wide_ffn_masked_noalloc(
            _dev_ptr(x, "x"), _dev_ptr(w_gate, "w_gate"), _dev_ptr(w_up, "w_up"),
            _dev_ptr(w_down, "w_down"), _dev_ptr(mask_words, "mask_words"),
            _dev_ptr(out, "out"), ctypes.byref(d), _stream(stream, dev)))
    return out


def wide_ffn_packed_bytes(hidden: int, inter: int) -> int:
    return int(_L.wide_ffn_packed_bytes(hidden, inter))


def wide_ffn_pack(w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor,
                  packed: torch.Tensor = None, stream=None) -> torch.Tensor:
    """The decode kernel's packed copy of W_gate, W_up [I][H] and W_down
    [H][I] (bf16) as a uint8 device tensor of wide_ffn_packed_bytes(H, I)."""
    I, H = w_gate.shape
    for name, t in (("w_gate", w_gate), ("w_up", w_up), ("w_down", w_down)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} is {t.dtype}; the packed layout is bf16")
    if tuple(w_up.shape) != (I, H) or tuple(w_down.shape) != (H, I):
        raise ValueError(f"weights {tuple(w_gate.shape)}, {tuple(w_up.shape)}, "
                         f"{tuple(w_down.shape)}: expected W_gate, W_up [I][H], W_down [H][I]")
    dev = _one_device("wide_ffn_pack", w_gate=w_gate, w_up=w_up, w_down=w_down, packed=packed)
    need = wide_ffn_packed_bytes(H, I)
    if need == 0:
        raise WideError("wide_ffn_pack", WIDE_EUNSUPPORTED)
    if packed is None:
        packed = torch.empty(need, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check("wide_ffn_pack", _L.wide_ffn_pack(
            _dev_ptr(w_gate, "w_gate"), _dev_ptr(w_up, "w_up"), _dev_ptr(w_down, "w_down"), H, I,
            _dev_ptr(packed, "packed"), packed.numel(), _stream(stream, dev)))
    return packed


def wide_ffn_masked_packed(x: torch.Tensor, packed: torch.Tensor, mask_words: torch.Tensor,
                           group_size: int, inter: int, out: torch.Tensor = None,
                           workspace: torch.Tensor = None, stream=None,
                           weights: tuple = None) -> torch.Tensor:
    """The decode-path masked FFN on a wide_ffn_pack copy of the weights.
    ``weights``: optionally the nn.Linear (w_gate, w_up, w_down) as well, so
    the library can pick the faster kernel per launch (small batches)."""
    T, H = x.shape
    if x.dtype != torch.bfloat16:
        raise TypeError(f"x is {x.dtype}; the packed decode FFN is bf16")
    if packed.dtype != torch.uint8 or packed.numel() < wide_ffn_packed_bytes(H, inter):
        raise ValueError("packed must be the uint8 tensor wide_ffn_pack returned for these sizes")
    if group_size > 0 and inter % group_size == 0:
        W = (inter // group_size + 31) // 32
        if mask_words.dtype != torch.int32 or tuple(mask_words.shape) != (T, W):
            raise ValueError(f"mask_words must be int32 [{T}][{W}], got {mask_words.dtype} "
                             f"{tuple(mask_words.shape)}")
    wg = wu = wd = None
    if weights is not None:
        wg, wu, wd = weights
        _check_ffn(x, wg, wu, wd, mask_words, group_size, out)
    dev = _one_device("wide_ffn_masked_packed", x=x, packed=packed, mask_words=mask_words, out=out,
                      workspace=workspace, w_gate=wg, w_up=wu, w_down=wd)
    d = WideFFNDims(T, H, inter, group_size, WIDE_BF16, WIDE_PATH_DECODE)
    if out is None:
        out = torch.empty_like(x)
    need = int(_L.wide_ffn_workspace_bytes(ctypes.byref(d)))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        lin = [None, None, None] if weights is None else \
            [_dev_ptr(wg, "w_gate"), _dev_ptr(wu, "w_up"), _dev_ptr(wd, "w_down")]
        _check("wide_ffn_masked_packed", _L.wide_ffn_masked_packed(
            _dev_ptr(x, "x"), _dev_ptr(packed, "packed"), *lin, _dev_ptr(mask_words, "mask_words"),
            _dev_ptr(out, "out"), ctypes.byref(d), workspace.data_ptr(), workspace.numel(),
            _stream(stream, dev)))
    return out


# ----------------------------------------------------------- masked layer

LAYER_WEIGHT_NAMES = ("gamma1", "wq", "wk", "wv", "wo", "gamma2", "w_gate", "w_up", "w_down",
                      "ffn_packed")


def wide_layer_dims(n_seq: int, seq_len: int, cache_len: int, cache_cap: int, hidden: int,
                    inter: int, ffn_group_size: int, n_q_heads: int, n_kv_heads: int,
                    head_dim: int = 128, rope_theta: float = 5e5,
                    eps: float = 1e-5) -> WideLayerDims:
    return WideLayerDims(n_seq, seq_len, cache_len, cache_cap, hidden, inter, ffn_group_size,
                         n_q_heads, n_kv_heads, head_dim, rope_theta, eps)


def _weights(w: dict, names=LAYER_WEIGHT_NAMES) -> WideLayerWeights:
    vals = {}
    for n in LAYER_WEIGHT_NAMES:
        t = w.get(n)
        vals[n] = _dev_ptr(t, n) if (t is not None and n in names) else None
    return WideLayerWeights(**vals)


def wide_layer_workspace_bytes(d: WideLayerDims) -> int:
    return int(_L.wide_layer_workspace_bytes(ctypes.byref(d)))


def wide_layer_masked(x: torch.Tensor, weights: dict, k_cache: torch.Tensor,
                      v_cache: torch.Tensor, head_mask: torch.Tensor, ffn_mask: torch.Tensor,
                      d: WideLayerDims, out: torch.Tensor = None, attn_out: torch.Tensor = None,
                      ffn_out: torch.Tensor = None, workspace: torch.Tensor = None,
                      stream=None) -> torch.Tensor:
    """The masked layer (pre-norm block); appends K/V to the caches.
    weights: dict with gamma1, wq, wk, wv, wo, gamma2, w_gate, w_up, w_down,
    and optionally ffn_packed (wide_ffn_pack of the FFN weights), which the
    decode layer's FFN then reads."""
    dev = _one_device("wide_layer_masked", x=x, k_cache=k_cache, v_cache=v_cache,
                      head_mask=head_mask, ffn_mask=ffn_mask, out=out, attn_out=attn_out,
                      ffn_out=ffn_out, workspace=workspace,
                      **{n: weights.get(n) for n in LAYER_WEIGHT_NAMES})
    if out is None:
        out = torch.empty_like(x)
    need = wide_layer_workspace_bytes(d)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    w = _weights(weights)
    with torch.cuda.device(dev):
        _check("wide_layer_masked", _L.wide_layer_masked(
            _dev_ptr(x, "x"), ctypes.byref(w), _dev_ptr(k_cache, "k_cache"),
            _dev_ptr(v_cache, "v_cache"), _dev_ptr(head_mask, "head_mask"),
            _dev_ptr(ffn_mask, "ffn_mask"), _dev_ptr(out, "out"),
            None if attn_out is None else _dev_ptr(attn_out, "attn_out"),
            None if ffn_out is None else _dev_ptr(ffn_out, "ffn_out"),
            ctypes.byref(d), workspace.data_ptr(), workspace.numel(), _stream(stream, dev)))
    return out


def wide_attn_masked(x: torch.Tensor, weights: dict, k_cache: torch.Tensor,
                     v_cache: torch.Tensor, head_mask: torch.Tensor, d: WideLayerDims,
                     attn_out: torch.Tensor = None, workspace: torch.Tensor = None,
                     stream=None) -> torch.Tensor:
    """The masked attention half: attn_out = o_proj(attn(RMSNorm(x) * gamma1))."""
    names = ("gamma1", "wq", "wk", "wv", "wo")
    dev = _one_device("wide_attn_masked", x=x, k_cache=k_cache, v_cache=v_cache,
                      head_mask=head_mask, attn_out=attn_out, workspace=workspace,
                      **{n: weights.get(n) for n in names})
    if attn_out is None:
        attn_out = torch.empty_like(x)
    need = wide_layer_workspace_bytes(d)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    w = _weights(weights, names=names)
    with torch.cuda.device(dev):
        _check("wide_attn_masked", _L.wide_attn_masked(
            _dev_ptr(x, "x"), ctypes.byref(w), _dev_ptr(k_cache, "k_cache"),
            _dev_ptr(v_cache, "v_cache"), _dev_ptr(head_mask, "head_mask"),
            _dev_ptr(attn_out, "attn_out"), ctypes.byref(d), workspace.data_ptr(),
            workspace.numel(), _stream(stream, dev)))
    return attn_out


# ------------------------------------------------------------------ router

def wide_route(x: torch.Tensor, w_r1: torch.Tensor, w_r2: torch.Tensor,
               b_r2: torch.Tensor = None, act: int = WIDE_ACT_RELU,
               mask_words: torch.Tensor = None, logits: torch.Tensor = None,
               stream=None) -> torch.Tensor:
    """Bottleneck router (section 2.A): execute bits of act(x W_r1^T) W_r2^T
    + b_r2 > 0, packed.  x bf16 [T][H]; W_r1 bf16 [R][H]; W_r2 bf16 [G][R];
    b_r2 fp32 [G] or None; returns int32 mask words [T][ceil(G/32)].  If
    `logits` (fp32 [T][G]) is given, the logits are written there too."""
    T, H = x.shape
    R, G = w_r1.shape[0], w_r2.shape[0]
    for name, t in (("x", x), ("w_r1", w_r1), ("w_r2", w_r2)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if tuple(w_r1.shape) != (R, H) or tuple(w_r2.shape) != (G, R):
        raise ValueError(f"w_r1 {tuple(w_r1.shape)} / w_r2 {tuple(w_r2.shape)} do not fit "
                         f"x [{T}][{H}]: expected [R][{H}] and [G][R]")
    if b_r2 is not None and (b_r2.dtype != torch.float32 or tuple(b_r2.shape) != (G,)):
        raise ValueError(f"b_r2 must be float32 [{G}]")
    if mask_words is not None and (mask_words.dtype != torch.int32 or
                                   tuple(mask_words.shape) != (T, (G + 31) // 32)):
        raise ValueError(f"mask_words must be int32 [{T}][{(G + 31) // 32}]")
    if logits is not None and (logits.dtype != torch.float32 or tuple(logits.shape) != (T, G)):
        raise ValueError(f"logits must be float32 [{T}][{G}]")
    dev = _one_device("wide_route", x=x, w_r1=w_r1, w_r2=w_r2, b_r2=b_r2,
                      mask_words=mask_words, logits=logits)
    if mask_words is None:
        mask_words = torch.empty((T, (G + 31) // 32), dtype=torch.int32, device=dev)
    d = WideRouterDims(T, H, R, G, act)
    with torch.cuda.device(dev):
        _check("wide_route", _L.wide_route(
            _dev_ptr(x, "x"), _dev_ptr(w_r1, "w_r1"), _dev_ptr(w_r2, "w_r2"),
            None if b_r2 is None else _dev_ptr(b_r2, "b_r2"),
            _dev_ptr(mask_words, "mask_words"),
            None if logits is None else _dev_ptr(logits, "logits"), ctypes.byref(d),
            _stream(stream, dev)))
    return mask_words
