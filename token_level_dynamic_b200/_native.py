"""ctypes declarations of libwide.so (the C ABI in include/wide.h).

Loading fails loudly: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwide.so")

c_void_p, c_int, c_int32, c_int64, c_size_t = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int32,
                                              ctypes.c_int64, ctypes.c_size_t)

# constants mirrored from wide.h
WIDE_OK = 0
WIDE_EINVAL = -1
WIDE_EUNSUPPORTED = -2
WIDE_EWORKSPACE = -3
WIDE_ECUDA = -4
WIDE_ETOOLARGE = -5
WIDE_NOALLOC_SCRATCH_BYTES = 2097152
WIDE_DEV_BAD_MASK = 0x1
WIDE_DEV_TIMEOUT = 0x2
WIDE_DEV_BAD_ITEM = 0x4
WIDE_DEV_LAYOUT = 0x8
WIDE_BF16 = 0
WIDE_F32 = 1
WIDE_PATH_AUTO = 0
WIDE_PATH_DECODE = 1
WIDE_PATH_PREFILL = 2
WIDE_ACT_RELU = 0
WIDE_ACT_SILU = 1


class WideWorklist(ctypes.Structure):
    _fields_ = [("count", c_void_p), ("perm", c_void_p), ("items", c_void_p),
                ("n_items", c_void_p), ("sig_perm", c_void_p), ("sig_pos", c_void_p),
                ("tile_union", c_void_p), ("scratch", c_void_p),
                ("tokens", c_int64), ("groups", c_int64),
                ("tile_m", c_int32), ("scratch_splits", c_int32)]


class WideFFNDims(ctypes.Structure):
    _fields_ = [("tokens", c_int64), ("hidden", c_int64), ("inter", c_int64),
                ("group_size", c_int64), ("dtype", c_int32), ("path", c_int32)]


class WideLayerDims(ctypes.Structure):
    _fields_ = [("n_seq", c_int64), ("seq_len", c_int64), ("cache_len", c_int64),
                ("cache_cap", c_int64), ("hidden", c_int64), ("inter", c_int64),
                ("ffn_group_size", c_int64), ("n_q_heads", c_int32), ("n_kv_heads", c_int32),
                ("head_dim", c_int32), ("rope_theta", ctypes.c_float), ("eps", ctypes.c_float)]


class WideLayerWeights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("gamma1", "wq", "wk", "wv", "wo",
                                        "gamma2", "w_gate", "w_up", "w_down", "ffn_packed")]


class WideRouterDims(ctypes.Structure):
    _fields_ = [("tokens", c_int64), ("hidden", c_int64), ("bottleneck", c_int64),
                ("groups", c_int64), ("act", c_int32)]


# name -> (restype, argtypes); every symbol include/wide.h declares
SIGNATURES = {
    "wide_status_string": (ctypes.c_char_p, [c_int]),
    "wide_abi_version": (c_int, []),
    "wide_last_error": (ctypes.c_char_p, []),
    "wide_get_device_status": (c_int, [c_void_p, c_void_p]),
    "wide_clear_device_status": (c_int, [c_void_p]),
    "wide_profile_start": (c_int, [c_int32]),
    "wide_profile_stop": (c_int, []),
    "wide_profile_read": (c_int, [c_void_p, c_void_p, c_int32, c_void_p]),
    "wide_kernel_name": (ctypes.c_char_p, [c_int32]),
    "wide_launch_count": (c_int64, []),
    "wide_set_decode_ffn_path": (c_int, [c_int]),
    "wide_worklist_bytes": (c_size_t, [c_int64, c_int64, c_int32]),
    "wide_worklist_carve": (c_int, [c_void_p, c_size_t, c_int64, c_int64, c_int32,
                                    ctypes.POINTER(WideWorklist)]),
    "wide_reorder": (c_int, [c_void_p, c_int64, c_int64, c_int32,
                             ctypes.POINTER(WideWorklist), c_void_p]),
    "wide_ffn_workspace_bytes": (c_size_t, [ctypes.POINTER(WideFFNDims)]),
    "wide_ffn_masked": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                ctypes.POINTER(WideFFNDims), ctypes.POINTER(WideWorklist),
                                c_void_p, c_size_t, c_void_p]),
    "wide_ffn_packed_bytes": (c_size_t, [c_int64, c_int64]),
    "wide_ffn_pack": (c_int, [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_void_p, c_size_t,
                              c_void_p]),
    "wide_ffn_masked_packed": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, ctypes.POINTER(WideFFNDims), c_void_p, c_size_t,
                                       c_void_p]),
    "wide_ffn_masked_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                        c_void_p, ctypes.POINTER(WideFFNDims), c_void_p]),
    "wide_layer_workspace_bytes": (c_size_t, [ctypes.POINTER(WideLayerDims)]),
    "wide_layer_masked": (c_int, [c_void_p, ctypes.POINTER(WideLayerWeights), c_void_p, c_void_p,
                                  c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                  ctypes.POINTER(WideLayerDims), c_void_p, c_size_t, c_void_p]),
    "wide_attn_masked": (c_int, [c_void_p, ctypes.POINTER(WideLayerWeights), c_void_p, c_void_p,
                                 c_void_p, c_void_p, ctypes.POINTER(WideLayerDims), c_void_p,
                                 c_size_t, c_void_p]),
    "wide_route": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                           ctypes.POINTER(WideRouterDims), c_void_p]),
}

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python token_level_dynamic_b200/build.py`"
                " (there is no non-CUDA implementation)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib
