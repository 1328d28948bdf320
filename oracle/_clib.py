"""Build and load the oracle's C library (fp64 CPU reference).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the CUDA path.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wide_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_OUT_DIR, "libwide_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile wide_oracle.c with gcc (-O2, OpenMP); returns the .so path."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".{os.getpid()}.tmp"
    cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        _lib.oracle_check_mask.argtypes = [P, I64, I64]
        _lib.oracle_reorder.argtypes = [P, I64, I64, I64, P, P, P, P, P, P]
        _lib.oracle_ffn_token_loop.argtypes = [P, P, P, P, P, I64, I64, I64, I64, I, P]
        _lib.oracle_num_threads.argtypes = []
        for f in (_lib.oracle_check_mask, _lib.oracle_reorder, _lib.oracle_ffn_token_loop,
                  _lib.oracle_num_threads):
            f.restype = ctypes.c_int
    return _lib
