"""The plain CPU baseline (``plain_rht_quant.c``): build and call.

TEST INFRASTRUCTURE ONLY: the timed CPU speed line of the rotate + quantise step (a scalar
O(K log K) FWHT + group quantisation loop per row, in the style of the Hadamard-Int4-Accuracy
wiki's probe, Method: fwht_norm, q_dequant_vec), pinned against the fp64 definitions of this
package by ``tests/test_oracle_pins.py``. Never called by the library.
"""
from __future__ import annotations

import ctypes as C
import os
import shutil
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "plain_rht_quant.c")
LIB = os.path.join(HERE, "_lib", "libplain_rht_quant.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C baseline with gcc (-O2, OpenMP) into ``oracle/_lib``."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        raise RuntimeError("no C compiler for the plain CPU baseline")
    cmd = [cc, "-O2", "-fopenmp", "-shared", "-fPIC", SRC, "-o", LIB, "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"building the plain CPU baseline failed:\n{r.stderr}")
    return LIB


def _load():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.plain_rht_quant.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_int, C.c_void_p, C.c_int, C.c_int,
                                         C.c_void_p, C.c_void_p, C.c_int]
        _lib.plain_rht_quant.restype = C.c_int
        _lib.plain_max_threads.restype = C.c_int
    return _lib


def max_threads() -> int:
    return int(_load().plain_max_threads())


def rht_quant(A: np.ndarray, signs, bits: int, G: int, threads: int = 0):
    """Rows of A (fp32) -> (packed codes uint8 [M, K*bits/8], scales fp16 [M, K/G])."""
    lib = _load()
    A = np.ascontiguousarray(A, dtype=np.float32)
    M, K = A.shape
    codes = np.empty((M, K * bits // 8), dtype=np.uint8)
    scales = np.empty((M, K // G), dtype=np.float16)
    sg = None
    if signs is not None:
        sg = np.ascontiguousarray(signs, dtype=np.int8)
    st = lib.plain_rht_quant(A.ctypes.data, M, K, K, sg.ctypes.data if sg is not None else None, bits, G,
                             codes.ctypes.data, scales.ctypes.data, threads)
    if st != 0:
        raise ValueError("plain_rht_quant: K must be a power of two, bits 2 or 4, G | K")
    return codes, scales
