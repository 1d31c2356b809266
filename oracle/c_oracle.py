"""ctypes wrapper around the C oracle -- TEST INFRASTRUCTURE ONLY.

Every function takes and returns numpy arrays; the arithmetic is in
`atom_oracle.c` (see its header for the readings S1-S6 of the Atom pages).
"""
from __future__ import annotations

import ctypes as ct
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ct.CDLL(path)
        i64, i32, p = ct.c_int64, ct.c_int32, ct.c_void_p
        _lib.atom_oracle_f16_to_f32.argtypes = [ct.c_uint16]
        _lib.atom_oracle_f16_to_f32.restype = ct.c_float
        _lib.atom_oracle_f32_to_f16.argtypes = [ct.c_float]
        _lib.atom_oracle_f32_to_f16.restype = ct.c_uint16
        _lib.atom_oracle_permutation.argtypes = [i64, p, i32, p]
        _lib.atom_oracle_quantize.argtypes = [p, i64, i64, i64, p, i32, i32, p, p, p]
        _lib.atom_oracle_partials.argtypes = [p, p, p, p, i64, i64, i64, p]
        _lib.atom_oracle_gemm.argtypes = [p, p, p, p, p, p, i64, i64, i64, p, p]
        _lib.atom_oracle_dequantize.argtypes = [p, p, p, i64, i64, p]
        for f in ("atom_oracle_permutation", "atom_oracle_quantize", "atom_oracle_partials",
                  "atom_oracle_gemm", "atom_oracle_dequantize"):
            getattr(_lib, f).restype = ct.c_int
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data_as(ct.c_void_p)


class OracleError(RuntimeError):
    pass


def set_threads(n: int) -> None:
    os.environ["OMP_NUM_THREADS"] = str(n)


def f16_to_f32(bits: int) -> float:
    return lib().atom_oracle_f16_to_f32(bits)


def f32_to_f16(x: float) -> int:
    return lib().atom_oracle_f32_to_f16(x)


def permutation(K: int, outlier_idx) -> np.ndarray:
    idx = np.ascontiguousarray(outlier_idx, dtype=np.int32)
    perm = np.empty(K, dtype=np.int32)
    rc = lib().atom_oracle_permutation(K, _ptr(idx), idx.size, _ptr(perm))
    if rc != 0:
        raise OracleError(f"permutation rc={rc}")
    return perm


def quantize(x: np.ndarray, outlier_idx, n_outlier: int = 128, group: int = 128):
    """x fp16 [rows, K] -> (q4 u8 [rows, (K-128)/2], q8 i8 [rows, 128], scales f32 [G, rows])."""
    x = np.ascontiguousarray(x, dtype=np.float16)
    rows, K = x.shape
    idx = np.ascontiguousarray(outlier_idx, dtype=np.int32)
    q4 = np.zeros((rows, max(K - 128, 0) // 2), dtype=np.uint8)
    q8 = np.zeros((rows, 128), dtype=np.int8)
    scales = np.zeros((max(K // 128, 0), rows), dtype=np.float32)
    rc = lib().atom_oracle_quantize(_ptr(x.view(np.uint16)), rows, K, K, _ptr(idx), n_outlier,
                                    group, _ptr(q4), _ptr(q8), _ptr(scales))
    if rc != 0:
        raise OracleError(f"quantize rc={rc}")
    return q4, q8, scales


def partials(qa4, qa8, qw4, qw8, K: int) -> np.ndarray:
    M, N = qa4.shape[0], qw4.shape[0]
    P = np.zeros((K // 128, M, N), dtype=np.int32)
    rc = lib().atom_oracle_partials(_ptr(qa4), _ptr(qa8), _ptr(qw4), _ptr(qw8), M, N, K, _ptr(P))
    if rc != 0:
        raise OracleError(f"partials rc={rc}")
    return P


def gemm(qa4, qa8, sa, qw4, qw8, sw, K: int, want_y32: bool = False):
    """Returns Y64 [M, N] float64 (and Y32 float32 if asked)."""
    M, N = qa4.shape[0], qw4.shape[0]
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    Y64 = np.zeros((M, N), dtype=np.float64)
    Y32 = np.zeros((M, N), dtype=np.float32) if want_y32 else None
    rc = lib().atom_oracle_gemm(_ptr(qa4), _ptr(qa8), _ptr(sa), _ptr(qw4), _ptr(qw8), _ptr(sw),
                                M, N, K, _ptr(Y64), _ptr(Y32) if want_y32 else None)
    if rc != 0:
        raise OracleError(f"gemm rc={rc}")
    return (Y64, Y32) if want_y32 else Y64


def dequantize(q4, q8, scales, K: int) -> np.ndarray:
    rows = q4.shape[0]
    out = np.zeros((rows, K), dtype=np.float64)
    rc = lib().atom_oracle_dequantize(_ptr(q4), _ptr(q8), _ptr(np.ascontiguousarray(scales)),
                                      rows, K, _ptr(out))
    if rc != 0:
        raise OracleError(f"dequantize rc={rc}")
    return out
