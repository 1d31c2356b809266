"""W4A8 variant -- TEST INFRASTRUCTURE ONLY (the GPU path never uses it).

The pages set Atom's W4A4 kernels beside 8-bit activation schemes; the W4A8
variant kept here changes only the activations: every 128-channel group of the
reordered activation row is quantized to INT8, the dense groups included
("Atom (mixed-precision block-outlier low-bit quantization for serving)",
fields Weight group size and notes: contiguous 128-element groups quantized
independently). The weights keep the W4A4 encoding (INT4 groups, the 128
outlier channels as one INT8 group). Per row and group g of the reordered row:

    scale = fl32(amax / 127), inv = fl32(127 / amax)   (both 0 when amax == 0)
    q     = rint(fl32(x * inv)), ties to even           (|q| <= 127)

stored as int8 [rows, K] in reordered order, scales float32 [K/128, rows]. The
GEMM is the W4A4 one with these codes:

    P[g, m, n] = sum_{k in g} qa[m, k] * qw[n, k]       (exact integers)
    Y64[m, n]  = sum_g sa[g, m] * sw[g, n] * P[g, m, n] (float64)
"""
from __future__ import annotations

import numpy as np

from . import numpy_oracle


def quantize_a8(x: np.ndarray, outlier_idx):
    """fp16 [rows, K] -> (q8 int8 [rows, K] in reordered order, scales [K/128, rows])."""
    x = np.asarray(x, dtype=np.float16)
    rows, K = x.shape
    G = K // 128
    perm = numpy_oracle.permutation(K, outlier_idx)
    xr = x[:, perm].astype(np.float32).reshape(rows, G, 128)
    amax = np.abs(xr).max(axis=2)
    qmax = np.float32(127.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        scale = np.where(amax > 0, amax / qmax, np.float32(0)).astype(np.float32)
        inv = np.where(amax > 0, qmax / amax, np.float32(0)).astype(np.float32)
    t = (xr * inv[:, :, None]).astype(np.float32)
    q = np.rint(t).astype(np.int64)
    if np.abs(q).max(initial=0) > 127:
        raise AssertionError("a code left [-127, 127]")
    return q.reshape(rows, K).astype(np.int8), np.ascontiguousarray(scale.T)


def partials(qa8: np.ndarray, qw4: np.ndarray, qw8: np.ndarray) -> np.ndarray:
    """Exact per-group P as int64 [G, M, N] (integer matmuls of the group slices)."""
    a = np.asarray(qa8).astype(np.int64)
    w = numpy_oracle.codes(qw4, qw8)
    if a.shape[1] != w.shape[1]:
        raise ValueError("activation and weight rows must have the same K")
    G = a.shape[1] // 128
    return np.stack([a[:, g * 128:(g + 1) * 128] @ w[:, g * 128:(g + 1) * 128].T
                     for g in range(G)])


def output64(P: np.ndarray, sa: np.ndarray, sw: np.ndarray) -> np.ndarray:
    """Y64[m, n] = sum_g sa[g, m] * sw[g, n] * P[g, m, n] in float64."""
    return np.einsum("gm,gn,gmn->mn", sa.astype(np.float64), sw.astype(np.float64),
                     P.astype(np.float64))
