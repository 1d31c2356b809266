"""W8A8 comparator output -- TEST INFRASTRUCTURE ONLY (the GPU path never uses it).

The Atom paper ("Atom: Low-bit Quantization for Efficient and Accurate LLM
Serving", summary of results) measures its W4A4 kernels against serving with
8-bit weights and activations. The pages give no INT8 kernel, so this states
the plain per-row x per-column scaled INT8 GEMM that the comparator computes:

    P[m, n] = sum_k qa[m, k] * qw[n, k]          (exact integer dot product)
    Y[m, n] = (P[m, n] * sa[m]) * sw[n]           (float64 here)

A per-tensor scale is the special case of constant sa and sw.
"""
from __future__ import annotations

import numpy as np


def partials(qa: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """Exact P as int64 [M, N]: the float64 product of integer matrices is exact
    while every partial sum stays below 2^53 (|P| <= K * 127^2 < 2^31 here)."""
    qa = np.asarray(qa)
    qw = np.asarray(qw)
    if qa.dtype != np.int8 or qw.dtype != np.int8 or qa.shape[1] != qw.shape[1]:
        raise ValueError("qa [M, K] and qw [N, K] must be int8 with the same K")
    a = qa.astype(np.float64)
    P = np.empty((qa.shape[0], qw.shape[0]), dtype=np.int64)
    for n0 in range(0, qw.shape[0], 2048):   # blocks of W rows bound the float64 copy
        P[:, n0:n0 + 2048] = np.rint(a @ qw[n0:n0 + 2048].astype(np.float64).T)
    return P


def output64(qa: np.ndarray, sa: np.ndarray, qw: np.ndarray, sw: np.ndarray) -> np.ndarray:
    """Y [M, N] in float64: (P * sa[m]) * sw[n]."""
    P = partials(qa, qw).astype(np.float64)
    sa = np.asarray(sa, dtype=np.float32).astype(np.float64)
    sw = np.asarray(sw, dtype=np.float32).astype(np.float64)
    return (P * sa[:, None]) * sw[None, :]
