"""Independent numpy restatement of the Atom W4A4 encoding -- TEST INFRASTRUCTURE ONLY.

Written separately from `atom_oracle.c` (vectorised over rows instead of plain
loops) so that the two can be compared bit for bit. It follows the same
readings of the Atom pages ("Atom (mixed-precision block-outlier low-bit
quantization for serving)", fields "Weight group size" and "notes": independent
128-element groups and a 128-channel high-precision outlier group):

  permutation : ascending non-outlier channels, then the outlier list in order;
  scale       : amax/qmax and inv = qmax/amax in float32 (qmax 7 or 127);
  code        : rint(float32(x*inv)), ties to even;
  packing     : element 2i -> low nibble of byte i, 2i+1 -> high nibble.
"""
from __future__ import annotations

import numpy as np


def permutation(K: int, outlier_idx) -> np.ndarray:
    idx = np.asarray(outlier_idx, dtype=np.int64)
    if idx.size != len(set(idx.tolist())) or (idx < 0).any() or (idx >= K).any():
        raise ValueError("outlier list must hold distinct channels in [0, K)")
    keep = np.ones(K, dtype=bool)
    keep[idx] = False
    return np.concatenate([np.nonzero(keep)[0], idx]).astype(np.int64)


def quantize(x: np.ndarray, outlier_idx, *, rounding=np.rint, high_nibble_first=False,
             int4_qmax=7.0, reorder=True):
    """fp16 [rows, K] -> (q4 [rows, (K-128)/2], q8 [rows, 128], scales [K/128, rows]).

    The keyword arguments exist only so the tests can plant a mistake in a copy
    of the encoding and check that the hand-worked pins catch it; their defaults
    are the readings above."""
    x = np.asarray(x, dtype=np.float16)
    rows, K = x.shape
    G = K // 128
    perm = permutation(K, outlier_idx)
    if not reorder:
        perm = np.arange(K)
    xr = x[:, perm].astype(np.float32).reshape(rows, G, 128)
    qmax = np.full(G, int4_qmax, dtype=np.float32)
    qmax[-1] = 127.0
    amax = np.abs(xr).max(axis=2)                                   # [rows, G]
    with np.errstate(divide="ignore", invalid="ignore"):
        scale = np.where(amax > 0, amax / qmax[None, :], np.float32(0)).astype(np.float32)
        inv = np.where(amax > 0, qmax[None, :] / amax, np.float32(0)).astype(np.float32)
    t = (xr * inv[:, :, None]).astype(np.float32)
    q = rounding(t).astype(np.int64)
    qmax_i = np.where(np.arange(G) < G - 1, 7, 127).astype(np.int64)
    q = np.clip(q, -(qmax_i + 1)[None, :, None], qmax_i[None, :, None])
    dense = q[:, :G - 1, :].reshape(rows, -1)
    nib = (dense & 0xF).astype(np.uint8)
    first, second = (nib[:, 1::2], nib[:, 0::2]) if high_nibble_first else (nib[:, 0::2], nib[:, 1::2])
    q4 = (first | (second << 4)).astype(np.uint8)
    q8 = q[:, G - 1, :].astype(np.int8)
    return q4, q8, np.ascontiguousarray(scale.T)                    # scales [G, rows]


def codes(q4: np.ndarray, q8: np.ndarray) -> np.ndarray:
    """Signed code per reordered position, int64 [rows, K]."""
    lo = (q4 & 0xF).astype(np.int64)
    hi = (q4 >> 4).astype(np.int64)
    nib = np.empty((q4.shape[0], q4.shape[1] * 2), dtype=np.int64)
    nib[:, 0::2] = lo
    nib[:, 1::2] = hi
    nib = np.where(nib >= 8, nib - 16, nib)
    return np.concatenate([nib, q8.astype(np.int64)], axis=1)


def partials(qa4, qa8, qw4, qw8) -> np.ndarray:
    a = codes(qa4, qa8)
    w = codes(qw4, qw8)
    G = a.shape[1] // 128
    P = np.stack([a[:, g * 128:(g + 1) * 128] @ w[:, g * 128:(g + 1) * 128].T for g in range(G)])
    assert np.abs(P).max(initial=0) < 2 ** 31
    return P.astype(np.int64)


def output64(P: np.ndarray, sa: np.ndarray, sw: np.ndarray) -> np.ndarray:
    """Y64[m,n] = sum_g sa[g,m]*sw[g,n]*P[g,m,n] in float64."""
    return np.einsum("gm,gn,gmn->mn", sa.astype(np.float64), sw.astype(np.float64),
                     P.astype(np.float64))
