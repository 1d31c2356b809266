"""INT4 KV-cache quantization -- TEST INFRASTRUCTURE ONLY (the GPU path never uses it).

The pages file Atom under KV-cache quantization ("Atom: Low-bit Quantization
for Efficient and Accurate LLM Serving", key facts: placed in KV cache
quantization) but give no KV-cache recipe. The plainest reading that the rest
of the pages supports, used here: every (token, head) vector of
head_dim = 128 elements is one group, quantized exactly like an Atom INT4
activation group ("Atom (mixed-precision block-outlier low-bit quantization
for serving)", fields Bits and Weight group size: 4-bit, independent groups of
128), with no reorder and no outlier channels:

  scale = fl32(amax / 7), inv = fl32(7 / amax)   (0 and 0 for an all-zero group)
  q     = rint(fl32(x * inv)), ties to even, in [-7, 7]
  bytes = element 2i in the low nibble of byte i, 2i+1 in the high nibble
  dequantized x' = fp16_rn(fl32(q * scale))
"""
from __future__ import annotations

import numpy as np

HEAD_DIM = 128


def quantize(x: np.ndarray):
    """fp16 [..., 128] -> (q4 uint8 [..., 64], scale float32 [...])."""
    x = np.asarray(x, dtype=np.float16)
    if x.shape[-1] != HEAD_DIM:
        raise ValueError("the last axis must be head_dim = 128")
    xf = x.astype(np.float32)
    amax = np.abs(xf).max(axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        scale = np.where(amax > 0, amax / np.float32(7), np.float32(0)).astype(np.float32)
        inv = np.where(amax > 0, np.float32(7) / amax, np.float32(0)).astype(np.float32)
    t = (xf * inv[..., None]).astype(np.float32)
    q = np.rint(t).astype(np.int64)
    nib = (q & 0xF).astype(np.uint8)
    q4 = (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)
    return q4, scale


def codes(q4: np.ndarray) -> np.ndarray:
    """Signed codes int64 [..., 128] from the packed bytes."""
    q4 = np.asarray(q4, dtype=np.uint8)
    lo = (q4 & 0xF).astype(np.int64)
    hi = (q4 >> 4).astype(np.int64)
    nib = np.empty(q4.shape[:-1] + (q4.shape[-1] * 2,), dtype=np.int64)
    nib[..., 0::2] = lo
    nib[..., 1::2] = hi
    return np.where(nib >= 8, nib - 16, nib)


def dequantize(q4: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """fp16 [..., 128]: fp16_rn(fl32(q * scale))."""
    q = codes(q4).astype(np.float32)
    return (q * np.asarray(scale, dtype=np.float32)[..., None]).astype(np.float32).astype(np.float16)
