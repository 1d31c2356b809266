"""Helpers shared by the GPU parity tests (host-side marshalling and the
output tolerance). The expected values always come from the CPU oracle run on
the same seeded fp16 inputs, never from the CUDA path."""
from __future__ import annotations

import numpy as np
import torch

from w4a4_mixed_precision_b200 import atom

# Output tolerance: max |y - Y64| / max(|Y64|, 1e-2 * rms(Y64)) <= 1e-3.
# fp16 rounding alone contributes up to 2^-11 (4.9e-4) relative; the floor of
# 1e-2*rms keeps elements that cancel to ~0 from demanding an impossible
# relative accuracy of the fp32 accumulation.
Y_TOL = 1e-3


def y_rel_err(y: np.ndarray, Y64: np.ndarray) -> float:
    rms = float(np.sqrt(np.mean(Y64 * Y64))) if Y64.size else 0.0
    denom = np.maximum(np.abs(Y64), max(1e-2 * rms, 1e-30))
    return float(np.max(np.abs(y.astype(np.float64) - Y64) / denom)) if Y64.size else 0.0


def fp16_dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a, dtype=np.float16)
    return torch.from_numpy(a.view(np.uint16)).cuda().view(torch.float16)


def idx_dev(idx: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).cuda()


def quant_dev(x: np.ndarray, idx: np.ndarray, weights: bool = False) -> atom.Quantized:
    fn = atom.atom_quant_weights if weights else atom.atom_reorder_quant
    return fn(fp16_dev(x), idx_dev(idx))


def host(q: atom.Quantized):
    torch.cuda.synchronize()
    return q.q4.cpu().numpy(), q.q8.cpu().numpy(), q.scales.cpu().numpy()


def rows_of(q: atom.Quantized, r0: int, r1: int) -> atom.Quantized:
    """Row window [r0, r1) of a quantized operand, as contiguous tensors."""
    return atom.Quantized(q.q4[r0:r1].contiguous(), q.q8[r0:r1].contiguous(),
                          q.scales[:, r0:r1].contiguous())


def assert_codes_equal(got, want, what=""):
    names = ("q4", "q8", "scales")
    for name, g, w in zip(names, got, want):
        assert g.shape == w.shape, (what, name, g.shape, w.shape)
        gb, wb = g.view(np.uint8), w.view(np.uint8)
        if not np.array_equal(gb, wb):
            bad = np.argwhere(g != w)
            raise AssertionError(f"{what} {name}: {len(bad)} mismatches, first at {bad[:3].tolist()}")
