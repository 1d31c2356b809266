"""Seeded synthetic inputs for the Atom W4A4 hot path.

This module only draws random numbers. It holds none of the method's
arithmetic (no permutation, no scales, no codes), so both the CPU oracle and
the CUDA path can consume the same inputs without sharing any of the method.

Workloads are the Llama-shaped projections the Atom quantization record is
evaluated on (arXiv 2310.19102, Atom abstract: W4A4 serving with 128-element
groups and 128 high-precision outlier channels). Each workload is

  A fp16 [M, K]  activations: standard normal or standard Student-t draws, with
                 128 seeded channels multiplied by an outlier factor;
  W fp16 [N, K]  weights: N(0, sigma) draws, no planted outliers;
  outlier_idx    int32[128], the planted channels, sorted ascending.

Recipe (fixed, so that results are reproducible anywhere):
  * numpy Generator(PCG64(seed)), seeds 1000+c (A), 2000+c (W), 3000+c
    (outlier choice) for workload index c;
  * values drawn in float64 row-chunk by row-chunk from one generator (the
    chunking does not change the stream), scaled, then cast to float16 with
    round-to-nearest-even; finiteness asserted after the cast;
  * outliers = sorted(rng.choice(K, 128, replace=False)); those A columns are
    multiplied by the factor before the cast.
"""
from __future__ import annotations

import dataclasses

import numpy as np

N_OUTLIER = 128
GROUP = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int
    name: str
    M: int
    N: int
    K: int
    a_dist: str          # "normal" or "t"
    a_param: float       # sigma for "normal", degrees of freedom for "t"
    outlier_factor: float
    w_sigma: float

    @property
    def groups(self) -> int:
        return self.K // GROUP

    def describe(self) -> str:
        a = (f"N(0,{self.a_param:g})" if self.a_dist == "normal"
             else f"Student-t(df={self.a_param:g})")
        return (f"{self.name}: A fp16[{self.M},{self.K}] {a}, 128 outlier channels "
                f"x{self.outlier_factor:g}; W fp16[{self.N},{self.K}] N(0,{self.w_sigma:g}); "
                f"{self.groups - 1} INT4 groups of 128 + 1 INT8 outlier group")


WORKLOADS = (
    Workload(0, "tiny", 16, 256, 512, "normal", 1.0, 20.0, 0.02),
    Workload(1, "llama7b_decode_q_proj", 64, 4096, 4096, "t", 4.0, 30.0, 0.02),
    Workload(2, "llama7b_prefill_up_proj", 4096, 11008, 4096, "t", 4.0, 30.0, 0.02),
    Workload(3, "llama7b_down_proj", 8192, 4096, 11008, "t", 3.0, 50.0, 0.015),
    Workload(4, "llama70b_mlp_up", 8192, 28672, 8192, "t", 4.0, 30.0, 0.01),
)

_CHUNK_ROWS = 2048


def workload(c: int) -> Workload:
    return WORKLOADS[c]


def outlier_channels(c: int) -> np.ndarray:
    w = WORKLOADS[c]
    rng = np.random.Generator(np.random.PCG64(3000 + c))
    idx = np.sort(rng.choice(w.K, N_OUTLIER, replace=False))
    return idx.astype(np.int32)


def _draw_rows(rng, dist: str, param: float, rows: int, K: int) -> np.ndarray:
    if dist == "normal":
        return rng.standard_normal((rows, K)) * param
    if dist == "t":
        return rng.standard_t(param, (rows, K))
    raise ValueError(dist)


def activations(c: int, rows: int | None = None) -> np.ndarray:
    """A fp16 [rows, K]: the first `rows` rows of workload c's activations."""
    w = WORKLOADS[c]
    rows = w.M if rows is None else min(rows, w.M)
    rng = np.random.Generator(np.random.PCG64(1000 + c))
    idx = outlier_channels(c)
    out = np.empty((rows, w.K), dtype=np.float16)
    for r0 in range(0, rows, _CHUNK_ROWS):
        r1 = min(rows, r0 + _CHUNK_ROWS)
        v = _draw_rows(rng, w.a_dist, w.a_param, r1 - r0, w.K)
        v[:, idx] *= w.outlier_factor
        out[r0:r1] = v.astype(np.float16)
    assert np.isfinite(out).all(), "activation draw overflowed fp16"
    return out


def weights(c: int, rows: int | None = None) -> np.ndarray:
    """W fp16 [rows, K]: the first `rows` rows of workload c's weights."""
    w = WORKLOADS[c]
    rows = w.N if rows is None else min(rows, w.N)
    rng = np.random.Generator(np.random.PCG64(2000 + c))
    out = np.empty((rows, w.K), dtype=np.float16)
    for r0 in range(0, rows, _CHUNK_ROWS):
        r1 = min(rows, r0 + _CHUNK_ROWS)
        out[r0:r1] = (rng.standard_normal((r1 - r0, w.K)) * w.w_sigma).astype(np.float16)
    assert np.isfinite(out).all()
    return out


def random_case(seed: int, M: int, N: int, K: int, dist: str = "t", param: float = 4.0,
                outlier_factor: float = 30.0, w_sigma: float = 0.02,
                sorted_outliers: bool = True):
    """A free-form seeded case (ragged sizes, edge cases) with the same recipe."""
    rng = np.random.Generator(np.random.PCG64(seed))
    idx = rng.choice(K, N_OUTLIER, replace=False)
    if sorted_outliers:
        idx = np.sort(idx)
    a = _draw_rows(rng, dist, param, M, K)
    a[:, idx] *= outlier_factor
    wt = rng.standard_normal((N, K)) * w_sigma
    A = a.astype(np.float16)
    W = wt.astype(np.float16)
    assert np.isfinite(A).all() and np.isfinite(W).all()
    return A, W, idx.astype(np.int32)


def int8_case(seed: int, M: int, N: int, K: int):
    """Operands of the W8A8 comparator: int8 qa [M, K] and qw [N, K] uniform on
    [-127, 127], and positive fp32 row scales sa [M] and column scales sw [N]
    (log-uniform over two decades), all from Generator(PCG64(seed))."""
    rng = np.random.Generator(np.random.PCG64(seed))
    qa = rng.integers(-127, 128, size=(M, K), dtype=np.int16).astype(np.int8)
    qw = rng.integers(-127, 128, size=(N, K), dtype=np.int16).astype(np.int8)
    sa = (10.0 ** rng.uniform(-4.0, -2.0, size=M)).astype(np.float32)
    sw = (10.0 ** rng.uniform(-4.0, -2.0, size=N)).astype(np.float32)
    return qa, qw, sa, sw


def kv_cache(seed: int, tokens: int, heads: int, head_dim: int = 128) -> np.ndarray:
    """fp16 [tokens, heads, head_dim] key/value vectors: standard normal draws,
    each (token, head) vector scaled by a log-uniform factor over four decades,
    and one seeded element per vector in 64 multiplied by 8 (an outlier);
    Generator(PCG64(seed))."""
    rng = np.random.Generator(np.random.PCG64(seed))
    v = rng.standard_normal((tokens, heads, head_dim))
    v *= 10.0 ** rng.uniform(-2.0, 2.0, size=(tokens, heads, 1))
    spikes = rng.random((tokens, heads, head_dim)) < 1.0 / 64
    v[spikes] *= 8.0
    out = v.astype(np.float16)
    assert np.isfinite(out).all()
    return out
