"""Python binding of the C ABI in include/atom.h (argument marshalling only).

Every function here forwards to `libatom_b200.so`: the tensors' device
pointers, sizes and the current CUDA stream go in, a status code comes back,
and any status other than ATOM_OK raises AtomError. There is no fallback: if
the library is missing or the device is not an sm_100 part, the calls fail.

Layouts (see include/atom.h): for R rows of K channels with G = K/128,
  q4     uint8  [R, (K-128)/2]   two INT4 codes per byte, element 2i low nibble
  q8     int8   [R, 128]         INT8 codes of the outlier channels, list order
  scales float32 [G, R]          group-major scales (last row = outlier group)
"""
from __future__ import annotations

import ctypes as ct
import os
from typing import NamedTuple, Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libatom_b200.so")

STATUS = {
    0: "ATOM_OK",
    1: "ATOM_ERR_INVALID_ARG",
    2: "ATOM_ERR_SHAPE",
    3: "ATOM_ERR_ALIGN",
    4: "ATOM_ERR_UNSUPPORTED",
    5: "ATOM_ERR_CUDA",
    6: "ATOM_ERR_TIMEOUT",
}

N_OUTLIER = 128
GROUP = 128

#: every entry point include/atom.h declares, with its argument types
SIGNATURES = {
    "atom_reorder_quant": ([ct.c_void_p, ct.c_int64, ct.c_int64, ct.c_int64, ct.c_void_p,
                            ct.c_int32, ct.c_int32, ct.c_void_p, ct.c_void_p, ct.c_void_p,
                            ct.c_void_p], ct.c_int),
    "atom_reorder_quant_a8": ([ct.c_void_p, ct.c_int64, ct.c_int64, ct.c_int64, ct.c_void_p,
                               ct.c_int32, ct.c_int32, ct.c_void_p, ct.c_void_p, ct.c_void_p],
                              ct.c_int),
    "atom_w4a8_gemm": ([ct.c_void_p] * 6 + [ct.c_int64, ct.c_int64, ct.c_int64, ct.c_int32,
                                            ct.c_int32, ct.c_void_p], ct.c_int),
    "atom_w4a8_gemm_partials": ([ct.c_void_p] * 7 + [ct.c_int64, ct.c_int64, ct.c_int64,
                                                     ct.c_int32, ct.c_int32, ct.c_void_p],
                                ct.c_int),
    "atom_quant_weights": ([ct.c_void_p, ct.c_int64, ct.c_int64, ct.c_int64, ct.c_void_p,
                            ct.c_int32, ct.c_int32, ct.c_void_p, ct.c_void_p, ct.c_void_p,
                            ct.c_void_p], ct.c_int),
    "atom_w4a4_gemm": ([ct.c_void_p] * 7 + [ct.c_int64, ct.c_int64, ct.c_int64, ct.c_int32,
                                            ct.c_int32, ct.c_void_p, ct.c_size_t, ct.c_void_p],
                       ct.c_int),
    "atom_w4a4_gemm_partials": ([ct.c_void_p] * 8 + [ct.c_int64, ct.c_int64, ct.c_int64,
                                                     ct.c_int32, ct.c_int32, ct.c_void_p],
                                ct.c_int),
    "atom_w4a4_gemm_quant": ([ct.c_void_p] * 6 + [ct.c_int64, ct.c_int64, ct.c_int64, ct.c_int32,
                              ct.c_int32] + [ct.c_void_p] * 4, ct.c_int),
    "atom_gemm_workspace_bytes": ([ct.c_int64, ct.c_int64, ct.c_int64], ct.c_size_t),
    "atom_tiled_weights_bytes": ([ct.c_int64, ct.c_int64], ct.c_size_t),
    "atom_pack_weights_tiled": ([ct.c_void_p, ct.c_int64, ct.c_int64, ct.c_void_p, ct.c_void_p],
                                ct.c_int),
    "atom_unpack_weights_tiled": ([ct.c_void_p, ct.c_int64, ct.c_int64, ct.c_void_p, ct.c_void_p],
                                  ct.c_int),
    "atom_w4a4_gemm_tiled": ([ct.c_void_p] * 7 + [ct.c_int64, ct.c_int64, ct.c_int64, ct.c_int32,
                                                  ct.c_int32, ct.c_void_p, ct.c_size_t,
                                                  ct.c_void_p], ct.c_int),
    "atom_w4a4_gemm_noalloc": ([ct.c_void_p] * 7 + [ct.c_int64, ct.c_int64, ct.c_int64, ct.c_int32,
                                                    ct.c_int32, ct.c_void_p], ct.c_int),
    "atom_w8a8_gemm": ([ct.c_void_p] * 5 + [ct.c_int64, ct.c_int64, ct.c_int64, ct.c_void_p],
                       ct.c_int),
    "atom_kv_quant": ([ct.c_void_p, ct.c_int64, ct.c_void_p, ct.c_void_p, ct.c_void_p], ct.c_int),
    "atom_kv_dequant": ([ct.c_void_p, ct.c_void_p, ct.c_int64, ct.c_void_p, ct.c_void_p],
                        ct.c_int),
    "atom_debug_wait_timeout": ([ct.c_uint64, ct.c_void_p], ct.c_int),
    "atom_probe_mma_i8": ([ct.c_int64, ct.POINTER(ct.c_int32), ct.c_void_p], ct.c_int),
    "atom_device_status": ([ct.c_int], ct.c_int),
    "atom_status_string": ([ct.c_int], ct.c_char_p),
    "atom_version": ([], ct.c_int),
}


class AtomError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


_lib: Optional[ct.CDLL] = None


def lib() -> ct.CDLL:
    """Load libatom_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m w4a4_mixed_precision_b200.build`")
        handle = ct.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            f = getattr(handle, name)
            f.argtypes = args
            f.restype = res
        _lib = handle
    return _lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise AtomError(fn, status)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, dtype: torch.dtype, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


MAX_K = 32768   # the largest K the library accepts (include/atom.h)


def _valid_k(K: int) -> bool:
    return K % GROUP == 0 and 2 * GROUP <= K <= MAX_K


def _expect_shape(t: torch.Tensor, shape, name: str) -> None:
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _check_quantized(q, K: int, name: str, rows: Optional[int] = None) -> None:
    """Shapes of a quantized operand (Quantized) for K. Only checked for a K the
    library accepts: it reports any other K itself, with its own status."""
    if not _valid_k(K):
        return
    rows = q.q4.shape[0] if rows is None else rows
    _expect_shape(q.q4, (rows, (K - N_OUTLIER) // 2), name + ".q4")
    _expect_shape(q.q8, (rows, N_OUTLIER), name + ".q8")
    _expect_shape(q.scales, (K // GROUP, rows), name + ".scales")


def _check_quantized_a8(q, K: int, name: str, rows: Optional[int] = None) -> None:
    """Shapes of W4A8 activations (QuantizedA8) for K, as _check_quantized."""
    if not _valid_k(K):
        return
    rows = q.q8.shape[0] if rows is None else rows
    _expect_shape(q.q8, (rows, K), name + ".q8")
    _expect_shape(q.scales, (K // GROUP, rows), name + ".scales")


class Quantized(NamedTuple):
    """One quantized operand: INT4 codes, INT8 outlier codes, group-major scales."""
    q4: torch.Tensor
    q8: torch.Tensor
    scales: torch.Tensor

    @property
    def rows(self) -> int:
        return self.q4.shape[0]


def empty_quantized(rows: int, K: int, device) -> Quantized:
    return Quantized(torch.empty((rows, (K - N_OUTLIER) // 2), dtype=torch.uint8, device=device),
                     torch.empty((rows, N_OUTLIER), dtype=torch.int8, device=device),
                     torch.empty((K // GROUP, rows), dtype=torch.float32, device=device))


def _quant(fn: str, x: torch.Tensor, outlier_idx: torch.Tensor, out: Optional[Quantized], stream):
    if x.dim() != 2:
        raise ValueError("input must be 2-D [rows, K]")
    rows, K = x.shape
    if x.stride(1) != 1:
        raise ValueError("input rows must be contiguous")
    if out is None:
        out = empty_quantized(rows, K, x.device)
    _check_quantized(out, K, "out", rows)
    if not x.is_cuda or x.dtype != torch.float16:
        raise ValueError("input must be a CUDA float16 tensor")
    st = getattr(lib(), fn)(x.data_ptr(), rows, K, x.stride(0),
                            _dev(outlier_idx, torch.int32, "outlier_idx"), outlier_idx.numel(),
                            GROUP, _dev(out.q4, torch.uint8, "q4"), _dev(out.q8, torch.int8, "q8"),
                            _dev(out.scales, torch.float32, "scales"), _stream(stream))
    _check(fn, st)
    return out


def atom_reorder_quant(x: torch.Tensor, outlier_idx: torch.Tensor,
                       out: Optional[Quantized] = None, stream=None) -> Quantized:
    """Fused outlier reorder + INT4/INT8 quantization of fp16 activations [M, K]."""
    return _quant("atom_reorder_quant", x, outlier_idx, out, stream)


class QuantizedA8(NamedTuple):
    """W4A8 activations: INT8 codes [rows, K] in reordered order, scales [K/128, rows]."""
    q8: torch.Tensor
    scales: torch.Tensor

    @property
    def rows(self) -> int:
        return self.q8.shape[0]


def atom_reorder_quant_a8(x: torch.Tensor, outlier_idx: torch.Tensor,
                          out: Optional[QuantizedA8] = None, stream=None) -> QuantizedA8:
    """W4A8 activations: the outlier reorder, then INT8 in every group (see include/atom.h)."""
    if x.dim() != 2 or x.stride(1) != 1 or not x.is_cuda or x.dtype != torch.float16:
        raise ValueError("input must be a 2-D CUDA float16 tensor with contiguous rows")
    rows, K = x.shape
    if out is None:
        out = QuantizedA8(torch.empty((rows, K), dtype=torch.int8, device=x.device),
                          torch.empty((K // GROUP, rows), dtype=torch.float32, device=x.device))
    _check_quantized_a8(out, K, "out", rows)
    st = lib().atom_reorder_quant_a8(x.data_ptr(), rows, K, x.stride(0),
                                     _dev(outlier_idx, torch.int32, "outlier_idx"),
                                     outlier_idx.numel(), GROUP, _dev(out.q8, torch.int8, "q8"),
                                     _dev(out.scales, torch.float32, "scales"), _stream(stream))
    _check("atom_reorder_quant_a8", st)
    return out


def atom_w4a8_gemm(qa: QuantizedA8, qw: Quantized, K: int, y: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """W4A8: Y fp16 [M, N] from INT8 activations and the W4A4 weights (see include/atom.h)."""
    M, N = qa.rows, qw.rows
    _check_quantized_a8(qa, K, "qa")
    _check_quantized(qw, K, "qw")
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=qa.q8.device)
    _expect_shape(y, (M, N), "y")
    st = lib().atom_w4a8_gemm(
        _dev(qa.q8, torch.int8, "qa8"), _dev(qa.scales, torch.float32, "sa"),
        _dev(qw.q4, torch.uint8, "qw4"), _dev(qw.q8, torch.int8, "qw8"),
        _dev(qw.scales, torch.float32, "sw"), _dev(y, torch.float16, "y"),
        M, N, K, N_OUTLIER, GROUP, _stream(stream))
    _check("atom_w4a8_gemm", st)
    return y


def atom_w4a8_gemm_partials(qa: QuantizedA8, qw: Quantized, K: int, stream=None):
    """Debug entry of the W4A8 GEMM: per-group int32 partial sums [G, M, N] and Y."""
    M, N = qa.rows, qw.rows
    dev = qa.q8.device
    _check_quantized_a8(qa, K, "qa")
    _check_quantized(qw, K, "qw")
    partials = torch.empty((K // GROUP, M, N), dtype=torch.int32, device=dev)
    y = torch.empty((M, N), dtype=torch.float16, device=dev)
    st = lib().atom_w4a8_gemm_partials(
        _dev(qa.q8, torch.int8, "qa8"), _dev(qa.scales, torch.float32, "sa"),
        _dev(qw.q4, torch.uint8, "qw4"), _dev(qw.q8, torch.int8, "qw8"),
        _dev(qw.scales, torch.float32, "sw"), _dev(partials, torch.int32, "partials"),
        _dev(y, torch.float16, "y"), M, N, K, N_OUTLIER, GROUP, _stream(stream))
    _check("atom_w4a8_gemm_partials", st)
    return partials, y


def atom_quant_weights(w: torch.Tensor, outlier_idx: torch.Tensor,
                       out: Optional[Quantized] = None, stream=None) -> Quantized:
    """Offline weight quantization of fp16 W [N, K] (same encoding as the activations)."""
    return _quant("atom_quant_weights", w, outlier_idx, out, stream)


def gemm_workspace(M: int, N: int, K: int, device) -> Optional[torch.Tensor]:
    """Scratch for atom_w4a4_gemm on this shape (None when it needs none)."""
    n = atom_gemm_workspace_bytes(M, N, K)
    return torch.empty(n, dtype=torch.uint8, device=device) if n > 0 else None


def atom_w4a4_gemm(qa: Quantized, qw: Quantized, K: int, y: Optional[torch.Tensor] = None,
                   stream=None, workspace: Optional[torch.Tensor] = None,
                   split: bool = True) -> torch.Tensor:
    """Y fp16 [M, N] = sum_g sa*sw*P_g (see include/atom.h).

    `workspace` (uint8 CUDA tensor) is the scratch a split-K launch uses; when it
    is None and `split` is true, one of atom_gemm_workspace_bytes() bytes is
    allocated here. `split=False` runs without a workspace (no K split)."""
    M, N = qa.rows, qw.rows
    dev = qa.q4.device
    _check_quantized(qa, K, "qa")
    _check_quantized(qw, K, "qw")
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
    _expect_shape(y, (M, N), "y")
    if workspace is None and split:
        workspace = gemm_workspace(M, N, K, dev)
    ws_ptr, ws_bytes = (None, 0) if workspace is None or not split else (
        _dev(workspace, torch.uint8, "workspace"), workspace.numel())
    st = lib().atom_w4a4_gemm(
        _dev(qa.q4, torch.uint8, "qa4"), _dev(qa.q8, torch.int8, "qa8"),
        _dev(qa.scales, torch.float32, "sa"), _dev(qw.q4, torch.uint8, "qw4"),
        _dev(qw.q8, torch.int8, "qw8"), _dev(qw.scales, torch.float32, "sw"),
        _dev(y, torch.float16, "y"), M, N, K, N_OUTLIER, GROUP, ws_ptr, ws_bytes, _stream(stream))
    _check("atom_w4a4_gemm", st)
    return y


class TiledWeights(NamedTuple):
    """Quantized weights with the INT4 codes in the tiled layout (see
    include/atom.h): q4t uint8 [ceil(N/128), K/128 - 1, 128, 64]; q8 and scales as
    in Quantized."""
    q4t: torch.Tensor
    q8: torch.Tensor
    scales: torch.Tensor

    @property
    def rows(self) -> int:
        return self.q8.shape[0]


def _tiled_shape(N: int, K: int):
    return ((N + 127) // 128, K // GROUP - 1, 128, 64)


def atom_pack_weights_tiled(qw: Quantized, K: int, stream=None) -> TiledWeights:
    """One-off repack of quantized weights into the tiled layout."""
    N = qw.rows
    _check_quantized(qw, K, "qw")
    q4t = torch.empty(_tiled_shape(N, K), dtype=torch.uint8, device=qw.q4.device)
    st = lib().atom_pack_weights_tiled(_dev(qw.q4, torch.uint8, "qw4"), N, K,
                                       _dev(q4t, torch.uint8, "qw4t"), _stream(stream))
    _check("atom_pack_weights_tiled", st)
    return TiledWeights(q4t, qw.q8, qw.scales)


def atom_unpack_weights_tiled(qwt: TiledWeights, K: int, stream=None) -> torch.Tensor:
    """The row layout [N, (K-128)/2] of tiled INT4 weight codes (the inverse repack)."""
    N = qwt.rows
    if _valid_k(K):
        _expect_shape(qwt.q4t, _tiled_shape(N, K), "qw4t")
    q4 = torch.empty((N, (K - N_OUTLIER) // 2), dtype=torch.uint8, device=qwt.q4t.device)
    st = lib().atom_unpack_weights_tiled(_dev(qwt.q4t, torch.uint8, "qw4t"), N, K,
                                         _dev(q4, torch.uint8, "qw4"), _stream(stream))
    _check("atom_unpack_weights_tiled", st)
    return q4


def atom_w4a4_gemm_tiled(qa: Quantized, qwt: TiledWeights, K: int,
                         y: Optional[torch.Tensor] = None, stream=None,
                         workspace: Optional[torch.Tensor] = None,
                         split: bool = True) -> torch.Tensor:
    """atom_w4a4_gemm with the weights in the tiled layout (bit-identical Y)."""
    M, N = qa.rows, qwt.rows
    dev = qa.q4.device
    _check_quantized(qa, K, "qa")
    if _valid_k(K):
        _expect_shape(qwt.q4t, _tiled_shape(N, K), "qw4t")
        _expect_shape(qwt.q8, (N, N_OUTLIER), "qw.q8")
        _expect_shape(qwt.scales, (K // GROUP, N), "qw.scales")
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
    _expect_shape(y, (M, N), "y")
    if workspace is None and split:
        workspace = gemm_workspace(M, N, K, dev)
    ws_ptr, ws_bytes = (None, 0) if workspace is None or not split else (
        _dev(workspace, torch.uint8, "workspace"), workspace.numel())
    st = lib().atom_w4a4_gemm_tiled(
        _dev(qa.q4, torch.uint8, "qa4"), _dev(qa.q8, torch.int8, "qa8"),
        _dev(qa.scales, torch.float32, "sa"), _dev(qwt.q4t, torch.uint8, "qw4t"),
        _dev(qwt.q8, torch.int8, "qw8"), _dev(qwt.scales, torch.float32, "sw"),
        _dev(y, torch.float16, "y"), M, N, K, N_OUTLIER, GROUP, ws_ptr, ws_bytes, _stream(stream))
    _check("atom_w4a4_gemm_tiled", st)
    return y


def atom_tiled_weights_bytes(N: int, K: int) -> int:
    return int(lib().atom_tiled_weights_bytes(N, K))


def atom_w4a4_gemm_noalloc(qa: Quantized, qw: Quantized, K: int,
                           y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """atom_w4a4_gemm for callers that cannot allocate device memory around the
    call (a runtime whose device memory all sits in a fixed pool, a C caller
    without an allocator): a split of K keeps its partials in the library's
    fixed 8 MiB device array (see include/atom.h). Pass `y` to keep this wrapper
    allocation-free as well."""
    M, N = qa.rows, qw.rows
    _check_quantized(qa, K, "qa")
    _check_quantized(qw, K, "qw")
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=qa.q4.device)
    _expect_shape(y, (M, N), "y")
    st = lib().atom_w4a4_gemm_noalloc(
        _dev(qa.q4, torch.uint8, "qa4"), _dev(qa.q8, torch.int8, "qa8"),
        _dev(qa.scales, torch.float32, "sa"), _dev(qw.q4, torch.uint8, "qw4"),
        _dev(qw.q8, torch.int8, "qw8"), _dev(qw.scales, torch.float32, "sw"),
        _dev(y, torch.float16, "y"), M, N, K, N_OUTLIER, GROUP, _stream(stream))
    _check("atom_w4a4_gemm_noalloc", st)
    return y


def atom_w4a4_gemm_partials(qa: Quantized, qw: Quantized, K: int,
                            partials: Optional[torch.Tensor] = None,
                            y: Optional[torch.Tensor] = None, want_y: bool = True,
                            stream=None):
    """Debug entry: per-group int32 partial sums [G, M, N] (and Y unless want_y is False)."""
    M, N = qa.rows, qw.rows
    dev = qa.q4.device
    _check_quantized(qa, K, "qa")
    _check_quantized(qw, K, "qw")
    if partials is None:
        partials = torch.empty((K // GROUP, M, N), dtype=torch.int32, device=dev)
    if _valid_k(K):
        _expect_shape(partials, (K // GROUP, M, N), "partials")
    if want_y and y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
    if want_y:
        _expect_shape(y, (M, N), "y")
    st = lib().atom_w4a4_gemm_partials(
        _dev(qa.q4, torch.uint8, "qa4"), _dev(qa.q8, torch.int8, "qa8"),
        _dev(qa.scales, torch.float32, "sa"), _dev(qw.q4, torch.uint8, "qw4"),
        _dev(qw.q8, torch.int8, "qw8"), _dev(qw.scales, torch.float32, "sw"),
        _dev(partials, torch.int32, "partials"),
        _dev(y, torch.float16, "y") if want_y else None,
        M, N, K, N_OUTLIER, GROUP, _stream(stream))
    _check("atom_w4a4_gemm_partials", st)
    return partials, y


def atom_w4a4_gemm_quant(qa: Quantized, qw: Quantized, K: int, out: Optional[Quantized] = None,
                         stream=None) -> Quantized:
    """The GEMM with the next layer's activation quantization in its epilogue: the codes
    and scales atom_reorder_quant would write for Y (unsplit, fp16) with Y's last 128
    columns as the outlier channels (see include/atom.h). N must be a multiple of 128."""
    M, N = qa.rows, qw.rows
    _check_quantized(qa, K, "qa")
    _check_quantized(qw, K, "qw")
    if out is None:
        out = empty_quantized(M, N, qa.q4.device)
    _check_quantized(out, N, "out", M)   # Y's N is the next layer's K
    st = lib().atom_w4a4_gemm_quant(
        _dev(qa.q4, torch.uint8, "qa4"), _dev(qa.q8, torch.int8, "qa8"),
        _dev(qa.scales, torch.float32, "sa"), _dev(qw.q4, torch.uint8, "qw4"),
        _dev(qw.q8, torch.int8, "qw8"), _dev(qw.scales, torch.float32, "sw"),
        M, N, K, N_OUTLIER, GROUP,
        _dev(out.q4, torch.uint8, "qy4"), _dev(out.q8, torch.int8, "qy8"),
        _dev(out.scales, torch.float32, "sy"), _stream(stream))
    _check("atom_w4a4_gemm_quant", st)
    return out


def atom_w8a8_gemm(qa: torch.Tensor, sa: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor,
                   y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """W8A8 comparator: y = fp16(float(qa @ qw^T) * sa[:, None] * sw[None, :]) with int8
    qa [M, K], qw [N, K] and fp32 scales sa [M], sw [N] (see include/atom.h)."""
    M, K = qa.shape
    N = qw.shape[0]
    if qw.shape[1] != K or sa.shape != (M,) or sw.shape != (N,):
        raise ValueError("atom_w8a8_gemm: shapes must be qa [M, K], qw [N, K], sa [M], sw [N]")
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=qa.device)
    st = lib().atom_w8a8_gemm(
        _dev(qa, torch.int8, "qa"), _dev(sa, torch.float32, "sa"), _dev(qw, torch.int8, "qw"),
        _dev(sw, torch.float32, "sw"), _dev(y, torch.float16, "y"), M, N, K, _stream(stream))
    _check("atom_w8a8_gemm", st)
    return y


def atom_kv_quant(x: torch.Tensor, q4: Optional[torch.Tensor] = None,
                  scales: Optional[torch.Tensor] = None, stream=None):
    """INT4 KV-cache quantization of fp16 [..., 128] (one group per 128-vector):
    returns (q4 uint8 [..., 64], scales fp32 [...]) (see include/atom.h)."""
    if x.shape[-1] != 128:
        raise ValueError("atom_kv_quant: the last axis must be head_dim = 128")
    lead = tuple(x.shape[:-1])
    groups = x.numel() // 128
    if q4 is None:
        q4 = torch.empty(lead + (64,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(lead, dtype=torch.float32, device=x.device)
    st = lib().atom_kv_quant(_dev(x, torch.float16, "x"), groups, _dev(q4, torch.uint8, "q4"),
                             _dev(scales, torch.float32, "scales"), _stream(stream))
    _check("atom_kv_quant", st)
    return q4, scales


def atom_kv_dequant(q4: torch.Tensor, scales: torch.Tensor, out: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """fp16 [..., 128] from atom_kv_quant's codes and scales."""
    if q4.shape[-1] != 64 or tuple(scales.shape) != tuple(q4.shape[:-1]):
        raise ValueError("atom_kv_dequant: q4 [..., 64] and scales [...] must match")
    groups = scales.numel()
    if out is None:
        out = torch.empty(tuple(q4.shape[:-1]) + (128,), dtype=torch.float16, device=q4.device)
    st = lib().atom_kv_dequant(_dev(q4, torch.uint8, "q4"), _dev(scales, torch.float32, "scales"),
                               groups, _dev(out, torch.float16, "out"), _stream(stream))
    _check("atom_kv_dequant", st)
    return out


def atom_gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().atom_gemm_workspace_bytes(M, N, K))


def atom_probe_mma_i8(groups: int, stream=None) -> int:
    """Measurement aid: launches the INT8 tensor-core peak loop (see
    include/atom.h) and returns the integer operations it performs."""
    pairs = ct.c_int32(0)
    _check("atom_probe_mma_i8", lib().atom_probe_mma_i8(groups, ct.byref(pairs), _stream(stream)))
    return 2 * 256 * 256 * 128 * groups * pairs.value


def atom_debug_wait_timeout(limit_ns: int, stream=None) -> None:
    """Test aid: runs the library's bounded mbarrier wait on a barrier nothing
    arrives on, with a limit of `limit_ns`; the wait gives up and the device
    status becomes ATOM_ERR_TIMEOUT (see include/atom.h)."""
    _check("atom_debug_wait_timeout", lib().atom_debug_wait_timeout(limit_ns, _stream(stream)))


def atom_device_status(clear: bool = True) -> int:
    """First device-detected error since the last clear (0 = none); synchronises."""
    return int(lib().atom_device_status(1 if clear else 0))


def atom_status_string(status: int) -> str:
    return lib().atom_status_string(status).decode()


def atom_version() -> int:
    return int(lib().atom_version())
