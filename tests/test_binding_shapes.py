"""The Python binding checks tensor shapes before it hands pointers to the library
(no GPU needed). With CPU tensors, correct shapes get past every shape check and
stop at the first "must be a CUDA tensor" check; wrong shapes stop earlier with a
shape error. Shapes the library itself rejects (K or N not whole groups) are left
to the library, so that its own status reaches the caller."""
import pytest
import torch

from w4a4_mixed_precision_b200 import atom

M, N, K = 4, 256, 512
CPU = torch.device("cpu")


def q(rows, k):
    return atom.empty_quantized(rows, k, CPU)


def a8(rows, k):
    return atom.QuantizedA8(torch.empty((rows, k), dtype=torch.int8),
                            torch.empty((k // 128, rows), dtype=torch.float32))


def passes_shape_checks(fn, *args, **kw):
    with pytest.raises(ValueError) as e:
        fn(*args, **kw)
    assert "CUDA" in str(e.value) and "shape" not in str(e.value), str(e.value)


def fails_shape_check(fn, *args, **kw):
    with pytest.raises(ValueError) as e:
        fn(*args, **kw)
    assert "must have shape" in str(e.value), str(e.value)


def test_quantizer_output():
    x = torch.zeros((M, K), dtype=torch.float16)
    idx = torch.arange(128, dtype=torch.int32)
    passes_shape_checks(atom.atom_reorder_quant, x, idx, out=q(M, K))
    fails_shape_check(atom.atom_reorder_quant, x, idx, out=q(M + 1, K))
    fails_shape_check(atom.atom_reorder_quant, x, idx, out=q(M, K + 128))


def test_gemm_operands_and_output():
    passes_shape_checks(atom.atom_w4a4_gemm, q(M, K), q(N, K), K, split=False)
    passes_shape_checks(atom.atom_w4a4_gemm, q(0, K), q(N, K), K, split=False)    # empty M
    fails_shape_check(atom.atom_w4a4_gemm, q(M, K), q(N, K + 128), K, split=False)
    fails_shape_check(atom.atom_w4a4_gemm, q(M, K), q(N, K), K, split=False,
                      y=torch.empty((M, N - 8), dtype=torch.float16))
    passes_shape_checks(atom.atom_w4a4_gemm_noalloc, q(M, K), q(N, K), K)
    fails_shape_check(atom.atom_w4a4_gemm_noalloc, q(M + 1, K - 128), q(N, K), K)


def test_partials_windows_and_buffers():
    passes_shape_checks(atom.atom_w4a4_gemm_partials, q(M, K), q(N, K), K)
    passes_shape_checks(atom.atom_w4a4_gemm_partials, q(M, K), q(N, K), K, want_y=False)
    fails_shape_check(atom.atom_w4a4_gemm_partials, q(M, K), q(N, K), K,
                      partials=torch.empty((K // 128, N, M), dtype=torch.int32))


def test_quantizing_gemm_output():
    passes_shape_checks(atom.atom_w4a4_gemm_quant, q(M, K), q(N, K), K)
    passes_shape_checks(atom.atom_w4a4_gemm_quant, q(M, K), q(N, K), K, out=q(M, N))
    fails_shape_check(atom.atom_w4a4_gemm_quant, q(M, K), q(N, K), K, out=q(M, N + 128))
    # an N the library rejects goes to the library (its ATOM_ERR_SHAPE), not to a shape error
    for bad_n in (128, 200, 392):
        passes_shape_checks(atom.atom_w4a4_gemm_quant, q(M, K), q(bad_n, K), K, out=q(M, 512))


def test_w4a8_operands():
    passes_shape_checks(atom.atom_w4a8_gemm, a8(M, K), q(N, K), K)
    passes_shape_checks(atom.atom_w4a8_gemm_partials, a8(M, K), q(N, K), K)
    fails_shape_check(atom.atom_w4a8_gemm, a8(M, K + 128), q(N, K), K)
    fails_shape_check(atom.atom_w4a8_gemm, a8(M, K), q(N, K), K,
                      y=torch.empty((M + 1, N), dtype=torch.float16))
