"""Parity of the W4A8 variant with its oracle (oracle/w4a8_oracle.py).

Activation codes and scales bit-exact on every row of the five workloads'
activations and on ragged shapes; per-group int32 partial sums bit-exact and Y
within gpu_util.y_rel_err's tolerance on small and ragged shapes; Y on sampled
rows of two full-size workloads."""
import numpy as np
import pytest
import torch

from oracle import numpy_oracle, w4a8_oracle
from w4a4_mixed_precision_b200 import atom, inputs

from gpu_util import Y_TOL, fp16_dev, idx_dev, quant_dev, y_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _clear_status():
    atom.atom_device_status(clear=True)
    yield
    assert atom.atom_device_status(clear=True) == 0


def _a8_dev(A, idx):
    return atom.atom_reorder_quant_a8(fp16_dev(A), idx_dev(idx))


def _assert_a8_equal(got: atom.QuantizedA8, A, idx, what):
    torch.cuda.synchronize()
    q, s = w4a8_oracle.quantize_a8(A, idx)
    gq, gs = got.q8.cpu().numpy(), got.scales.cpu().numpy()
    bad = np.argwhere(gq != q)
    assert bad.size == 0, f"{what}: {len(bad)} code mismatches, first {bad[:3].tolist()}"
    assert np.array_equal(gs.view(np.uint32), s.view(np.uint32)), f"{what}: scales differ"


@pytest.mark.parametrize("c", [0, 1, 2, 3, 4])
def test_activation_codes_bit_exact_all_rows(c):
    A, idx = inputs.activations(c), inputs.outlier_channels(c)
    _assert_a8_equal(_a8_dev(A, idx), A, idx, f"workload {c}")


@pytest.mark.parametrize("M,K,seed", [(1, 256, 1), (333, 1152, 2), (64, 32768, 3), (1000, 24576, 4)])
def test_ragged_sizes_unsorted_outliers(M, K, seed):
    A, _, idx = inputs.random_case(seed, M, 8, K, dist="t", param=3.0, outlier_factor=50.0,
                                   sorted_outliers=False)
    _assert_a8_equal(_a8_dev(A, idx), A, idx, f"{M}x{K}")


@pytest.mark.parametrize("M,N,K,seed", [(16, 256, 512, 11), (300, 520, 1152, 12), (1, 8, 256, 13),
                                        (130, 256, 4096, 14), (257, 264, 640, 15)])
def test_partials_bit_exact_and_output_within_tolerance(M, N, K, seed):
    A, W, idx = inputs.random_case(seed, M, N, K, dist="t", param=4.0, outlier_factor=30.0)
    qa, qw = _a8_dev(A, idx), quant_dev(W, idx, weights=True)
    P, y = atom.atom_w4a8_gemm_partials(qa, qw, K)
    y2 = atom.atom_w4a8_gemm(qa, qw, K)
    torch.cuda.synchronize()
    q, sa = w4a8_oracle.quantize_a8(A, idx)
    qw4, qw8, sw = numpy_oracle.quantize(W, idx)
    P_ref = w4a8_oracle.partials(q, qw4, qw8)
    Pg = P.cpu().numpy()
    bad = np.argwhere(Pg != P_ref)
    assert bad.size == 0, f"{len(bad)} partial mismatches, first {bad[:3].tolist()}"
    Y64 = w4a8_oracle.output64(P_ref, sa, sw)
    for got in (y, y2):
        assert y_rel_err(got.cpu().numpy(), Y64) <= Y_TOL
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("c", [1, 2])
def test_full_workload_sampled_rows(c):
    w = inputs.workload(c)
    A, W, idx = inputs.activations(c), inputs.weights(c), inputs.outlier_channels(c)
    y = atom.atom_w4a8_gemm(_a8_dev(A, idx), quant_dev(W, idx, weights=True), w.K)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.random.default_rng(7 + c).choice(w.M, 15, replace=False),
                                     [w.M - 1]]))
    q, sa = w4a8_oracle.quantize_a8(A[rows], idx)
    qw4, qw8, sw = numpy_oracle.quantize(W, idx)
    Y64 = w4a8_oracle.output64(w4a8_oracle.partials(q, qw4, qw8), sa, sw)
    assert y_rel_err(y.cpu().numpy()[rows], Y64) <= Y_TOL


def test_bad_outlier_list_is_rejected_on_the_device():
    K = 512
    A = np.ones((4, K), dtype=np.float16)
    idx = np.arange(128, dtype=np.int32)
    idx[5] = idx[4]                           # a repeated channel
    out = atom.QuantizedA8(torch.full((4, K), 7, dtype=torch.int8, device="cuda"),
                           torch.zeros((K // 128, 4), dtype=torch.float32, device="cuda"))
    atom.atom_reorder_quant_a8(fp16_dev(A), idx_dev(idx), out=out)
    assert atom.atom_device_status(clear=True) == 1   # ATOM_ERR_INVALID_ARG
    assert (out.q8 == 7).all()                 # nothing written
