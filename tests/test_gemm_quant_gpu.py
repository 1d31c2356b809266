"""Parity of atom_w4a4_gemm_quant: the W4A4 GEMM with the next layer's activation
quantization in its epilogue (Y's last 128 columns as the outlier channels).

Two checks per shape:
  * against the oracle: the oracle's dequantization of the codes lies within half
    a quantization step of the oracle's fp64 Y, plus the GEMM's output tolerance
    (gpu_util.y_rel_err); each group's scale times qmax is the group's max |Y|
    within the same tolerance;
  * bit for bit against the unfused path on the GPU: atom_reorder_quant applied to
    the unsplit fp16 output of atom_w4a4_gemm, with the outlier list
    N-128 .. N-1 (the same fp32 steps, so the codes and scales must be equal).
"""
import numpy as np
import pytest
import torch

from w4a4_mixed_precision_b200 import atom, inputs

from gpu_util import Y_TOL, assert_codes_equal, host, quant_dev

pytestmark = pytest.mark.gpu

SHAPES = [(300, 384, 1152, 61),   # ragged M; second tile half outside N
          (70, 256, 512, 62),     # one INT4 group of Y and the INT8 group
          (1, 1024, 2048, 63),    # one token
          (257, 2560, 4096, 64)]  # several tiles each way


@pytest.fixture(scope="module", autouse=True)
def _clear_status():
    atom.atom_device_status(clear=True)
    yield
    assert atom.atom_device_status(clear=True) == 0


def _case(seed, M, N, K, zero_rows=()):
    A, W, idx = inputs.random_case(seed, M, N, K, dist="t", param=4.0, outlier_factor=30.0)
    for r in zero_rows:
        A[r] = 0
    return A, W, idx


@pytest.mark.parametrize("M,N,K,seed", SHAPES)
def test_codes_reproduce_the_oracle_output_within_half_a_step(c_oracle, M, N, K, seed):
    A, W, idx = _case(seed, M, N, K)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    q4, q8, sy = host(atom.atom_w4a4_gemm_quant(qa, qw, K))
    ra, rw = c_oracle.quantize(A, idx), c_oracle.quantize(W, idx)
    Y64 = c_oracle.gemm(*ra, *rw, K)
    dq = c_oracle.dequantize(q4, q8, sy, N)      # identity reorder: column n of Y
    rms = float(np.sqrt(np.mean(Y64 * Y64)))
    tol = Y_TOL * np.maximum(np.abs(Y64), 1e-2 * rms)
    G = N // 128
    step = np.repeat(sy.T.astype(np.float64), 128, axis=1)
    err = np.abs(dq - Y64) - (0.5 * step * (1 + 1e-5) + tol)
    assert err.max() <= 0, f"worst excess {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}"
    qmax = np.array([7.0] * (G - 1) + [127.0])
    amax64 = np.abs(Y64).reshape(M, G, 128).max(axis=2)
    tolg = tol.reshape(M, G, 128).max(axis=2)
    gap = np.abs(sy.T.astype(np.float64) * qmax - amax64) - (tolg + 1e-6 * amax64)
    assert gap.max() <= 0, f"scale off by {gap.max():.3e}"


@pytest.mark.parametrize("M,N,K,seed", SHAPES)
def test_equals_quantizing_the_unsplit_output(M, N, K, seed):
    A, W, idx = _case(seed, M, N, K)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    fused = atom.atom_w4a4_gemm_quant(qa, qw, K)
    y = atom.atom_w4a4_gemm(qa, qw, K, split=False)
    tail = torch.arange(N - 128, N, dtype=torch.int32, device="cuda")
    assert_codes_equal(host(fused), host(atom.atom_reorder_quant(y, tail)), f"{M}x{N}x{K}")


def test_zero_rows_give_zero_codes_and_scales():
    M, N, K = 130, 512, 512
    A, W, idx = _case(65, M, N, K, zero_rows=(0, 77, 129))
    q4, q8, sy = host(atom.atom_w4a4_gemm_quant(quant_dev(A, idx), quant_dev(W, idx, weights=True), K))
    for r in (0, 77, 129):
        assert not q4[r].any() and not q8[r].any() and not sy[:, r].any()
    assert sy[:, 1].all()


def test_runs_again_into_the_same_buffers():
    M, N, K = 96, 768, 1024
    A, W, idx = _case(66, M, N, K)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    out = atom.empty_quantized(M, N, torch.device("cuda"))
    first = [a.copy() for a in host(atom.atom_w4a4_gemm_quant(qa, qw, K, out=out))]
    out.q4.fill_(0x5A)
    out.q8.fill_(-3)
    out.scales.fill_(float("nan"))
    assert_codes_equal(host(atom.atom_w4a4_gemm_quant(qa, qw, K, out=out)), first, "rerun")


@pytest.mark.parametrize("N", [128, 200, 384 + 8])
def test_rejects_an_n_that_is_not_whole_groups(N):
    M, K = 64, 512
    A, W, idx = _case(67, M, max(N, 8) // 8 * 8, K)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    with pytest.raises(atom.AtomError) as e:
        atom.atom_w4a4_gemm_quant(qa, qw, K, out=atom.empty_quantized(M, 512, torch.device("cuda")))
    assert e.value.status == 2   # ATOM_ERR_SHAPE
