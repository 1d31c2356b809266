"""The tiled weight layout (atom_pack_weights_tiled, atom_unpack_weights_tiled,
atom_w4a4_gemm_tiled).

The layout is pure data movement, so its check is bit for bit: the tiled bytes
must equal a numpy rearrangement of the CPU oracle's packed weight codes, and
the round trip must give the codes back. The GEMM on tiled weights runs the
same kernels in the same order as on the row layout, so its Y must be
bit-identical to atom_w4a4_gemm's (whose parity with the oracle is checked in
test_gemm_gpu.py), and within tolerance of the oracle's fp64 output."""
import numpy as np
import pytest
import torch

from w4a4_mixed_precision_b200 import atom, inputs

from gpu_util import Y_TOL, fp16_dev, idx_dev, quant_dev, y_rel_err

pytestmark = pytest.mark.gpu


def _tiled_reference(q4: np.ndarray, K: int) -> np.ndarray:
    """The tiled layout written out from its definition: block (t, g) holds rows
    128t..128t+127 (zero past N) of bytes 64g..64g+63 of the row layout."""
    N = q4.shape[0]
    T, G4 = (N + 127) // 128, K // 128 - 1
    padded = np.zeros((T * 128, q4.shape[1]), dtype=np.uint8)
    padded[:N] = q4
    out = np.zeros((T, G4, 128, 64), dtype=np.uint8)
    for t in range(T):
        for g in range(G4):
            out[t, g] = padded[128 * t:128 * t + 128, 64 * g:64 * g + 64]
    return out


@pytest.mark.parametrize("N,K,seed", [(256, 512, 71), (264, 1152, 72), (1000, 4096, 73),
                                      (8, 256, 74), (4096, 11008, 75)])
def test_pack_matches_layout_definition_and_round_trips(c_oracle, N, K, seed):
    _, W, idx = inputs.random_case(seed, 1, N, K)
    q4_ref = c_oracle.quantize(W, idx)[0]
    qw = atom.atom_quant_weights(fp16_dev(W), idx_dev(idx))
    qwt = atom.atom_pack_weights_tiled(qw, K)
    assert qwt.q4t.numel() == atom.atom_tiled_weights_bytes(N, K)
    assert np.array_equal(qwt.q4t.cpu().numpy(), _tiled_reference(q4_ref, K))
    back = atom.atom_unpack_weights_tiled(qwt, K)
    torch.cuda.synchronize()
    assert np.array_equal(back.cpu().numpy(), q4_ref)


# M <= 64: the small-M kernel (with and without its K split); M > 64: the large
# kernel, including N = 264, where the second 256-column pair tile's upper 128
# weight rows lie wholly past N (no tiled block exists for them).
@pytest.mark.parametrize("M,N,K,seed", [(1, 4096, 4096, 81), (16, 264, 1152, 82),
                                        (64, 4096, 4096, 83), (40, 520, 32768, 84),
                                        (300, 520, 1152, 85), (257, 264, 640, 86),
                                        (130, 1024, 4096, 87), (512, 2048, 2048, 88)])
def test_tiled_gemm_is_bit_identical_to_row_layout(c_oracle, M, N, K, seed):
    A, W, idx = inputs.random_case(seed, M, N, K, dist="t", param=3.0, outlier_factor=50.0)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    qwt = atom.atom_pack_weights_tiled(qw, K)
    for split in (True, False):
        y_row = atom.atom_w4a4_gemm(qa, qw, K, split=split)
        y_til = atom.atom_w4a4_gemm_tiled(qa, qwt, K, split=split)
        torch.cuda.synchronize()
        assert torch.equal(y_row.view(torch.int16), y_til.view(torch.int16)), split
    ra, rw = c_oracle.quantize(A, idx), c_oracle.quantize(W, idx)
    assert y_rel_err(y_til.cpu().numpy(), c_oracle.gemm(*ra, *rw, K)) <= Y_TOL
    assert atom.atom_device_status(clear=True) == 0


@pytest.mark.parametrize("c", [1, 2])
def test_tiled_gemm_full_size_workload(c_oracle, c):
    """The decode and prefill workloads on tiled weights: Y bit-identical to the
    row layout, and every row within tolerance of the oracle."""
    w = inputs.workload(c)
    A, W, idx = inputs.activations(c), inputs.weights(c), inputs.outlier_channels(c)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    qwt = atom.atom_pack_weights_tiled(qw, w.K)
    y_row = atom.atom_w4a4_gemm(qa, qw, w.K)
    y_til = atom.atom_w4a4_gemm_tiled(qa, qwt, w.K)
    torch.cuda.synchronize()
    assert torch.equal(y_row.view(torch.int16), y_til.view(torch.int16))
    if c == 1:
        ra, rw = c_oracle.quantize(A, idx), c_oracle.quantize(W, idx)
        assert y_rel_err(y_til.cpu().numpy(), c_oracle.gemm(*ra, *rw, w.K)) <= Y_TOL
