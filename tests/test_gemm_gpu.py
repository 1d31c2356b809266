"""Parity of the tcgen05 W4A4 GEMM with the CPU oracle.

Per-group int32 partial sums must be bit-identical (debug entry point, full
tensor on small shapes and on the decode workload, 256x256 windows of the large
workloads; M <= 64 goes through the small-M kernel, as in production); the
fp16 output must be within the tolerance of gpu_util.y_rel_err of the oracle's
fp64 output, on every row of small shapes and of workloads 1 and 2, and on 512
seeded rows of workloads 3 and 4 (run exactly as the benchmark launches them)."""
import numpy as np
import pytest
import torch

from w4a4_mixed_precision_b200 import atom, inputs

from gpu_util import (Y_TOL, fp16_dev, host, idx_dev, quant_dev, rows_of, y_rel_err)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _clear_status():
    atom.atom_device_status(clear=True)
    yield
    assert atom.atom_device_status(clear=True) == 0


def _oracle_all(c_oracle, A, W, idx):
    K = A.shape[1]
    qa, qw = c_oracle.quantize(A, idx), c_oracle.quantize(W, idx)
    P = c_oracle.partials(qa[0], qa[1], qw[0], qw[1], K)
    Y64 = c_oracle.gemm(*qa, *qw, K)
    return P, Y64


def _gpu_partials(A, W, idx):
    K = A.shape[1]
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    P, y = atom.atom_w4a4_gemm_partials(qa, qw, K)
    y2 = atom.atom_w4a4_gemm(qa, qw, K)
    torch.cuda.synchronize()
    return P.cpu().numpy(), y.cpu().numpy(), y2.cpu().numpy()


def _case(name):
    if name == "tiny":
        return inputs.activations(0), inputs.weights(0), inputs.outlier_channels(0)
    shapes = {"ragged": (300, 520, 1152, 5), "one_row": (1, 8, 256, 6),
              "two_tiles_m": (257, 264, 640, 7), "many_groups": (130, 256, 4096, 9),
              "wide_k": (40, 72, 32768, 10)}
    M, N, K, seed = shapes[name]
    return inputs.random_case(seed, M, N, K, dist="t", param=3.0, outlier_factor=50.0,
                              sorted_outliers=(seed % 2 == 0))


@pytest.mark.parametrize("name", ["tiny", "ragged", "one_row", "two_tiles_m", "many_groups",
                                  "wide_k"])
def test_partials_bit_exact_and_output_within_tolerance(c_oracle, name):
    A, W, idx = _case(name)
    P_ref, Y64 = _oracle_all(c_oracle, A, W, idx)
    P, y, y2 = _gpu_partials(A, W, idx)
    assert P.shape == P_ref.shape
    mism = np.argwhere(P != P_ref)
    assert mism.size == 0, f"{len(mism)} partial mismatches, first {mism[:3].tolist()}"
    assert y_rel_err(y, Y64) <= Y_TOL
    assert y_rel_err(y2, Y64) <= Y_TOL
    if atom.atom_gemm_workspace_bytes(A.shape[0], W.shape[0], A.shape[1]) == 0:
        # no K split: the same mainloop in the same order gives the same Y
        assert np.array_equal(y.view(np.uint16), y2.view(np.uint16))


def test_lossless_integers_give_the_exact_integer_matmul(c_oracle):
    """Integer inputs whose groups have amax exactly 7 / 127 quantize with scale 1;
    with small products the fp16 output is then the textbook integer matmul."""
    rng = np.random.default_rng(42)
    M, N, K = 70, 48, 512
    idx = np.sort(rng.choice(K, 128, replace=False)).astype(np.int32)
    perm = c_oracle.permutation(K, idx)

    def make(rows, lim4, lim8, hot, cold):
        # every group holds its qmax at position `hot` and a zero at `cold`, so the
        # A and W anchors never meet and all products stay small
        xr = np.zeros((rows, K))
        xr[:, :K - 128] = rng.integers(-lim4, lim4 + 1, (rows, K - 128))
        xr[:, K - 128:] = rng.integers(-lim8, lim8 + 1, (rows, 128))
        for g in range(K // 128):
            xr[:, g * 128 + hot] = 7 if g < K // 128 - 1 else 127
            xr[:, g * 128 + cold] = 0
        x = np.zeros_like(xr)
        x[:, perm] = xr
        return x.astype(np.float16), xr

    A, Ar = make(M, 2, 3, hot=0, cold=1)
    W, Wr = make(N, 1, 1, hot=1, cold=0)
    ref = Ar.astype(np.int64) @ Wr.astype(np.int64).T
    assert np.abs(ref).max() <= 2048                      # exactly representable in fp16
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    y = atom.atom_w4a4_gemm(qa, qw, K).cpu().numpy().astype(np.float64)
    assert np.array_equal(y, ref.astype(np.float64))


@pytest.mark.parametrize("M,N,K,seed", [(1, 264, 1024, 51), (16, 4096, 4096, 52),
                                        (40, 520, 2048, 53), (64, 392, 32768, 54),
                                        (33, 128, 256, 55)])
def test_small_m_kernel_partials_bit_exact(c_oracle, M, N, K, seed):
    """M <= 64 runs the small-M kernel (weights on the MMA's M side) for the
    partials entry point as for atom_w4a4_gemm: its per-group int32 partials
    must equal the oracle's, and its unsplit Y must equal atom_w4a4_gemm's
    unsplit Y bit for bit (same kernel, same order)."""
    A, W, idx = inputs.random_case(seed, M, N, K, dist="t", param=3.0, outlier_factor=50.0,
                                   sorted_outliers=(seed % 2 == 0))
    P_ref, Y64 = _oracle_all(c_oracle, A, W, idx)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    P, y = atom.atom_w4a4_gemm_partials(qa, qw, K)
    y_plain = atom.atom_w4a4_gemm(qa, qw, K, split=False)
    torch.cuda.synchronize()
    P = P.cpu().numpy()
    mism = np.argwhere(P != P_ref)
    assert mism.size == 0, f"{len(mism)} partial mismatches, first {mism[:3].tolist()}"
    y = y.cpu().numpy()
    assert y_rel_err(y, Y64) <= Y_TOL
    assert np.array_equal(y.view(np.uint16), y_plain.cpu().numpy().view(np.uint16))


def test_decode_workload_partials_bit_exact_in_full(c_oracle):
    """Every per-group partial of the full 64 x 4096 x 4096 decode workload,
    computed by the small-M kernel, equals the oracle's."""
    c = 1
    w = inputs.workload(c)
    A, W, idx = inputs.activations(c), inputs.weights(c), inputs.outlier_channels(c)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    P, _ = atom.atom_w4a4_gemm_partials(qa, qw, w.K, want_y=False)
    P = P.cpu().numpy()
    ra, rw = c_oracle.quantize(A, idx), c_oracle.quantize(W, idx)
    P_ref = c_oracle.partials(ra[0], ra[1], rw[0], rw[1], w.K)
    mism = np.argwhere(P != P_ref)
    assert mism.size == 0, f"{len(mism)} partial mismatches, first {mism[:3].tolist()}"


@pytest.mark.parametrize("c", [1, 2, 3, 4])
def test_partials_window_bit_exact_full_size_workload(c_oracle, c):
    """A 256x256 window of the per-group partials of a full-size workload."""
    w = inputs.workload(c)
    rng = np.random.default_rng(100 + c)
    m0 = int(rng.integers(0, max(1, w.M - 256 + 1)))
    n0 = int(rng.integers(0, w.N - 256 + 1)) // 8 * 8
    A = inputs.activations(c)
    W = inputs.weights(c, rows=n0 + 256)
    idx = inputs.outlier_channels(c)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    m1 = min(w.M, m0 + 256)
    P, _ = atom.atom_w4a4_gemm_partials(rows_of(qa, m0, m1), rows_of(qw, n0, n0 + 256), w.K,
                                        want_y=False)
    P = P.cpu().numpy()
    ra = c_oracle.quantize(np.ascontiguousarray(A[m0:m1]), idx)
    rw = c_oracle.quantize(np.ascontiguousarray(W[n0:n0 + 256]), idx)
    P_ref = c_oracle.partials(ra[0], ra[1], rw[0], rw[1], w.K)
    assert np.array_equal(P, P_ref)


# Rows of full-size Y compared with the oracle: every row of workloads 1 and 2,
# and 512 seeded rows (always including the last) of workloads 3 and 4.
FULL_Y_ROWS = {1: None, 2: None, 3: 512, 4: 512}


@pytest.mark.parametrize("c", [1, 2, 3, 4])
def test_full_size_output(c_oracle, c):
    """The full-size GEMM exactly as the benchmark launches it; Y checked on all
    N columns of every row (workloads 1, 2) or of 512 seeded rows (3, 4)
    against the oracle's fp64 output."""
    w = inputs.workload(c)
    A, W, idx = inputs.activations(c), inputs.weights(c), inputs.outlier_channels(c)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    y = atom.atom_w4a4_gemm(qa, qw, w.K)
    torch.cuda.synchronize()
    n_rows = FULL_Y_ROWS[c]
    if n_rows is None or n_rows >= w.M:
        rows = np.arange(w.M)
    else:
        rng = np.random.default_rng(200 + c)
        rows = np.sort(rng.choice(w.M - 1, n_rows - 1, replace=False))
        rows = np.append(rows, w.M - 1)                     # always include the last row
    assert len(np.unique(rows)) == len(rows) == min(w.M, n_rows or w.M)
    ys = y[torch.from_numpy(rows).cuda()].cpu().numpy()
    ra = c_oracle.quantize(np.ascontiguousarray(A[rows]), idx)
    rw = c_oracle.quantize(W, idx)
    Y64 = c_oracle.gemm(*ra, *rw, w.K)
    err = y_rel_err(ys, Y64)
    assert err <= Y_TOL, err
    assert np.isfinite(ys).all()


def test_empty_m_is_a_noop():
    K = 512
    A, W, idx = inputs.random_case(3, 1, 64, K)
    qw = quant_dev(W, idx, weights=True)
    qa = atom.empty_quantized(0, K, "cuda")
    y = atom.atom_w4a4_gemm(qa, qw, K)
    assert y.shape == (0, 64)


def test_back_to_back_calls_are_deterministic():
    A, W, idx = _case("ragged")
    K = A.shape[1]
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    y1 = atom.atom_w4a4_gemm(qa, qw, K).clone()
    y2 = atom.atom_w4a4_gemm(qa, qw, K)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("M,N,K,seed", [(64, 4096, 4096, 21), (40, 520, 2048, 22),
                                        (1, 256, 32768, 23), (130, 1024, 1152, 24)])
def test_split_k_output_matches_oracle_and_unsplit(c_oracle, M, N, K, seed):
    """Small-M shapes split K across CTA pairs (fp32 partial tiles in the
    workspace, summed in split order). Y must be within tolerance of the
    oracle on every row, with and without the split."""
    ws = atom.atom_gemm_workspace_bytes(M, N, K)
    assert ws > 0 and ws % (4 * M * N) == 0        # these shapes do split
    A, W, idx = inputs.random_case(seed, M, N, K, dist="t", param=4.0, outlier_factor=30.0)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    y_split = atom.atom_w4a4_gemm(qa, qw, K).cpu().numpy()
    y_plain = atom.atom_w4a4_gemm(qa, qw, K, split=False).cpu().numpy()
    ra, rw = c_oracle.quantize(A, idx), c_oracle.quantize(W, idx)
    Y64 = c_oracle.gemm(*ra, *rw, K)
    for y in (y_split, y_plain):
        err = y_rel_err(y, Y64)
        assert err <= Y_TOL, err


@pytest.mark.parametrize("N,S", [(8192, 2), (5120, 3), (4096, 4), (3584, 5), (3072, 6),
                                 (2688, 7), (2304, 8)])
def test_small_m_every_cluster_size(c_oracle, N, S):
    """The small-M kernel splits K over a cluster of S CTAs, S = 2 .. 8 as the
    weight tiles fill the 148 SMs, and sums the ranges' partial tiles in
    distributed shared memory, each CTA a slice of the rows (slices of 4-row
    quads, uneven when S does not divide 32). Y must be within tolerance of
    the oracle, split and unsplit."""
    M, K = 17, 2048
    assert atom.atom_gemm_workspace_bytes(M, N, K) == S * M * N * 4
    A, W, idx = inputs.random_case(40 + S, M, N, K, dist="t", param=4.0, outlier_factor=30.0)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    y_split = atom.atom_w4a4_gemm(qa, qw, K).cpu().numpy()
    y_plain = atom.atom_w4a4_gemm(qa, qw, K, split=False).cpu().numpy()
    ra, rw = c_oracle.quantize(A, idx), c_oracle.quantize(W, idx)
    Y64 = c_oracle.gemm(*ra, *rw, K)
    for y in (y_split, y_plain):
        assert y_rel_err(y, Y64) <= Y_TOL


def test_split_k_is_deterministic_and_ignores_a_short_workspace():
    M, N, K = 64, 4096, 4096
    A, W, idx = inputs.random_case(25, M, N, K)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    y1 = atom.atom_w4a4_gemm(qa, qw, K).clone()
    y2 = atom.atom_w4a4_gemm(qa, qw, K)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    # a workspace one byte short of the size asked for runs without the split
    short = torch.empty(atom.atom_gemm_workspace_bytes(M, N, K) - 1, dtype=torch.uint8,
                        device="cuda")
    y3 = atom.atom_w4a4_gemm(qa, qw, K, workspace=short)
    y4 = atom.atom_w4a4_gemm(qa, qw, K, split=False)
    torch.cuda.synchronize()
    assert torch.equal(y3.view(torch.int16), y4.view(torch.int16))


def test_large_shapes_do_not_split():
    assert atom.atom_gemm_workspace_bytes(8192, 28672, 8192) == 0
    assert atom.atom_gemm_workspace_bytes(4096, 11008, 4096) == 0
