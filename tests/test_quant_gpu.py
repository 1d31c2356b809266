"""Parity of the CUDA reorder+quantize kernel with the CPU oracle: INT4 codes,
INT8 outlier codes and fp32 scales must be bit-identical on every row of every
workload, plus ragged, padded and degenerate cases."""
import numpy as np
import pytest
import torch

from w4a4_mixed_precision_b200 import atom, inputs

from gpu_util import assert_codes_equal, fp16_dev, host, idx_dev, quant_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _clear_status():
    atom.atom_device_status(clear=True)
    yield
    assert atom.atom_device_status(clear=True) == 0


@pytest.mark.parametrize("c", [0, 1, 2, 3, 4])
def test_activation_codes_bit_exact_all_rows(c_oracle, c):
    A, idx = inputs.activations(c), inputs.outlier_channels(c)
    got = host(quant_dev(A, idx))
    assert_codes_equal(got, c_oracle.quantize(A, idx), f"workload {c} activations")


@pytest.mark.parametrize("c", [0, 1, 2, 3, 4])
def test_weight_codes_bit_exact_all_rows(c_oracle, c):
    W, idx = inputs.weights(c), inputs.outlier_channels(c)
    got = host(quant_dev(W, idx, weights=True))
    assert_codes_equal(got, c_oracle.quantize(W, idx), f"workload {c} weights")


@pytest.mark.parametrize("M,K,seed", [(1, 256, 1), (3, 384, 2), (333, 1152, 3), (777, 4224, 4),
                                      (64, 32768, 5), (1000, 24576, 6)])
def test_ragged_sizes_unsorted_outliers(c_oracle, M, K, seed):
    A, _, idx = inputs.random_case(seed, M, 8, K, dist="t", param=3.0, outlier_factor=50.0,
                                   sorted_outliers=False)
    assert_codes_equal(host(quant_dev(A, idx)), c_oracle.quantize(A, idx), f"{M}x{K}")


def test_padded_rows_leading_dimension(c_oracle):
    M, K, ld = 50, 640, 648
    A, _, idx = inputs.random_case(8, M, 8, ld, sorted_outliers=True)
    idx = idx[idx < K]
    rng = np.random.default_rng(3)
    extra = np.setdiff1d(np.arange(K), idx)
    idx = np.concatenate([idx, rng.choice(extra, 128 - idx.size, replace=False)]).astype(np.int32)
    full = fp16_dev(A)                        # [M, ld] with ld > K
    got = atom.atom_reorder_quant(full[:, :K], idx_dev(idx))
    assert_codes_equal(host(got), c_oracle.quantize(np.ascontiguousarray(A[:, :K]), idx), "padded")


def test_degenerate_rows(c_oracle):
    """All-zero rows, constant rows, fp16 subnormals, exact ties and +-65504."""
    K = 512
    idx = np.arange(0, K, 4, dtype=np.int32)          # 128 outliers spread over the row
    rows = [np.zeros(K), np.full(K, 0.75), np.full(K, -2.5),
            np.full(K, 2.0 ** -24) * np.arange(K) % 7,     # subnormal fp16 values
            np.tile([7.0, 0.5, -0.5, 1.5, -1.5, 2.5, -2.5, 0.0], K // 8),
            np.tile([65504.0, -65504.0, 1.0, 0.0], K // 4),
            np.linspace(-1e-3, 1e-3, K)]
    A = np.stack(rows).astype(np.float16)
    assert_codes_equal(host(quant_dev(A, idx)), c_oracle.quantize(A, idx), "degenerate")


def test_empty_input_is_a_noop():
    x = torch.empty((0, 512), dtype=torch.float16, device="cuda")
    idx = torch.arange(128, dtype=torch.int32, device="cuda")
    q = atom.atom_reorder_quant(x, idx)
    assert q.q4.shape == (0, 192)


@pytest.mark.parametrize("bad", ["repeated", "out_of_range"])
def test_bad_outlier_list_writes_nothing_and_sets_status(bad):
    M, K = 40, 512
    A, _, idx = inputs.random_case(4, M, 8, K)
    idx = idx.copy()
    if bad == "repeated":
        idx[7] = idx[3]
    else:
        idx[0] = K + 5
    out = atom.empty_quantized(M, K, "cuda")
    for t in out:
        t.view(torch.uint8).fill_(0xAB)
    atom.atom_reorder_quant(fp16_dev(A), idx_dev(idx), out=out)
    assert atom.atom_device_status(clear=True) == 1          # ATOM_ERR_INVALID_ARG
    for t in out:
        assert bool((t.view(torch.uint8) == 0xAB).all())
    # the context stays usable afterwards
    q = quant_dev(A, np.sort(np.random.default_rng(0).choice(K, 128, replace=False)))
    torch.cuda.synchronize()
    assert atom.atom_device_status(clear=True) == 0
    assert q.q4.shape == (M, 192)


def test_runs_on_a_side_stream(c_oracle):
    A, _, idx = inputs.random_case(21, 300, 8, 1024)
    s = torch.cuda.Stream()
    x, i = fp16_dev(A), idx_dev(idx)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        q = atom.atom_reorder_quant(x, i, stream=s)
    s.synchronize()
    assert_codes_equal(host(q), c_oracle.quantize(A, idx), "side stream")
