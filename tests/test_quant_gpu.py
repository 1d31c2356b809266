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


def _expected_dev(c_oracle, A, idx):
    q4, q8, sc = c_oracle.quantize(A, idx)
    return tuple(torch.from_numpy(np.ascontiguousarray(t)).cuda() for t in (q4, q8, sc))


def _matches(q, want) -> bool:
    return all(torch.equal(g.view(torch.uint8), w.view(torch.uint8)) for g, w in zip(q, want))


def test_row_counter_slots_reused_over_many_calls(c_oracle):
    """Rows are claimed from a per-call counter slot that the launch resets as
    it ends; 1100 calls take every slot of the ring at least once. Each call
    writes over a poisoned output, so a slot left non-zero by an earlier
    launch (rows skipped) or a row claimed twice shows up as a mismatch. Two
    inputs of different heights alternate, so that grid sizes differ too."""
    cases = [inputs.random_case(31, 300, 8, 1024), inputs.random_case(32, 7, 8, 1024)]
    devs = [(fp16_dev(A), idx_dev(idx), _expected_dev(c_oracle, A, idx)) for A, _, idx in cases]
    outs = [atom.empty_quantized(300, 1024, "cuda"), atom.empty_quantized(7, 1024, "cuda")]
    bad = 0
    for i in range(1100):
        x, idx, want = devs[i % 2]
        out = outs[i % 2]
        for t in out:
            t.view(torch.uint8).fill_(0xAB)
        atom.atom_reorder_quant(x, idx, out=out)
        if not _matches(out, want):
            bad += 1
    assert bad == 0
    assert atom.atom_device_status(clear=True) == 0


def test_concurrent_calls_on_two_streams(c_oracle):
    """Launches on two streams run at the same time on separate counter
    slots; each must still quantize every one of its own rows exactly once."""
    (A, _, idx), (B, _, jdx) = inputs.random_case(41, 2000, 8, 2048), inputs.random_case(42, 1500, 8, 4096)
    xa, ia, wa = fp16_dev(A), idx_dev(idx), _expected_dev(c_oracle, A, idx)
    xb, ib, wb = fp16_dev(B), idx_dev(jdx), _expected_dev(c_oracle, B, jdx)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    outs = []
    for _ in range(20):
        with torch.cuda.stream(s1):
            qa = atom.atom_reorder_quant(xa, ia, stream=s1)
        with torch.cuda.stream(s2):
            qb = atom.atom_reorder_quant(xb, ib, stream=s2)
        outs.append((qa, qb))
    torch.cuda.synchronize()
    for qa, qb in outs:
        assert _matches(qa, wa) and _matches(qb, wb)
    assert atom.atom_device_status(clear=True) == 0


def test_bad_list_call_leaves_counter_slot_clean(c_oracle):
    """A launch that stops at an invalid outlier list still resets its counter
    slot: the next 1024 calls (which reuse that slot last) quantize every row."""
    M, K = 200, 512
    A, _, idx = inputs.random_case(51, M, 8, K)
    bad_idx = idx.copy()
    bad_idx[5] = bad_idx[9]
    x, i, want = fp16_dev(A), idx_dev(idx), _expected_dev(c_oracle, A, idx)
    atom.atom_reorder_quant(x, idx_dev(bad_idx))
    torch.cuda.synchronize()
    assert atom.atom_device_status(clear=True) == 1
    out = atom.empty_quantized(M, K, "cuda")
    bad = 0
    for _ in range(1024):
        for t in out:
            t.view(torch.uint8).fill_(0xAB)
        atom.atom_reorder_quant(x, i, out=out)
        if not _matches(out, want):
            bad += 1
    assert bad == 0
    assert atom.atom_device_status(clear=True) == 0


def test_every_fp16_group_maximum(c_oracle):
    """INT4 groups whose maximum |x| runs through every positive finite fp16
    value (subnormals included, up to 65504), the other 127 elements spread
    below it: scales and codes bit-exact with the oracle's fp32 divisions."""
    K, G = 4096, 4096 // 128
    idx = np.arange(5, K, K // 128, dtype=np.int32)[:128]
    amaxes = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16)   # 31743 values
    rows = -(-amaxes.size // (G - 1))
    rng = np.random.default_rng(7)
    R = np.zeros((rows, K), dtype=np.float16)              # reordered positions
    for n, a in enumerate(amaxes):
        r, g = divmod(n, G - 1)
        grp = (rng.uniform(-1.0, 1.0, 128) * np.float32(a)).astype(np.float16)
        grp[rng.integers(128)] = a if n % 2 else -a
        R[r, g * 128:(g + 1) * 128] = grp
    R[:, (G - 1) * 128:] = rng.standard_normal((rows, 128)).astype(np.float16)
    mask = np.ones(K, bool)
    mask[idx] = False
    order = np.concatenate([np.nonzero(mask)[0], idx])
    A = np.empty_like(R)
    A[:, order] = R
    assert_codes_equal(host(quant_dev(A, idx)), c_oracle.quantize(A, idx), "every fp16 amax")
