"""Pins of the W4A8 oracle (oracle/w4a8_oracle.py) against things other than itself:
the independent C oracle's INT8 group, hand-worked codes, the round-trip bound,
brute-force partial sums and the textbook integer matmul."""
import numpy as np
import pytest

from oracle import numpy_oracle, w4a8_oracle

from w4a4_mixed_precision_b200 import inputs


def test_every_group_is_the_int8_group_of_the_w4a4_encoding(c_oracle):
    """The W4A4 encoding quantizes its outlier group to INT8 with the same
    formula; the C oracle (separate code) must agree with every INT8 group here:
    shift each group in turn into the outlier slot and compare."""
    rng = np.random.default_rng(3)
    K = 512
    x = (rng.standard_t(4.0, size=(7, K)) * 3).astype(np.float16)
    q8a, sa = w4a8_oracle.quantize_a8(x, np.arange(K - 128, K))
    for g in range(K // 128):
        ch = np.arange(g * 128, (g + 1) * 128)
        _, q8, s = c_oracle.quantize(x, ch)
        assert np.array_equal(q8a[:, g * 128:(g + 1) * 128], q8), g
        assert np.array_equal(sa[g].view(np.uint32), s[-1].view(np.uint32)), g


def test_hand_worked_codes():
    """Group 0 has amax 127, so scale = inv = 1 and q = rint(x) with ties to even;
    group 1 has amax 254, so scale 2, inv 0.5; group 2 is zero."""
    K = 384
    x = np.zeros((1, K), dtype=np.float16)
    x[0, :8] = [127, -127, 63.5, 64.5, 0.5, 1.5, -2.5, 3.0]
    x[0, 128:134] = [254, 1, 3, 5, -7, -254]
    q, s = w4a8_oracle.quantize_a8(x, np.arange(K - 128, K))
    assert q[0, :8].tolist() == [127, -127, 64, 64, 0, 2, -2, 3]
    assert not q[0, 8:128].any()
    assert q[0, 128:134].tolist() == [127, 0, 2, 2, -4, -127]   # 0.5->0, 1.5->2, 2.5->2, -3.5->-4
    assert s[:, 0].tolist() == [1.0, 2.0, 0.0]
    assert not q[0, 256:].any()


def test_round_trip_bound_and_amax_maps_to_127():
    A, _, idx = inputs.random_case(11, 64, 8, 1152, dist="t", param=3.0, outlier_factor=50.0)
    q, s = w4a8_oracle.quantize_a8(A, idx)
    perm = numpy_oracle.permutation(1152, idx)
    xr = A[:, perm].astype(np.float64).reshape(64, 9, 128)
    qq = q.astype(np.float64).reshape(64, 9, 128)
    step = s.T.astype(np.float64)[:, :, None]
    # |x - q*scale| <= scale/2 up to the fp32 rounding of scale, inv and x*inv,
    # which moves x*inv by at most 127 * 3 * 2^-24 code units
    assert (np.abs(xr - qq * step) <= (0.5 + 127 * 2.0 ** -22) * step).all()
    am = np.abs(xr).argmax(axis=2)
    assert (np.abs(np.take_along_axis(qq, am[:, :, None], axis=2)) == 127).all()


def test_partials_brute_force():
    A, W, idx = inputs.random_case(12, 3, 2, 256, dist="t", param=4.0, outlier_factor=30.0)
    qa, _ = w4a8_oracle.quantize_a8(A, idx)
    qw4, qw8, _ = numpy_oracle.quantize(W, idx)
    w = numpy_oracle.codes(qw4, qw8)
    P = w4a8_oracle.partials(qa, qw4, qw8)
    for g in range(2):
        for m in range(3):
            for n in range(2):
                ref = 0
                for k in range(g * 128, (g + 1) * 128):
                    ref += int(qa[m, k]) * int(w[n, k])
                assert P[g, m, n] == ref


def test_lossless_integers_give_the_textbook_integer_matmul():
    """Integer activations whose groups reach 127 and integer weights whose INT4
    groups reach 7 (INT8 group 127) all get scale 1; Y is then A @ W^T."""
    rng = np.random.default_rng(5)
    M, N, K = 9, 6, 512
    A = rng.integers(-127, 128, size=(M, K))
    A[:, ::128] = 127
    W = rng.integers(-7, 8, size=(N, K))
    W[:, ::128] = 7
    W[:, K - 128:] = rng.integers(-127, 128, size=(N, 128))
    W[:, K - 128] = 127
    idx = np.arange(K - 128, K)             # identity reorder
    qa, sa = w4a8_oracle.quantize_a8(A.astype(np.float16), idx)
    qw4, qw8, sw = numpy_oracle.quantize(W.astype(np.float16), idx)
    assert (sa == 1).all() and (sw == 1).all()
    Y = w4a8_oracle.output64(w4a8_oracle.partials(qa, qw4, qw8), sa, sw)
    assert np.array_equal(Y, (A @ W.T).astype(np.float64))


def test_rejects_mismatched_operands():
    qa = np.zeros((2, 256), dtype=np.int8)
    qw4, qw8, _ = numpy_oracle.quantize(np.zeros((3, 384), dtype=np.float16), np.arange(256, 384))
    with pytest.raises(ValueError):
        w4a8_oracle.partials(qa, qw4, qw8)
