"""Pins of the W8A8 comparator oracle (oracle/w8a8_oracle.py) to things other
than itself: a hand-worked case, brute force on tiny inputs, the per-tensor
special case against the textbook integer matmul, and the extreme sum."""
import numpy as np
import pytest

from oracle import w8a8_oracle as o


def test_hand_worked_case():
    # qa rows (1, -2, 3) and (4, 0, -1); qw rows (2, 1, 1) and (-1, 5, 0):
    #   P[0,0] = 2 - 2 + 3 = 3      P[0,1] = -1 - 10 + 0 = -11
    #   P[1,0] = 8 + 0 - 1 = 7      P[1,1] = -4 + 0 + 0 = -4
    qa = np.array([[1, -2, 3], [4, 0, -1]], dtype=np.int8)
    qw = np.array([[2, 1, 1], [-1, 5, 0]], dtype=np.int8)
    assert o.partials(qa, qw).tolist() == [[3, -11], [7, -4]]
    sa = np.array([0.5, 2.0], dtype=np.float32)
    sw = np.array([0.25, 1.0], dtype=np.float32)
    # Y = (P * sa) * sw: row 0 -> (0.375, -5.5), row 1 -> (3.5, -8)
    assert o.output64(qa, sa, qw, sw).tolist() == [[0.375, -5.5], [3.5, -8.0]]


def test_brute_force_on_tiny_random_inputs():
    rng = np.random.default_rng(7)
    qa = rng.integers(-127, 128, size=(3, 19), dtype=np.int64).astype(np.int8)
    qw = rng.integers(-127, 128, size=(5, 19), dtype=np.int64).astype(np.int8)
    sa = rng.uniform(0.01, 2, 3).astype(np.float32)
    sw = rng.uniform(0.01, 2, 5).astype(np.float32)
    Y = o.output64(qa, sa, qw, sw)
    for m in range(3):
        for n in range(5):
            p = 0
            for k in range(19):
                p += int(qa[m, k]) * int(qw[n, k])
            assert o.partials(qa, qw)[m, n] == p
            assert Y[m, n] == (float(p) * float(sa[m])) * float(sw[n])


def test_per_tensor_scale_is_the_textbook_integer_matmul():
    rng = np.random.default_rng(8)
    qa = rng.integers(-127, 128, size=(16, 64), dtype=np.int64).astype(np.int8)
    qw = rng.integers(-127, 128, size=(24, 64), dtype=np.int64).astype(np.int8)
    textbook = np.matmul(qa.astype(np.int64), qw.astype(np.int64).T)
    ones_a = np.ones(16, np.float32)
    ones_w = np.ones(24, np.float32)
    assert np.array_equal(o.output64(qa, ones_a, qw, ones_w), textbook.astype(np.float64))
    # a power-of-two per-tensor scale only moves the exponent
    assert np.array_equal(o.output64(qa, ones_a * 0.5, qw, ones_w * 0.125),
                          textbook.astype(np.float64) / 16.0)


@pytest.mark.parametrize("K", [16, 131072])
def test_extreme_sums(K):
    qa = np.full((1, K), 127, dtype=np.int8)
    qw = np.full((2, K), -127, dtype=np.int8)
    qw[1, :] = 127
    P = o.partials(qa, qw)
    assert P.tolist() == [[-127 * 127 * K, 127 * 127 * K]]
    assert abs(P).max() < 2 ** 31   # the int32 accumulator of the GPU path holds it


def test_rejects_mismatched_operands():
    with pytest.raises(ValueError):
        o.partials(np.zeros((2, 16), np.int8), np.zeros((2, 32), np.int8))
    with pytest.raises(ValueError):
        o.partials(np.zeros((2, 16), np.int16), np.zeros((2, 16), np.int8))
