"""Pins of the INT4 KV-cache oracle (oracle/kv_oracle.py): hand-worked groups,
the already-pinned activation oracle on a group it quantizes the same way, the
round-trip bound, and dequantization by hand."""
import numpy as np
import pytest

from oracle import kv_oracle as kv
from oracle import numpy_oracle as act


def test_hand_worked_groups():
    # constant +c: scale c/7, every code 7 -> bytes 0x77; constant -c: codes -7 -> 0x99
    x = np.stack([np.full(128, 3.0), np.full(128, -3.0), np.zeros(128)]).astype(np.float16)
    q4, s = kv.quantize(x)
    assert (q4[0] == 0x77).all() and (q4[1] == 0x99).all() and (q4[2] == 0).all()
    assert s[0] == np.float32(3.0) / np.float32(7) and s[1] == s[0] and s[2] == 0.0
    # amax 7 -> scale 1, inv 1; ties round half to even: 0.5 -> 0, 1.5 -> 2, 2.5 -> 2
    g = np.zeros(128, np.float16)
    g[0] = 7.0
    g[1:7] = [0.5, -0.5, 1.5, -1.5, 2.5, -2.5]
    q4, s = kv.quantize(g[None])
    assert s[0] == 1.0
    assert kv.codes(q4)[0, :7].tolist() == [7, 0, 0, 2, -2, 2, -2]
    # element 0 -> low nibble of byte 0 (7), element 1 -> high nibble (0): byte 0x07
    assert q4[0, 0] == 0x07


def test_same_encoding_as_the_activation_groups():
    # A K = 256 row whose 128 outlier channels are the tail: its only dense group is
    # channels 0..127 in order, which the (pinned) activation oracle encodes as INT4.
    rng = np.random.default_rng(3)
    x = (rng.standard_t(4, size=(64, 256)) * 2).astype(np.float16)
    q4a, _, sca = act.quantize(x, np.arange(128, 256))
    q4k, sck = kv.quantize(x[:, :128])
    assert np.array_equal(q4a, q4k)
    assert np.array_equal(sca[0], sck)


@pytest.mark.parametrize("seed", [0, 1])
def test_roundtrip_bound_and_code_range(seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((257, 8, 128)) * rng.uniform(0.01, 10, (257, 8, 1))).astype(np.float16)
    q4, s = kv.quantize(x)
    q = kv.codes(q4)
    assert q.min() >= -7 and q.max() <= 7
    err = np.abs(x.astype(np.float64) - q * s[..., None].astype(np.float64))
    assert (err <= s[..., None].astype(np.float64) / 2 * (1 + 2.0 ** -20)).all()
    # the element at amax maps to +-7
    assert (np.abs(q).max(axis=-1)[s > 0] == 7).all()


def test_dequantize_by_hand():
    # byte 0x7F: low nibble 0xF is element 0 (code -1), high nibble 0x7 is element 1 (code 7)
    q4 = np.array([[0x7F] + [0] * 63], dtype=np.uint8)
    y = kv.dequantize(q4, np.array([2.0], np.float32))
    assert y.dtype == np.float16
    assert y[0, 0] == -2.0 and y[0, 1] == 14.0 and (y[0, 2:] == 0).all()
    # fp16 rounding of the fp32 product: 7 * (1 + 2^-12) = 7.0017..., and the fp16
    # neighbours of 7 are 2^-8 apart, so it rounds to 7
    y = kv.dequantize(q4, np.array([1 + 2.0 ** -12], np.float32))
    assert y[0, 1] == 7.0


def test_rejects_other_head_dims():
    with pytest.raises(ValueError):
        kv.quantize(np.zeros((2, 64), np.float16))
