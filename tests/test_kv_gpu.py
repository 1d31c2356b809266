"""GPU parity of the INT4 KV-cache kernels (atom_kv_quant / atom_kv_dequant
through the C ABI) with oracle/kv_oracle.py: bit-exact codes, scales and
dequantized values on seeded caches (ragged group counts, hand-worked groups,
a large cache), and a side stream."""
import numpy as np
import pytest
import torch

from oracle import kv_oracle as kv
from w4a4_mixed_precision_b200 import atom, inputs

pytestmark = pytest.mark.gpu


def _dev16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.uint16)).cuda().view(torch.float16)


def _host16(t):
    torch.cuda.synchronize()
    return t.cpu().view(torch.int16).numpy().view(np.float16)


@pytest.mark.parametrize("tokens,heads,seed", [(1, 1, 1), (7, 3, 2), (33, 5, 3), (16384, 8, 4)])
def test_codes_scales_and_dequant_bit_exact(tokens, heads, seed):
    x = inputs.kv_cache(seed, tokens, heads)
    q4, s = atom.atom_kv_quant(_dev16(x))
    torch.cuda.synchronize()
    q4_ref, s_ref = kv.quantize(x)
    assert np.array_equal(q4.cpu().numpy(), q4_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    y = _host16(atom.atom_kv_dequant(q4, s))
    y_ref = kv.dequantize(q4_ref, s_ref)
    assert np.array_equal(y.view(np.uint16), y_ref.view(np.uint16))


def test_hand_worked_groups():
    x = np.zeros((4, 128), np.float16)
    x[0] = 3.0            # codes 7 -> 0x77
    x[1] = -3.0           # codes -7 -> 0x99
    x[3, 0] = 7.0         # scale 1; ties half to even
    x[3, 1:7] = [0.5, -0.5, 1.5, -1.5, 2.5, -2.5]
    q4, s = atom.atom_kv_quant(_dev16(x))
    q4 = q4.cpu().numpy()
    s = s.cpu().numpy()
    assert (q4[0] == 0x77).all() and (q4[1] == 0x99).all() and (q4[2] == 0).all()
    assert s[2] == 0.0 and s[3] == 1.0
    assert kv.codes(q4[3:4])[0, :7].tolist() == [7, 0, 0, 2, -2, 2, -2]


def test_empty_is_a_noop_and_side_stream():
    x = torch.empty((0, 8, 128), dtype=torch.float16, device="cuda")
    q4, s = atom.atom_kv_quant(x)
    assert q4.shape == (0, 8, 64) and s.shape == (0, 8)
    xs = inputs.kv_cache(9, 300, 8)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        q4, s = atom.atom_kv_quant(_dev16(xs), stream=side)
        y = atom.atom_kv_dequant(q4, s, stream=side)
    side.synchronize()
    q4_ref, s_ref = kv.quantize(xs)
    assert np.array_equal(q4.cpu().numpy(), q4_ref)
    assert np.array_equal(_host16(y).view(np.uint16), kv.dequantize(q4_ref, s_ref).view(np.uint16))
    assert atom.atom_device_status(clear=True) == 0
