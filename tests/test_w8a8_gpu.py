"""GPU parity of the W8A8 comparator (atom_w8a8_gemm through the C ABI) with
the CPU oracle in oracle/w8a8_oracle.py, on seeded int8 inputs: ragged and
multi-tile shapes, a K that is not a multiple of 128, the smallest shapes,
sampled rows of the full Llama-70B MLP-up shape, and determinism."""
import numpy as np
import pytest
import torch

from oracle import w8a8_oracle as o
from w4a4_mixed_precision_b200 import atom, inputs

from gpu_util import Y_TOL, y_rel_err

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run(qa, qw, sa, sw):
    y = atom.atom_w8a8_gemm(_dev(qa), _dev(sa), _dev(qw), _dev(sw))
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("M,N,K,seed", [
    (1, 8, 16, 1),          # smallest shape: one row, one 8-column chunk, one partial K step
    (16, 256, 512, 2),      # one tile, all of N
    (300, 520, 1040, 3),    # ragged M and N tails, K = 8 * 128 + 16
    (513, 776, 4096, 4),    # several tiles in both directions
    (256, 256, 131072, 5),  # the longest K the int32 accumulator allows
])
def test_matches_oracle(M, N, K, seed):
    qa, qw, sa, sw = inputs.int8_case(seed, M, N, K)
    y = _run(qa, qw, sa, sw)
    Y64 = o.output64(qa, sa, qw, sw)
    assert np.isfinite(y).all()
    assert y_rel_err(y, Y64) <= Y_TOL


def test_extreme_values_do_not_overflow():
    M, N, K = 128, 256, 131072
    qa = np.full((M, K), 127, dtype=np.int8)
    qw = np.full((N, K), -127, dtype=np.int8)
    qw[1::2] = 127
    sa = np.full(M, 2.0 ** -20, dtype=np.float32)
    sw = np.full(N, 2.0 ** -10, dtype=np.float32)
    y = _run(qa, qw, sa, sw)
    Y64 = o.output64(qa, sa, qw, sw)
    assert y_rel_err(y, Y64) <= Y_TOL


def test_full_shape_sampled_rows():
    # Llama-70B MLP up (8192 x 28672 x 8192); the oracle checks 64 seeded rows.
    M, N, K = 8192, 28672, 8192
    qa, qw, sa, sw = inputs.int8_case(11, M, N, K)
    y = _run(qa, qw, sa, sw)
    rows = np.sort(np.random.default_rng(12).choice(M, 64, replace=False))
    Y64 = o.output64(qa[rows], sa[rows], qw, sw)
    assert y_rel_err(y[rows], Y64) <= Y_TOL


def test_deterministic_and_stream_ordered():
    qa, qw, sa, sw = inputs.int8_case(21, 700, 1032, 2048)
    a, w, s1, s2 = _dev(qa), _dev(qw), _dev(sa), _dev(sw)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        y1 = atom.atom_w8a8_gemm(a, s1, w, s2, stream=side)
        y2 = atom.atom_w8a8_gemm(a, s1, w, s2, stream=side)
    side.synchronize()
    assert torch.equal(y1, y2)
    assert atom.atom_device_status(clear=True) == 0
