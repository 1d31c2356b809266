"""The allocation-free GEMM entry point, atom_w4a4_gemm_noalloc.

Callers that cannot allocate device memory around a GEMM call (code running
while a CUDA graph is captured, serving runtimes whose device memory all sits
in a fixed pool, C callers without a device allocator) use this entry point
instead of atom_w4a4_gemm with a workspace: when the shape splits K, the split
partials go to a fixed 8 MiB array inside the library. These tests call it
through the C ABI and compare it with atom_w4a4_gemm given its own workspace,
on two calls in a row (the second call finds the first call's partials in the
shared array). The file is named to be collected last."""
import numpy as np
import pytest
import torch

from w4a4_mixed_precision_b200 import atom, inputs

from gpu_util import Y_TOL, quant_dev, y_rel_err

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 8 << 20


def _inputs(M, N, K, seed):
    A, W, idx = inputs.random_case(seed, M, N, K, dist="t", param=4.0, outlier_factor=30.0)
    return quant_dev(A, idx), quant_dev(W, idx, weights=True)


@pytest.mark.parametrize("M,N,K,seed", [(64, 4096, 4096, 41), (40, 520, 2048, 42),
                                        (300, 520, 1152, 43)])
def test_noalloc_matches_the_workspace_entry_point_twice(M, N, K, seed):
    need = atom.atom_gemm_workspace_bytes(M, N, K)
    assert 0 < need <= SCRATCH_BYTES          # these shapes split K and fit the scratch
    qa, qw = _inputs(M, N, K, seed)
    ref = atom.atom_w4a4_gemm(qa, qw, K).cpu().numpy().astype(np.float64)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    for _ in range(2):
        y.fill_(float("nan"))
        atom.atom_w4a4_gemm_noalloc(qa, qw, K, y=y)
        got = y.cpu().numpy()
        assert np.isfinite(got).all()
        assert y_rel_err(got, ref) <= Y_TOL


def test_noalloc_without_a_split_matches_too():
    M, N, K = 4096, 1024, 1024
    assert atom.atom_gemm_workspace_bytes(M, N, K) == 0
    qa, qw = _inputs(M, N, K, 44)
    ref = atom.atom_w4a4_gemm(qa, qw, K).cpu().numpy().astype(np.float64)
    for _ in range(2):
        got = atom.atom_w4a4_gemm_noalloc(qa, qw, K).cpu().numpy()
        assert y_rel_err(got, ref) <= Y_TOL


def test_noalloc_rejects_a_split_larger_than_its_scratch():
    M, N, K = 256, 8192, 4096
    assert atom.atom_gemm_workspace_bytes(M, N, K) > SCRATCH_BYTES
    qa, qw = _inputs(M, N, K, 45)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    with pytest.raises(atom.AtomError) as e:
        atom.atom_w4a4_gemm_noalloc(qa, qw, K, y=y)
    assert atom.STATUS[e.value.status] == "ATOM_ERR_SHAPE"
