"""The allocation-free GEMM entry point, atom_w4a4_gemm_noalloc.

Some callers cannot allocate device memory around a GEMM call: a serving
runtime that hands all of its device memory to a fixed pool at start-up has
nothing left to allocate from, and a C or embedded caller may have no device
allocator at all. For them the library keeps the scratch of a K split (the fp32
partial tiles, M > 64 with few output tiles) in a fixed 8 MiB array of its own
device memory. These tests call the entry point through the C ABI, twice in a
row on the same shape (the second call finds the first call's partials still in
the shared array), and check each result against the CPU oracle's fp64 output
and bit for bit against atom_w4a4_gemm given its own workspace (same kernels,
same split, same order). The file is named to be collected last."""
import numpy as np
import pytest
import torch

from w4a4_mixed_precision_b200 import atom, inputs

from gpu_util import Y_TOL, quant_dev, y_rel_err

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 8 << 20


def _case(c_oracle, M, N, K, seed):
    A, W, idx = inputs.random_case(seed, M, N, K, dist="t", param=4.0, outlier_factor=30.0)
    ra, rw = c_oracle.quantize(A, idx), c_oracle.quantize(W, idx)
    Y64 = c_oracle.gemm(*ra, *rw, K)
    return quant_dev(A, idx), quant_dev(W, idx, weights=True), Y64


# M > 64: the large kernel writes its split's partial tiles into the scratch and a
# second kernel sums them; M <= 64: the small-M kernel sums its K ranges inside a
# thread-block cluster (the scratch only permits the split).
@pytest.mark.parametrize("M,N,K,seed", [(300, 520, 1152, 43), (96, 1024, 2048, 46),
                                        (130, 1024, 1152, 47), (64, 4096, 4096, 41),
                                        (40, 520, 2048, 42)])
def test_noalloc_matches_oracle_and_workspace_entry_twice(c_oracle, M, N, K, seed):
    need = atom.atom_gemm_workspace_bytes(M, N, K)
    assert 0 < need <= SCRATCH_BYTES          # these shapes split K and fit the scratch
    qa, qw, Y64 = _case(c_oracle, M, N, K, seed)
    ref = atom.atom_w4a4_gemm(qa, qw, K).clone()
    assert y_rel_err(ref.cpu().numpy(), Y64) <= Y_TOL
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    for _ in range(2):
        y.fill_(float("nan"))
        atom.atom_w4a4_gemm_noalloc(qa, qw, K, y=y)
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        assert np.isfinite(got).all()
        assert y_rel_err(got, Y64) <= Y_TOL
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


def test_noalloc_alternating_shapes_do_not_mix_partials(c_oracle):
    """Two split shapes called alternately: each call must overwrite every
    partial it sums, whatever the previous call left in the shared array."""
    cases = [(300, 520, 1152, 48), (96, 1024, 2048, 49)]
    data = [_case(c_oracle, *c) for c in cases]
    for _ in range(2):
        for (M, N, K, _s), (qa, qw, Y64) in zip(cases, data):
            got = atom.atom_w4a4_gemm_noalloc(qa, qw, K).cpu().numpy()
            assert y_rel_err(got, Y64) <= Y_TOL


def test_noalloc_without_a_split_matches_too(c_oracle):
    M, N, K = 4096, 1024, 1024
    assert atom.atom_gemm_workspace_bytes(M, N, K) == 0
    qa, qw, Y64 = _case(c_oracle, M, N, K, 44)
    ref = atom.atom_w4a4_gemm(qa, qw, K)
    for _ in range(2):
        got = atom.atom_w4a4_gemm_noalloc(qa, qw, K)
        torch.cuda.synchronize()
        assert y_rel_err(got.cpu().numpy(), Y64) <= Y_TOL
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_noalloc_rejects_a_split_larger_than_its_scratch():
    M, N, K = 256, 8192, 4096
    assert atom.atom_gemm_workspace_bytes(M, N, K) > SCRATCH_BYTES
    A, W, idx = inputs.random_case(45, M, N, K)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    with pytest.raises(atom.AtomError) as e:
        atom.atom_w4a4_gemm_noalloc(qa, qw, K, y=y)
    assert atom.STATUS[e.value.status] == "ATOM_ERR_SHAPE"
    assert atom.atom_device_status(clear=True) == 0
