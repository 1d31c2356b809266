"""Failure detection on the GPU: a bounded wait that runs out.

Every pipeline wait of the GEMM and quantizer kernels is an mbarrier wait with
a time limit; when a phase never completes, the wait gives up, records
ATOM_ERR_TIMEOUT in the device status word and the kernel ends instead of
hanging the GPU. atom_debug_wait_timeout runs that same wait on a barrier that
nothing arrives on (no copy or MMA tied to it), with a short limit. The test
checks that the status is reported, that it stays until cleared, and that the
context is still usable afterwards."""
import time

import pytest

from w4a4_mixed_precision_b200 import atom, inputs

from gpu_util import Y_TOL, quant_dev, y_rel_err

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_timeout(c_oracle):
    assert atom.atom_device_status(clear=True) == 0
    limit_ns = 2_000_000                                     # 2 ms
    t0 = time.perf_counter()
    atom.atom_debug_wait_timeout(limit_ns)
    status = atom.atom_device_status(clear=False)            # synchronises
    elapsed = time.perf_counter() - t0
    assert atom.STATUS[status] == "ATOM_ERR_TIMEOUT"
    assert elapsed >= limit_ns * 1e-9                        # it waited for its limit
    assert elapsed < 5.0                                     # and then gave up
    # the status stays until it is cleared
    assert atom.atom_device_status(clear=True) == status
    assert atom.atom_device_status(clear=True) == 0
    # the context is still usable: a GEMM afterwards is correct
    M, N, K = 70, 264, 512
    A, W, idx = inputs.random_case(61, M, N, K)
    qa, qw = quant_dev(A, idx), quant_dev(W, idx, weights=True)
    y = atom.atom_w4a4_gemm(qa, qw, K).cpu().numpy()
    ra, rw = c_oracle.quantize(A, idx), c_oracle.quantize(W, idx)
    assert y_rel_err(y, c_oracle.gemm(*ra, *rw, K)) <= Y_TOL
    assert atom.atom_device_status(clear=True) == 0

