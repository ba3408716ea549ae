"""Failure detection on the GPU without a fault (needs a B200).

Every wait inside this library's kernels is bounded: when the phase it waits
for never completes, the wait gives up, records STQ1_DEV_WAIT_LIMIT in the
device error word and the kernel returns, so the host learns of it through
stq1_status and the context stays usable.  The self-test kernel waits on a
barrier phase that nothing completes; nothing faults, traps or hangs.
"""

import time

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sub_bit_sparse_b200 as stq1


def test_completed_wait_records_nothing():
    assert stq1.selftest_wait(True) == 0


def test_wait_that_runs_out_is_reported_and_the_context_survives():
    t0 = time.perf_counter()
    err = stq1.selftest_wait(False)
    elapsed = time.perf_counter() - t0
    assert err & stq1.DEV_WAIT_LIMIT
    assert elapsed < 10.0
    # the word is cleared by the read, and the next kernels run normally
    assert stq1.status() == 0
    w, x_bits = oracle.encode_plain(workloads.gaussian_matrix(64, 512, 0.02, seed=3)), workloads.activations_bf16(1, 512, 4)
    y = stq1.gemv(torch.from_numpy(w).cuda(), torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16),
                  64, 512).cpu().numpy()
    assert stq1.status() == 0
    want = oracle.gemv(w, x_bits, 64, 512)
    tol = oracle.tolerance(oracle.gemv_abs(w, x_bits, 64, 512))
    assert np.all(np.abs(y - want) <= tol)
