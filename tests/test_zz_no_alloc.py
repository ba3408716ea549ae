"""stq1_gemv_noalloc, the GEMV entry point that allocates nothing (needs a B200).

It serves callers that cannot give the library a workspace or let it allocate
(hosts that own all device memory, code that must not call cudaMalloc).  Its
output is checked against the CPU oracle within the tolerance the parity
tests use, on two calls in a row: the built-in scratch is shared by every
call and keeps the previous call's contents, so the second call must come out
bit-identical to the first.  Shapes whose rows hold an odd number of blocks
take the entry point's direct kernel, which needs no scratch.  This file is
collected last on purpose.
"""

import ctypes

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _row_sample(n):
    """Rows checked against the oracle: all of a small matrix, else the first,
    a middle and the last 64 rows."""
    if n <= 512:
        return [(0, n)]
    mid = n // 2
    return [(0, 64), (mid - 32, mid + 32), (n - 64, n)]


@pytest.mark.parametrize("n,k,b", [(4096, 7168, 1), (512, 2048, 3), (4096, 7168, 8), (130, 1024, 2),
                                   (64, 1280, 1), (130, 768, 3)])
def test_noalloc_matches_oracle_on_two_calls(n, k, b):
    import sub_bit_sparse_b200 as stq1
    lib = stq1.LIB
    rng = np.random.default_rng(n + b)
    w = (rng.standard_normal((n, k)) * rng.uniform(0.005, 0.05, (n, 1))).astype(np.float32)
    packed = stq1.quantize_ref(w)
    x = workloads.activations_bf16(b, k, seed=7 + b)
    wd = torch.from_numpy(packed).cuda()
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rb = (k // 256) * 42
    outs = []
    for _ in range(2):
        y = torch.full((b, n), float("nan"), dtype=torch.float32, device="cuda")
        rc = lib.stq1_gemv_noalloc(wd.data_ptr(), xd.data_ptr(), y.data_ptr(), n, k, b, stream)
        assert rc == 0, stq1.ERRORS.get(rc, rc)
        got = y.cpu().numpy()
        for r0, r1 in _row_sample(n):
            sub = packed[r0 * rb:r1 * rb]
            ref = oracle.gemv(sub, x, r1 - r0, k)
            tol = oracle.tolerance(oracle.gemv_abs(sub, x, r1 - r0, k))
            err = np.abs(got[:, r0:r1].astype(np.float64) - ref)
            assert np.all(err <= tol), f"rows {r0}..{r1}: worst ratio {(err / tol).max():.3g}"
        outs.append(got)
    assert np.array_equal(outs[0], outs[1])       # the shared scratch does not leak between calls
    assert stq1.status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import sub_bit_sparse_b200 as stq1
    lib = stq1.LIB
    # [8192, 7168] at batch 16: 2 K splits x 16 x 8192 fp32 partials + 2 KiB counters > 1 MiB
    n, k, b = 8192, 7168, 16
    wd = torch.zeros(oracle.packed_size(n, k), dtype=torch.uint8, device="cuda")
    xd = torch.zeros((b, k), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((b, n), dtype=torch.float32, device="cuda")
    rc = lib.stq1_gemv_noalloc(wd.data_ptr(), xd.data_ptr(), y.data_ptr(), n, k, b,
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -9
