"""The roofline crossover workload at its full size, vs the CPU oracle (needs a B200).

One [18432, 7168] STQ1_0 matrix with the decode matrix's statistics (row
scales log-uniform in [0.005, 0.05], 0.1% outliers at 10 sigma; seeds 13-15),
Sherry-encoded with calibration importance (seed 16), and bf16 activations
x [1024, 7168] (seed 17); batches 1, 4, 16, 64, 256 and 1024 are prefixes of
x.  Every batch runs on each kernel the library has for it (forced), and on
the library's own choice.  The oracle recomputes three slabs of rows -- the
first, one in the middle and the last -- for every token: fp64 over 768 rows
is seconds, the whole matrix would be minutes.
Bar: |y_gpu - y_oracle| <= 1e-3 * sum_k |W^[j,k] x[t,k]| + 1e-6.
"""

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sub_bit_sparse_b200 as stq1

N, K = 18432, 7168
SLABS = [(0, 256), (9088, 9344), (N - 256, N)]


@pytest.fixture(scope="module")
def crossover():
    w, h, x = workloads.crossover_inputs()
    packed = stq1.quantize_ref(w, h, mode="sherry", rounds=3)
    rb = (K // 256) * 42
    ref = {}
    for r0, r1 in SLABS:
        sub = packed[r0 * rb:r1 * rb]
        ref[(r0, r1)] = (oracle.gemv(sub, x, r1 - r0, K), oracle.gemv_abs(sub, x, r1 - r0, K))
    wd = torch.from_numpy(packed).cuda()
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    return wd, xd, ref


@pytest.mark.parametrize("path", ["auto", "table", "mma", "tiles"])
@pytest.mark.parametrize("b", [1, 4, 16, 64, 256, 1024])
def test_crossover_workload(crossover, path, b):
    wd, xd, ref = crossover
    code = {"auto": stq1.PATH_AUTO, "table": stq1.PATH_TABLE, "mma": stq1.PATH_MMA,
            "tiles": stq1.PATH_TILES}[path]
    stq1.set_path(code)
    try:
        y = stq1.gemv(wd, xd[:b].contiguous(), N, K).cpu().numpy()
    finally:
        stq1.set_path(stq1.PATH_AUTO)
    assert stq1.status() == 0
    for (r0, r1), (yr, ya) in ref.items():
        err = np.abs(y[:, r0:r1].astype(np.float64) - yr[:b])
        tol = oracle.tolerance(ya[:b])
        bad = err > tol
        assert not bad.any(), (f"{path} b={b} rows {r0}..{r1}: {bad.sum()} outside tolerance, "
                               f"worst ratio {(err / tol).max():.3g}")
