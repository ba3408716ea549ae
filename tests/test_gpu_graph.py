"""The decode GEMV chain as the benchmark runs it: a CUDA graph of calls over
distinct [4096, 7168] matrices, each call prefetching the next matrix into L2
(needs a B200).

Replays of the graph must give the eager calls' bits, and sampled rows must be
within the oracle's tolerance (|dy| <= 1e-3 * sum|W x| + 1e-6).
"""

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sub_bit_sparse_b200 as stq1

N, K, CHAIN = 4096, 7168, 4
ROW_BYTES = K // 256 * 42


@pytest.mark.parametrize("b", [1, 2])
def test_graph_chain_with_prefetch_matches_eager_and_oracle(b):
    dev = torch.device("cuda", 0)
    packed = [workloads.random_packed_blocks(N * K // 256, seed=700 + i) for i in range(CHAIN)]
    stack = torch.stack([torch.from_numpy(p) for p in packed]).to(dev)
    x_bits = workloads.activations_bf16(b, K, seed=71)
    x = torch.from_numpy(x_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    ws = stq1.workspace(stq1.LIB.stq1_gemv_workspace(N, K, b), dev)
    y_eager = torch.empty((CHAIN, b, N), dtype=torch.float32, device=dev)
    y_graph = torch.full((CHAIN, b, N), float("nan"), dtype=torch.float32, device=dev)

    def chain(out):
        for i in range(CHAIN):
            stq1.gemv(stack[i], x, N, K, out=out[i], ws=ws, prefetch=stack[(i + 1) % CHAIN])

    side = torch.cuda.Stream(dev)
    with torch.cuda.stream(side):
        chain(y_eager)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        chain(y_graph)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert stq1.status() == 0
    assert torch.equal(y_graph, y_eager)

    rows = np.sort(np.random.default_rng(b).choice(N, 192, replace=False))
    for i in range(CHAIN):
        sub = packed[i].reshape(N, ROW_BYTES)[rows].reshape(-1)
        want = oracle.gemv(sub, x_bits, len(rows), K)
        tol = oracle.tolerance(oracle.gemv_abs(sub, x_bits, len(rows), K))
        got = y_graph[i][:, torch.from_numpy(rows).to(dev)].cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - want) <= tol), f"matrix {i}"
    del g
