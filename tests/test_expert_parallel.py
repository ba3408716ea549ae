"""Expert parallelism of the MoE feed-forward layer: partition and reduction on
CPU ranks (gloo, world sizes 2 and 3), and the per-rank kernels on one GPU."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sub_bit_sparse_b200.ep import expert_parallel, expert_range

import oracle
import workloads


@pytest.mark.parametrize("E,world", [(256, 8), (256, 3), (7, 7), (10, 4)])
def test_expert_ranges_cover_every_expert_once(E, world):
    seen = []
    sizes = []
    for r in range(world):
        b, c = expert_range(E, world, r)
        seen.extend(range(b, b + c))
        sizes.append(c)
    assert seen == list(range(E))
    assert max(sizes) - min(sizes) <= 1


def test_expert_range_rejects_bad_groups():
    with pytest.raises(ValueError):
        expert_range(4, 8, 0)
    with pytest.raises(ValueError):
        expert_range(16, 4, 4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# A stand-in for one rank's kernels with the same contract as stq1_moe_ffn_local:
# out[t] = sum over slots s with ids[t, s] in [begin, begin + count) of
# w[t, s] * f(expert, token), other slots contribute 0.
def _fake_layer(ids, w, begin, count, hidden):
    T, topk = ids.shape
    out = torch.zeros((T, hidden), dtype=torch.float64)
    for t in range(T):
        for s in range(topk):
            e = int(ids[t, s])
            if begin <= e < begin + count:
                out[t] += float(w[t, s]) * torch.arange(hidden, dtype=torch.float64) * (e + 1) * (t + 1)
    return out


def _worker(rank, world, port, E, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ids = workloads.zipf_topk_ids(6, E, 4, seed=3)
        w = workloads.softmax_route_weights(6, 4, seed=4)
        out = expert_parallel(lambda b, c: _fake_layer(ids, w, b, c, 5), E)
        results[rank] = out.numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_partial_outputs_sum_to_the_whole_layer(world):
    E = 16
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, port, E, results), nprocs=world, join=True)
        outs = dict(results)
    ids = workloads.zipf_topk_ids(6, E, 4, seed=3)
    w = workloads.softmax_route_weights(6, 4, seed=4)
    whole = _fake_layer(ids, w, 0, E, 5).numpy()
    for r in range(world):
        assert np.allclose(outs[r], whole, rtol=1e-12, atol=1e-12)   # every rank holds the sum


@pytest.mark.gpu
@pytest.mark.parametrize("world", [1, 4])
@pytest.mark.parametrize("n,hidden,T,flags", [
    (512, 512, 24, 0),      # down rows of one block (odd count): the generic whole-layer chain per rank
    (1024, 512, 24, 0),     # compact rank rows: few pairs per expert (table and tensor-core decode kernels)
    (1024, 512, 24, 1),     # the same with the routing weight on the up half
    (1024, 512, 600, 0),    # compact rank rows, many pairs per expert: the tcgen05 tile kernel
])
def test_rank_shares_on_one_gpu_sum_to_the_oracle(world, n, hidden, T, flags):
    # The per-rank kernels of a G-way expert-parallel layer, run one after the
    # other on one GPU (no collective: the sum is taken here), against the
    # oracle's whole layer.
    import sub_bit_sparse_b200 as stq1
    E, topk = 8, 3
    gu = [stq1.quantize_ref(workloads.gaussian_matrix(n, hidden, 0.05, seed=1100 + e)) for e in range(E)]
    dn = [stq1.quantize_ref(workloads.gaussian_matrix(hidden, n // 2, 0.05, seed=1200 + e)) for e in range(E)]
    x = workloads.activations_bf16(T, hidden, seed=13)
    ids = workloads.zipf_topk_ids(T, E, topk, seed=14)
    wts = workloads.softmax_route_weights(T, topk, seed=15)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    xd = dev(x.view(np.int16)).view(torch.bfloat16)
    total = torch.zeros((T, hidden), dtype=torch.float32, device="cuda")
    for r in range(world):
        b, c = expert_range(E, world, r)
        part = stq1.moe_ffn_local(dev(np.concatenate(gu[b:b + c])), dev(np.concatenate(dn[b:b + c])), xd,
                                  dev(ids.astype(np.int32)), dev(wts), n, hidden, c, b, flags=flags)
        total += part
    assert stq1.status() == 0                          # foreign ids are not errors
    ref, scale = oracle.moe_ffn(gu, dn, x, ids, wts, n, hidden, flags=flags, abs_sum=True)
    err = np.abs(total.cpu().numpy().astype(np.float64) - ref)
    # Bound for a sum of `world` partials: rank r's partial covers its own slots,
    # so it is within 1e-3 * S_r + 1e-6 of the oracle's partial (S_r = its share
    # of `scale`, and the S_r add up to `scale`); the world - 1 fp32 additions
    # each add at most one rounding, |sum| * 2^-24 <= (scale + 1e-6 world) * 2^-24.
    # Hence err <= 1e-3 * scale + world * 1e-6 + (world - 1) * 2^-24 * (scale + 1e-6 world).
    bound = oracle.tolerance(scale) + (world - 1) * (1e-6 + 2.0 ** -24 * (scale + 1e-6 * world))
    assert np.all(err <= bound)
