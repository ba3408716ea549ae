"""Row-sharded GEMV (all-gather) and expert parallelism with token dispatch
(two all-to-alls) on CPU ranks (gloo, world sizes 2 and 3).

The device steps are replaced by stand-ins with the same contracts, so these
tests check the partition, the exchange sizes and orders, and the reassembly;
tests/test_gpu_ep_exchange.py runs the library's kernels for the same steps.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sub_bit_sparse_b200.ep import expert_range, gemv_row_sharded, moe_ffn_all_to_all, row_range


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("n,world", [(10, 3), (4096, 8), (7, 7), (5, 2)])
def test_row_ranges_cover_every_row_once(n, world):
    rows = []
    for r in range(world):
        b, c = row_range(n, world, r)
        rows.extend(range(b, b + c))
    assert rows == list(range(n))


# ---- stand-ins for the device steps (CPU, float64) ----

def _fake_gemv(w_local, x, count, k):
    assert w_local.shape == (count, k)
    return x @ w_local.T


class FakeKernels:
    """Same contracts as the library's dispatch / one-slot FFN / combine."""

    out_dtype = "float64"

    @staticmethod
    def dispatch(topk_ids, x, topk_weights, n_experts, world):
        t, topk = topk_ids.shape
        flat = topk_ids.reshape(-1)
        owner = torch.tensor([next(r for r in range(world)
                                   if expert_range(n_experts, world, r)[0] <= int(e) <
                                   sum(expert_range(n_experts, world, r))) for e in flat])
        order = torch.argsort(owner, stable=True).to(torch.int32)
        inv = torch.empty_like(order)
        inv[order.long()] = torch.arange(len(order), dtype=torch.int32)
        counts = torch.zeros(world + 1, dtype=torch.int32)
        for r in range(world):
            counts[r] = int((owner == r).sum())
        counts[world] = len(order)
        local = torch.tensor([int(flat[p]) - expert_range(n_experts, world, int(owner[p]))[0] for p in order.tolist()],
                             dtype=torch.int32)
        x_send = x[(order // topk).long()]
        w_send = None if topk_weights is None else topk_weights.reshape(-1)[order.long()]
        return order, inv, counts, local, x_send, w_send

    @staticmethod
    def ffn_rows(gateup_local, down_local, x_rows, local_ids, w_rows, n, hidden, n_local, flags):
        # a per-row function of the row's global expert (begin from the rank) and token
        begin = gateup_local
        assert int(local_ids.max()) < n_local
        g = (local_ids.to(torch.float64) + begin + 1)[:, None] * x_rows[:, :hidden] * 0.5
        return g * w_rows[:, None]

    @staticmethod
    def combine(rows, inv, t, topk):
        out = torch.zeros((t, rows.shape[1]), dtype=rows.dtype)
        for p in range(t * topk):
            if int(inv[p]) >= 0:
                out[p // topk] += rows[int(inv[p])]
        return out


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(5)
        n, k, b = 11, 6, 3
        w = torch.from_numpy(rng.standard_normal((n, k)))
        x = torch.from_numpy(rng.standard_normal((b, k)))
        r0, rc = row_range(n, world, rank)
        y = gemv_row_sharded(w[r0:r0 + rc], x, n, k, gemv_fn=_fake_gemv)
        results[("gemv", rank)] = y.numpy()

        # tokens of this rank: its own slice of a global batch
        E, topk, hidden, t_all = 7, 3, 4, 10
        ids_all = torch.from_numpy(np.stack([np.random.default_rng(40 + i).choice(E, topk, replace=False)
                                             for i in range(t_all)]).astype(np.int32))
        wts_all = torch.from_numpy(np.random.default_rng(6).random((t_all, topk)))
        x_all = torch.from_numpy(np.random.default_rng(7).standard_normal((t_all, hidden)))
        t0, tc = row_range(t_all, world, rank)
        begin, _ = expert_range(E, world, rank)
        out = moe_ffn_all_to_all(begin, None, x_all[t0:t0 + tc], ids_all[t0:t0 + tc], wts_all[t0:t0 + tc],
                                 0, hidden, E, kernels=FakeKernels)
        results[("moe", rank)] = out.numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchanges_reassemble_the_whole_result(world):
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    rng = np.random.default_rng(5)
    w = rng.standard_normal((11, 6))
    x = rng.standard_normal((3, 6))
    for r in range(world):
        assert np.allclose(res[("gemv", r)], x @ w.T, rtol=1e-12, atol=1e-12)
    E, topk, hidden, t_all = 7, 3, 4, 10
    ids_all = np.stack([np.random.default_rng(40 + i).choice(E, topk, replace=False) for i in range(t_all)])
    wts_all = np.random.default_rng(6).random((t_all, topk))
    x_all = np.random.default_rng(7).standard_normal((t_all, hidden))
    whole = np.zeros((t_all, hidden))
    for t in range(t_all):
        for s in range(topk):
            whole[t] += (ids_all[t, s] + 1) * x_all[t] * 0.5 * wts_all[t, s]
    got = np.concatenate([res[("moe", r)] for r in range(world)])
    assert np.allclose(got, whole, rtol=1e-12, atol=1e-12)
