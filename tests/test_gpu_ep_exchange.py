"""Expert parallelism with token dispatch and the row-sharded GEMV, with the
library's kernels on one GPU (needs a B200).

The ranks run one after another and the all-to-all / all-gather are done
here by slicing (nothing waits on another rank).  Each rank's tokens are
grouped by owner (stq1_ep_dispatch), every owner runs the rows it receives
through its experts as one-slot tokens (stq1_moe_ffn_local), the results go
back in send order and are summed per token (stq1_ep_combine); the
concatenated outputs are checked against the oracle's whole layer.
Bar: |out - oracle| <= 1e-3 * sum |W_down act| |w| + 1e-6 per output (the
sum of at most topk rows, each within its own bound, plus their fp32 adds).
"""

import numpy as np
import pytest

import oracle
import workloads
from sub_bit_sparse_b200.ep import expert_range, row_range

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sub_bit_sparse_b200 as stq1


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("world,t_all,flags", [(2, 24, 0), (4, 40, 1), (3, 600, 0)])
def test_dispatch_experts_combine_equals_the_whole_layer(world, t_all, flags):
    n, hidden, E, topk = 1024, 512, 8, 3
    gu = [stq1.quantize_ref(workloads.gaussian_matrix(n, hidden, 0.05, seed=2100 + e)) for e in range(E)]
    dn = [stq1.quantize_ref(workloads.gaussian_matrix(hidden, n // 2, 0.05, seed=2200 + e)) for e in range(E)]
    x = workloads.activations_bf16(t_all, hidden, seed=23)
    ids = workloads.zipf_topk_ids(t_all, E, topk, seed=24)
    wts = workloads.softmax_route_weights(t_all, topk, seed=25)
    banks = []
    for r in range(world):
        b, c = expert_range(E, world, r)
        banks.append((_dev(np.concatenate(gu[b:b + c])), _dev(np.concatenate(dn[b:b + c])), c))
    # dispatch on every rank
    sent = []
    for r in range(world):
        t0, tc = row_range(t_all, world, r)
        xd = _dev(x[t0:t0 + tc].view(np.int16)).view(torch.bfloat16)
        order, inv, counts, local, x_send, w_send = stq1.ep_dispatch(_dev(ids[t0:t0 + tc]), xd, _dev(wts[t0:t0 + tc]),
                                                                     E, world)
        c = counts.cpu().numpy()
        assert c[world] == tc * topk and c[:world].sum() == c[world]
        # every pair once, grouped by owner, local ids in range
        o = order.cpu().numpy()
        assert sorted(o.tolist()) == list(range(tc * topk))
        assert np.array_equal(inv.cpu().numpy()[o], np.arange(tc * topk))
        start = np.concatenate([[0], np.cumsum(c[:world])])
        flat = ids[t0:t0 + tc].reshape(-1)
        for q in range(world):
            b, cnt = expert_range(E, world, q)
            seg = o[start[q]:start[q + 1]]
            assert np.all((flat[seg] >= b) & (flat[seg] < b + cnt))
            assert np.array_equal(local.cpu().numpy()[start[q]:start[q + 1]], flat[seg] - b)
        assert torch.equal(x_send, xd[(order // topk).long()])
        sent.append((start, local, x_send, w_send, inv, tc))
    # every owner: rows from ranks 0..world-1 in rank order, through its experts
    back = [[None] * world for _ in range(world)]
    for q in range(world):
        rows_x = torch.cat([s[2][s[0][q]:s[0][q + 1]] for s in sent])
        rows_id = torch.cat([s[1][s[0][q]:s[0][q + 1]] for s in sent])
        rows_w = torch.cat([s[3][s[0][q]:s[0][q + 1]] for s in sent])
        gq, dq, cq = banks[q]
        res = stq1.moe_ffn_local(gq, dq, rows_x, rows_id.view(-1, 1), rows_w.view(-1, 1), n, hidden, cq, 0,
                                 flags=flags)
        pos = 0
        for r in range(world):
            m = int(sent[r][0][q + 1] - sent[r][0][q])
            back[r][q] = res[pos:pos + m]
            pos += m
    out = [stq1.ep_combine(torch.cat(back[r]), sent[r][4], sent[r][5], topk) for r in range(world)]
    assert stq1.status() == 0
    got = torch.cat(out).cpu().numpy().astype(np.float64)
    ref, scale = oracle.moe_ffn(gu, dn, x, ids, wts, n, hidden, flags=flags, abs_sum=True)
    bound = oracle.tolerance(scale) + topk * (1e-6 + 2.0 ** -24 * (scale + 1e-6 * topk))
    assert np.all(np.abs(got - ref) <= bound)


@pytest.mark.parametrize("world", [2, 3, 8])
def test_row_shards_concatenate_to_the_gemv(world):
    n, k, b = 4096, 7168, 3
    w = workloads.gaussian_matrix(n, k, 0.02, seed=31)
    packed = stq1.quantize_ref(w)
    x = workloads.activations_bf16(b, k, seed=32)
    xd = _dev(x.view(np.int16)).view(torch.bfloat16)
    rb = (k // 256) * 42
    parts = []
    for r in range(world):
        r0, rc = row_range(n, world, r)
        parts.append(stq1.gemv(_dev(packed[r0 * rb:(r0 + rc) * rb]), xd, rc, k))
    y = torch.cat(parts, dim=1).cpu().numpy()
    err = np.abs(y.astype(np.float64) - oracle.gemv(packed, x, n, k))
    assert np.all(err <= oracle.tolerance(oracle.gemv_abs(packed, x, n, k)))
