"""MoE decode calls whose experts are split between the table kernel and the
tensor-core decode kernel (needs a B200).

Such a call runs the tensor-core part on a second stream that the library
keeps per device and host thread, forked from the caller's stream and joined
before the call returns.  These tests check that:
- a CUDA graph captured from such calls replays to the eager calls' bits;
- calls from two host threads on their own streams give the same bits as
  the same calls made one after another;
- work enqueued on the caller's stream after the call sees both parts.
The routing is fixed so that experts 0, 1 and 2 get three or more pairs
(tensor-core part) and experts 3..7 one or two (table part).
Bar against the oracle: |y - y_oracle| <= 1e-3 * sum_k |W^[j,k] x[t,k]| + 1e-6.
"""

import threading

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sub_bit_sparse_b200 as stq1

E, N, K, TOPK = 8, 1024, 1536, 3
IDS = np.array([[0, 1, 2], [0, 1, 3], [0, 2, 4], [0, 5, 6], [0, 7, 1], [2, 3, 5]], dtype=np.int32)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _inputs(seed):
    mats = [oracle.encode_plain(workloads.gaussian_matrix(N, K, 0.03, seed=seed + e)) for e in range(E)]
    x = workloads.activations_bf16(IDS.shape[0], K, seed=seed + 100)
    wts = workloads.softmax_route_weights(IDS.shape[0], TOPK, seed=seed + 101)
    return mats, x, wts


def _call(bank, xd, idd, wd, out=None):
    return stq1.moe_gateup(bank, xd, idd, wd, N, K, E, flags=stq1.MOE_WEIGHT_UP, out=out)


def test_split_call_matches_the_oracle_and_later_work_sees_both_parts():
    mats, x, wts = _inputs(500)
    bank, xd, idd, wd = _dev(np.concatenate(mats)), _dev(x.view(np.int16)).view(torch.bfloat16), _dev(IDS), _dev(wts)
    y = torch.full((IDS.shape[0], TOPK, N), float("nan"), dtype=torch.float32, device="cuda")
    _call(bank, xd, idd, wd, out=y)
    early = y.clone()                                  # enqueued right after the call on the same stream
    ref, bound = oracle.moe_gateup(mats, x, IDS, wts, N, K, flags=stq1.MOE_WEIGHT_UP, abs_sum=True)
    assert stq1.status() == 0
    assert torch.equal(early, y)                       # the copy saw both parts' rows
    err = np.abs(y.cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= oracle.tolerance(bound))


def test_graph_of_split_calls_replays_to_the_eager_bits():
    mats, x, wts = _inputs(600)
    bank, xd, idd, wd = _dev(np.concatenate(mats)), _dev(x.view(np.int16)).view(torch.bfloat16), _dev(IDS), _dev(wts)
    eager = _call(bank, xd, idd, wd).clone()
    side = torch.cuda.Stream()
    outs = [torch.full_like(eager, float("nan")) for _ in range(3)]
    with torch.cuda.stream(side):
        _call(bank, xd, idd, wd, out=outs[0])          # first call of this thread: creates its side stream
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for o in outs:
            _call(bank, xd, idd, wd, out=o)
    for o in outs:
        o.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    for o in outs:
        assert torch.equal(o, eager)
    assert stq1.status() == 0
    del g


def test_calls_from_two_host_threads_give_the_serial_bits():
    data = []
    for seed in (700, 800):
        mats, x, wts = _inputs(seed)
        data.append((_dev(np.concatenate(mats)), _dev(x.view(np.int16)).view(torch.bfloat16), _dev(IDS), _dev(wts)))
    serial = [_call(*d).clone() for d in data]
    torch.cuda.synchronize()
    results, errors = [None, None], []

    def worker(i):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                outs = [_call(*data[i]) for _ in range(20)]
            s.synchronize()
            results[i] = outs
        except Exception as exc:  # reported below
            errors.append(exc)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for i in range(2):
        for o in results[i]:
            assert torch.equal(o, serial[i])
    assert stq1.status() == 0
