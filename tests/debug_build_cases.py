"""Small parity cases run on the bounds-checking build (libstq1_debug.so).

Run as a script in a process of its own with STQ1_DEBUG=1 in the environment
(tests/test_gpu_debug_build.py does that): the package then loads the debug
build.  Every case is checked against the CPU oracle and must leave the
device error word at zero, so no bounds check fires on valid input; the
self-test shows that a check which fails records STQ1_DEV_BOUNDS and leaves
the context usable.  The shapes cover the paths whose indices the checks
guard:
- the table, tensor-core decode and tile kernels, and the split-K plans;
- ragged row counts with a partial last super-row (tail slots) and experts
  that start inside a super-row;
- MoE decode with small and large experts, and MoE prefill in bf16 and fp8;
- one rank's compact experts, the token dispatch and combine;
- the GEMV that allocates nothing.
Prints "OK" and exits 0 when every case passes.
Bar: |y_gpu - y_oracle| <= 1e-3 * sum_k |W^[j,k] x[t,k]| + 1e-6.
"""

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import oracle  # noqa: E402
import workloads  # noqa: E402
import sub_bit_sparse_b200 as stq1  # noqa: E402
from sub_bit_sparse_b200.ep import expert_range, row_range  # noqa: E402


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _bf16(x_bits):
    return _dev(x_bits.view(np.int16)).view(torch.bfloat16)


def _close(y, ref, bound, what):
    err = np.abs(np.asarray(y, dtype=np.float64) - ref)
    tol = oracle.tolerance(bound)
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst {(err / tol).max():.3g}"


def _clean(what):
    err = stq1.status()
    assert err == 0, f"{what}: device error bits {err:#x}"


def check_build_and_selftest():
    assert stq1.DEBUG_BUILD and stq1.build_flags() == stq1.BUILD_DEBUG
    assert stq1.selftest_bounds(5, 10) == 0
    assert stq1.selftest_bounds(12, 10) == stq1.DEV_BOUNDS
    assert stq1.selftest_bounds(-1, 4) == stq1.DEV_BOUNDS
    _clean("after the self-test")                      # the read cleared the word


def check_gemv():
    # K = 1536: 252-byte rows, four rows per super-row; N = 302 leaves a
    # partial last super-row of two rows.  K = 1024: two rows per super-row.
    for n, k in ((302, 1536), (258, 1024)):
        w = workloads.gaussian_matrix(n, k, 0.03, seed=n + k)
        packed = oracle.encode_plain(w)
        wd = _dev(packed)
        for b in (1, 2, 3, 5, 8, 16, 40):
            x = workloads.activations_bf16(b, k, seed=b)
            ref, bound = oracle.gemv(packed, x, n, k), oracle.gemv_abs(packed, x, n, k)
            for path in (stq1.PATH_AUTO, stq1.PATH_TABLE, stq1.PATH_MMA, stq1.PATH_TILES):
                stq1.set_path(path)
                try:
                    y = stq1.gemv(wd, _bf16(x), n, k).cpu().numpy()
                finally:
                    stq1.set_path(stq1.PATH_AUTO)
                _close(y, ref, bound, f"gemv n={n} k={k} b={b} path={path}")
                _clean(f"gemv n={n} k={k} b={b} path={path}")
            if b <= 8:
                y = stq1.gemv_noalloc(wd, _bf16(x), n, k).cpu().numpy()
                _close(y, ref, bound, f"gemv_noalloc n={n} k={k} b={b}")
                _clean(f"gemv_noalloc n={n} k={k} b={b}")


def _bank(E, n, k, seed):
    mats = [oracle.encode_plain(workloads.gaussian_matrix(n, k, 0.03, seed=seed + e)) for e in range(E)]
    return mats, _dev(np.concatenate(mats))


def check_moe_gateup():
    # N = 518: expert e starts at row 518 e, inside a super-row for odd e.
    E, n, k, topk = 6, 518, 1536, 3
    mats, bank = _bank(E, n, k, 300)
    for T in (7, 40, 300):
        x = workloads.activations_bf16(T, k, seed=T)
        ids = workloads.zipf_topk_ids(T, E, topk, seed=T + 1)
        wts = workloads.softmax_route_weights(T, topk, seed=T + 2)
        for flags in (0, stq1.MOE_WEIGHT_UP):
            for path in (stq1.PATH_AUTO, stq1.PATH_TABLE, stq1.PATH_MMA, stq1.PATH_TILES):
                stq1.set_path(path)
                try:
                    y = stq1.moe_gateup(bank, _bf16(x), _dev(ids), _dev(wts), n, k, E, flags=flags).cpu().numpy()
                finally:
                    stq1.set_path(stq1.PATH_AUTO)
                ref, bound = oracle.moe_gateup(mats, x, ids, wts, n, k, flags=flags, abs_sum=True)
                _close(y, ref, bound, f"moe T={T} flags={flags} path={path}")
                _clean(f"moe T={T} flags={flags} path={path}")
        # fp8 variant (tile kernel) against the oracle's fp8 reading
        y = stq1.moe_gateup(bank, _bf16(x), _dev(ids), _dev(wts), n, k, E, flags=stq1.MOE_FP8).cpu().numpy()
        ref, bound = oracle.moe_gateup_fp8(mats, x, ids, wts, n, k, abs_sum=True)
        if T >= 40:                                     # fewer pairs than that take the bf16 decode paths
            _close(y, ref, bound, f"moe fp8 T={T}")
        _clean(f"moe fp8 T={T}")


def check_expert_parallel():
    E, n, hidden, topk = 6, 1024, 512, 3
    gu = [oracle.encode_plain(workloads.gaussian_matrix(n, hidden, 0.05, seed=400 + e)) for e in range(E)]
    dn = [oracle.encode_plain(workloads.gaussian_matrix(hidden, n // 2, 0.05, seed=500 + e)) for e in range(E)]
    for T in (9, 200):
        x = workloads.activations_bf16(T, hidden, seed=T + 7)
        ids = workloads.zipf_topk_ids(T, E, topk, seed=T + 8)
        wts = workloads.softmax_route_weights(T, topk, seed=T + 9)
        ref, scale = oracle.moe_ffn(gu, dn, x, ids, wts, n, hidden, abs_sum=True)
        # compact rank shares, summed here
        world = 2
        total = torch.zeros((T, hidden), dtype=torch.float32, device="cuda")
        for r in range(world):
            b, c = expert_range(E, world, r)
            total += stq1.moe_ffn_local(_dev(np.concatenate(gu[b:b + c])), _dev(np.concatenate(dn[b:b + c])),
                                        _bf16(x), _dev(ids), _dev(wts), n, hidden, c, b)
        _clean(f"moe_ffn_local T={T}")
        bound = oracle.tolerance(scale) + (world - 1) * (1e-6 + 2.0 ** -24 * (scale + 1e-6 * world))
        assert np.all(np.abs(total.cpu().numpy().astype(np.float64) - ref) <= bound), f"ranks T={T}"
        # token dispatch: every rank's pairs grouped by owner, computed as one-slot
        # tokens by the owner, returned in send order and combined per token
        sent = []
        for r in range(world):
            t0, tc = row_range(T, world, r)
            order, inv, counts, local, xs, ws = stq1.ep_dispatch(_dev(ids[t0:t0 + tc]), _bf16(x[t0:t0 + tc]),
                                                                 _dev(wts[t0:t0 + tc]), E, world)
            sent.append((np.concatenate([[0], np.cumsum(counts.cpu().numpy()[:world])]), local, xs, ws, inv, tc))
        _clean(f"ep_dispatch T={T}")
        back = [[None] * world for _ in range(world)]
        for q in range(world):
            b, c = expert_range(E, world, q)
            rx = torch.cat([s[2][s[0][q]:s[0][q + 1]] for s in sent])
            rid = torch.cat([s[1][s[0][q]:s[0][q + 1]] for s in sent])
            rw = torch.cat([s[3][s[0][q]:s[0][q + 1]] for s in sent])
            res = stq1.moe_ffn_local(_dev(np.concatenate(gu[b:b + c])), _dev(np.concatenate(dn[b:b + c])), rx,
                                     rid.view(-1, 1), rw.view(-1, 1), n, hidden, c, 0)
            pos = 0
            for r in range(world):
                m = int(sent[r][0][q + 1] - sent[r][0][q])
                back[r][q] = res[pos:pos + m]
                pos += m
        out = torch.cat([stq1.ep_combine(torch.cat(back[r]), sent[r][4], sent[r][5], topk) for r in range(world)])
        _clean(f"ep exchange T={T}")
        bound = oracle.tolerance(scale) + topk * (1e-6 + 2.0 ** -24 * (scale + 1e-6 * topk))
        assert np.all(np.abs(out.cpu().numpy().astype(np.float64) - ref) <= bound), f"exchange T={T}"


def main():
    assert torch.cuda.is_available()
    check_build_and_selftest()
    check_gemv()
    check_moe_gateup()
    check_expert_parallel()
    print("OK")


if __name__ == "__main__":
    main()
