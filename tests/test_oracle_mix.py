"""Pins of the mixed-precision allocation oracle (no GPU).

The pages pick each layer's format by full-Hessian sensitivity, greedily by
error reduction per added byte, between STQ1_0 and a 2.06-bpw partner format
("AngelSlim Shrinks ..." bullet list; lemmy.durstig.online post 66506,
"Full-Hessian scoring").  The partner here is STQ2, this library's 2-bit
format at the same rate.  Each check ties the oracle to something outside it:
hand-built blocks with known codes and ties, tr(D H D^T) written out with H
formed explicitly, the diagonal form when calibration columns are orthogonal,
and brute force over all layer subsets where greedy is optimal.
"""

import itertools

import numpy as np
import pytest

import oracle
import workloads


# ---------------------------------------------------------------------------
# STQ2 storage
# ---------------------------------------------------------------------------


def test_stq2_rate_is_the_partner_formats():
    # 66 bytes per 256 weights = 2.0625 bits per weight, the partner format's rate
    assert oracle.STQ2_BLOCK_BYTES * 8 / 256 == 2.0625


def test_stq2_hand_built_block():
    # amax 3.0 (an fp16 value) puts the levels at -3, -1, 1, 3 (codes 0..3)
    w = np.tile(np.array([-3.0, -1.0, 1.0, 3.0], np.float32), 64)
    b = oracle.encode_stq2(w.reshape(1, 256))
    assert b[0] == 0x00 and b[1] == 0x42                      # fp16(3.0) = 0x4200, little-endian
    assert np.all(b[2:] == 0b11100100)                        # codes 0,1,2,3 from the low bits up
    assert np.array_equal(oracle.decode_stq2(b, 1, 256), w.reshape(1, 256).astype(np.float64))


def test_stq2_ties_take_the_lower_code():
    # 0.0 is midway between -1 and 1, 2.0 between 1 and 3, -2.0 between -3 and -1
    w = np.zeros(256, np.float32)
    w[0] = 3.0
    w[1], w[2], w[3] = 0.0, 2.0, -2.0
    b = oracle.encode_stq2(w.reshape(1, 256))
    assert b[2] == (3 | (1 << 2) | (2 << 4) | (0 << 6))
    # the rest are 0.0: code 1 (level -1)
    assert np.all(b[3:] == 0b01010101)


def test_stq2_all_zero_block_decodes_to_zero():
    b = oracle.encode_stq2(np.zeros((2, 256), np.float32))
    assert np.all(b[[0, 1, 66, 67]] == 0)
    assert np.all(oracle.decode_stq2(b, 2, 256) == 0.0)


def test_stq2_error_is_within_half_a_level_step():
    w = workloads.expert_like_matrix(16, 1024, seeds=(11, 12, 13))
    b = oracle.encode_stq2(w)
    wh = oracle.decode_stq2(b, 16, 1024)
    d = oracle.fp16_value(b.reshape(-1, 66)[:, 0].astype(np.uint16) | (b.reshape(-1, 66)[:, 1].astype(np.uint16) << 8))
    amax = np.max(np.abs(w.reshape(-1, 256)), axis=1).astype(np.float64)
    err = np.abs(w.reshape(-1, 256).astype(np.float64) - wh.reshape(-1, 256))
    # levels are 2d/3 apart inside [-d, d]; beyond it the clipped part |amax - d| adds
    bound = d / 3.0 + np.abs(amax - d) + 1e-12
    assert np.all(err <= bound[:, None])
    # and each weight sits at its nearest level: no other level is strictly closer
    levels = d[:, None] * (2.0 * np.arange(4) - 3.0)[None, :] / 3.0
    all_d = np.abs(w.reshape(-1, 256, 1).astype(np.float64) - levels[:, None, :])
    assert np.all(err <= all_d.min(axis=2) + 0.0)


def test_stq2_beats_stq1_on_gaussian_weights():
    # two bits per weight resolve more than the one-zero ternary pattern
    w = workloads.gaussian_matrix(8, 2048, 0.02, seed=5)
    e2 = np.sum((w - oracle.decode_stq2(oracle.encode_stq2(w), 8, 2048)) ** 2)
    p1 = oracle.encode_plain(w)
    e1 = np.sum((w - oracle.decode(p1, 8, 2048)) ** 2)
    assert e2 < 0.6 * e1


def test_stq2_wls_scale_is_the_weighted_least_squares_minimiser():
    # against a library least-squares solve of the sqrt(h)-weighted system
    rng = np.random.default_rng(21)
    wb = rng.standard_normal((5, 256)) * 0.02
    hb = rng.uniform(0.0, 4.0, (5, 256))
    q = rng.integers(0, 4, (5, 256))
    got = oracle.stq2_wls_scale(wb, hb, q)
    for b in range(5):
        a = (np.sqrt(hb[b]) * (2.0 * q[b] - 3.0) / 3.0)[:, None]
        want = np.linalg.lstsq(a, np.sqrt(hb[b]) * wb[b], rcond=None)[0][0]
        assert got[b] == pytest.approx(want, rel=1e-12)


def test_stq2_fit_never_increases_the_weighted_error():
    w = workloads.expert_like_matrix(8, 1024, seeds=(31, 32, 33))
    h = workloads.calibration_importance(1024, seed=34)
    _, tr = oracle.encode_stq2(w, h, rounds=5, trace=True)
    wb = w.reshape(-1, 256).astype(np.float64)
    hb = tr["h_blocks"]
    errs = [oracle.stq2_weighted_error(wb, hb, d, q) for d, q in tr["rounds"]]
    for a, b in zip(errs, errs[1:]):
        assert np.all(b <= a * (1 + 1e-12) + 1e-300)
    assert np.sum(errs[-1]) < 0.95 * np.sum(errs[0])


def test_stq2_fit_follows_the_important_columns():
    # one large weight on an unimportant column sets amax; the fit shrinks d
    # towards the small weights that carry the importance
    w = np.full((1, 256), 0.01, np.float32)
    w[0, 0] = 1.0
    h = np.ones(256, np.float32)
    h[0] = 1e-6
    plain = oracle.encode_stq2(w)
    fitted = oracle.encode_stq2(w, h, rounds=3)
    d_plain = oracle.fp16_value(plain[0] | (np.uint16(plain[1]) << 8))
    d_fit = oracle.fp16_value(fitted[0] | (np.uint16(fitted[1]) << 8))
    assert d_plain == oracle.fp16_value(oracle.fp16_bits(1.0))
    assert d_fit < 0.1
    err = lambda p: float(np.sum(h * (w[0] - oracle.decode_stq2(p, 1, 256)[0]) ** 2))
    assert err(fitted) < 0.01 * err(plain)


def test_stq2_zero_importance_block_uses_unit_weights():
    w = workloads.gaussian_matrix(2, 512, 0.02, seed=8)
    h = np.ones(512, np.float32)
    h[:256] = 0.0
    a = oracle.encode_stq2(w, h, rounds=2)
    b = oracle.encode_stq2(w, np.ones(512, np.float32), rounds=2)
    assert np.array_equal(a.reshape(2, 2, 66)[:, 0], b.reshape(2, 2, 66)[:, 0])


# ---------------------------------------------------------------------------
# Layer error under the full and the diagonal Hessian
# ---------------------------------------------------------------------------


def _brute_force_error(w, wh, x):
    """The definition, as loops: H_kl = sum_c x_ck x_cl, then sum_j sum_k sum_l D_jk H_kl D_jl."""
    n, k = w.shape
    h = [[sum(float(x[c, a]) * float(x[c, b]) for c in range(x.shape[0])) for b in range(k)] for a in range(k)]
    total = 0.0
    for j in range(n):
        for a in range(k):
            for b in range(k):
                total += (float(w[j, a]) - float(wh[j, a])) * h[a][b] * (float(w[j, b]) - float(wh[j, b]))
    return total


def test_hessian_error_equals_the_trace_definition():
    rng = np.random.default_rng(3)
    w = rng.standard_normal((3, 8))
    wh = rng.standard_normal((3, 8))
    x = rng.standard_normal((5, 8))
    got = oracle.hessian_error(w, wh, x)
    want = _brute_force_error(w, wh, x)
    assert got == pytest.approx(want, rel=1e-12)


def test_hessian_error_is_not_symmetric_in_the_operands_shapes():
    # D H D^T uses H over the input dimension: transposing D would need H over rows
    rng = np.random.default_rng(4)
    w = rng.standard_normal((2, 6))
    x = rng.standard_normal((9, 6)) @ rng.standard_normal((6, 6))       # correlated columns
    got = oracle.hessian_error(w, np.zeros_like(w), x)
    assert got == pytest.approx(float(np.sum((x @ w.T) ** 2)), rel=1e-12)


def test_diagonal_equals_full_for_orthogonal_columns():
    # x^T x diagonal (orthogonal calibration columns): the imatrix score is exact
    rng = np.random.default_rng(6)
    w = rng.standard_normal((4, 7))
    q, _ = np.linalg.qr(rng.standard_normal((7, 7)))
    x = q.T * rng.uniform(0.5, 2.0, size=7)[None, :]        # rows: x^T x = diag(scales^2)
    wh = np.zeros_like(w)
    assert oracle.diagonal_error(w, wh, x) == pytest.approx(oracle.hessian_error(w, wh, x), rel=1e-10)


def test_diagonal_misses_correlation():
    # two identical calibration columns and a difference with opposite signs on them:
    # the full score sees the cancellation, the diagonal one does not
    x = np.array([[1.0, 1.0], [2.0, 2.0]])
    w = np.array([[1.0, -1.0]])
    wh = np.zeros_like(w)
    assert oracle.hessian_error(w, wh, x) == 0.0
    assert oracle.diagonal_error(w, wh, x) == pytest.approx(10.0)


def test_errors_vanish_without_a_difference_and_scale_quadratically():
    rng = np.random.default_rng(7)
    w = rng.standard_normal((3, 10))
    x = rng.standard_normal((4, 10))
    assert oracle.hessian_error(w, w, x) == 0.0
    wh = w + rng.standard_normal((3, 10)) * 0.1
    e = oracle.hessian_error(w, wh, x)
    assert oracle.hessian_error(w, w + 2.0 * (wh - w), x) == pytest.approx(4.0 * e, rel=1e-12)
    assert oracle.hessian_error(w, wh, 3.0 * x) == pytest.approx(9.0 * e, rel=1e-12)


# ---------------------------------------------------------------------------
# Greedy allocation by error reduction per added byte
# ---------------------------------------------------------------------------


def _best_subset(el, eh, bl, bh, budget):
    best, best_pick = None, None
    n = len(el)
    for r in range(n + 1):
        for sub in itertools.combinations(range(n), r):
            cost = sum(bl) + sum(bh[i] - bl[i] for i in sub)
            if cost > budget:
                continue
            err = sum(eh[i] if i in sub else el[i] for i in range(n))
            if best is None or err < best - 1e-12:
                best, best_pick = err, set(sub)
    return best, best_pick


def test_greedy_is_optimal_when_layers_cost_the_same():
    # equal byte costs: the best k layers by error reduction are the optimum
    rng = np.random.default_rng(8)
    for trial in range(20):
        n = 7
        el = rng.uniform(1.0, 5.0, n)
        eh = el * rng.uniform(0.1, 0.9, n)
        bl = np.full(n, 42.0)
        bh = np.full(n, 66.0)
        budget = 42.0 * n + 24.0 * rng.integers(0, n + 1)
        pick = oracle.greedy_allocate(el, eh, bl, bh, budget)
        best, _ = _best_subset(el, eh, bl, bh, budget)
        got = float(np.sum(np.where(pick, eh, el)))
        assert got == pytest.approx(best, rel=1e-12)
        assert np.sum(np.where(pick, bh, bl)) <= budget


def test_greedy_orders_by_reduction_per_byte_not_by_reduction():
    # layer 0 saves more in total, layer 1 more per byte; the budget fits either
    # upgrade but not both, so the order decides
    el = [10.0, 4.0]
    eh = [4.0, 1.0]          # reductions 6 and 3
    bl = [100.0, 10.0]
    bh = [200.0, 20.0]       # costs 100 and 10: 0.06 and 0.3 per byte
    pick = oracle.greedy_allocate(el, eh, bl, bh, budget=110.0 + 100.0)
    assert list(pick) == [False, True]


def test_greedy_skips_a_layer_that_does_not_fit_and_takes_a_later_one():
    el = [10.0, 10.0, 10.0]
    eh = [0.0, 5.0, 8.0]
    bl = [10.0, 10.0, 10.0]
    bh = [30.0, 20.0, 11.0]          # per byte: 0.5, 0.5, 2.0
    pick = oracle.greedy_allocate(el, eh, bl, bh, budget=30.0 + 12.0)
    # order: layer 2 (2.0), then the tie 0 / 1 by index: 0 needs 20 (no room), 1 needs 10 (fits)
    assert list(pick) == [False, True, True]


def test_greedy_never_upgrades_a_layer_that_gets_worse():
    pick = oracle.greedy_allocate([1.0, 2.0], [1.5, 1.0], [1.0, 1.0], [2.0, 2.0], budget=100.0)
    assert list(pick) == [False, True]


def test_greedy_budget_extremes():
    el, eh = [3.0, 2.0, 1.0], [1.0, 1.0, 0.5]
    bl, bh = [10.0] * 3, [16.0] * 3
    assert not oracle.greedy_allocate(el, eh, bl, bh, budget=30.0).any()
    assert oracle.greedy_allocate(el, eh, bl, bh, budget=48.0).all()


@pytest.mark.parametrize("mistake", ["diagonal_for_full", "gain_without_bytes", "stq2_levels_by_half",
                                     "stq2_fit_unweighted"])
def test_planted_mix_mistakes_are_caught(monkeypatch, mistake):
    import oracle.stq1 as o

    def passes():
        try:
            test_stq2_hand_built_block()
            test_hessian_error_equals_the_trace_definition()
            test_diagonal_misses_correlation()
            test_greedy_orders_by_reduction_per_byte_not_by_reduction()
            test_stq2_wls_scale_is_the_weighted_least_squares_minimiser()
        except AssertionError:
            return False
        return True

    assert passes()

    def plant(name, fn):
        monkeypatch.setattr(o, name, fn)
        monkeypatch.setattr(oracle, name, fn)

    if mistake == "diagonal_for_full":
        plant("hessian_error", o.diagonal_error)
    elif mistake == "gain_without_bytes":
        def by_reduction(el, eh, bl, bh, budget):
            el, eh, bl, bh = (np.asarray(v, float) for v in (el, eh, bl, bh))
            pick, total = np.zeros(len(el), bool), float(np.sum(bl))
            for i in sorted(range(len(el)), key=lambda i: (-(el[i] - eh[i]), i)):
                if el[i] - eh[i] > 0 and total + bh[i] - bl[i] <= budget:
                    pick[i], total = True, total + bh[i] - bl[i]
            return pick
        plant("greedy_allocate", by_reduction)
    elif mistake == "stq2_fit_unweighted":
        orig_wls = o.stq2_wls_scale
        plant("stq2_wls_scale", lambda wb, hb, q: orig_wls(wb, np.ones_like(hb), q))
    elif mistake == "stq2_levels_by_half":
        orig_dec = o.decode_stq2
        plant("decode_stq2", lambda p, n, k: orig_dec(p, n, k) * 1.5)
    assert not passes()
