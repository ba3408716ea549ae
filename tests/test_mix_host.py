"""Host-side greedy allocation (stq1_mix_allocate) against the oracle (no GPU).

The allocator is plain fp64 host code with a fixed evaluation order; on the
same numbers it must pick exactly the layers the oracle's greedy picks,
including ties and layers that do not fit.
"""

import numpy as np
import pytest

import oracle
import sub_bit_sparse_b200 as stq1


def test_allocator_matches_oracle_on_random_cases():
    rng = np.random.default_rng(2024)
    for trial in range(400):
        n = int(rng.integers(1, 80))
        el = rng.uniform(0.0, 10.0, n)
        eh = el * rng.uniform(0.2, 1.3, n)          # some upgrades make a layer worse
        if trial % 3 == 0:                           # exact ties in the gains
            el, eh = np.round(el), np.round(eh)
        bl = rng.choice([42.0, 66.0, 100.0], n)
        bh = bl + rng.choice([24.0, 24.0, 50.0], n)
        budget = float(np.sum(bl) + rng.uniform(-0.1, 1.1) * np.sum(bh - bl))
        got = stq1.mix_allocate(el, eh, bl, bh, budget)
        assert np.array_equal(got, oracle.greedy_allocate(el, eh, bl, bh, budget)), trial


def test_allocator_pages_split():
    # 77 equal layers and the budget of 48 upgrades: the 48 largest reductions win
    rng = np.random.default_rng(77)
    el = rng.uniform(1.0, 2.0, 77)
    eh = el * rng.uniform(0.3, 0.7, 77)
    bl, bh = np.full(77, 42.0), np.full(77, 66.0)
    pick = stq1.mix_allocate(el, eh, bl, bh, 29 * 42.0 + 48 * 66.0)
    assert pick.sum() == 48
    red = el - eh
    assert red[pick].min() >= red[~pick].max()


@pytest.mark.parametrize("case", ["nan", "inf_budget", "no_extra_bytes", "empty"])
def test_allocator_rejects_bad_input(case):
    el, eh, bl, bh = np.ones(3), np.zeros(3), np.full(3, 42.0), np.full(3, 66.0)
    budget = 1000.0
    if case == "nan":
        el[1] = np.nan
    elif case == "inf_budget":
        budget = np.inf
    elif case == "no_extra_bytes":
        bh[2] = 42.0
    elif case == "empty":
        el = eh = bl = bh = np.zeros(0)
    with pytest.raises(stq1.Stq1Error):
        stq1.mix_allocate(el, eh, bl, bh, budget)
