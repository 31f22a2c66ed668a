"""Pins for the SASA oracle: Eq. 7-10 by hand, invariants of the augmentation."""
import numpy as np
import pytest

import oracle
import oracle.sasa as sasa
import synthetic as syn


def test_eq7_to_10_hand_example():
    # L_r = [10, 8, 9.5, 5]: L_max = 10, dL = [0, 2, 0.5, 5]; trigger 0.07*10 = 0.7
    r = sasa.budget([10.0, 8.0, 9.5, 5.0], n1=0.8, n2=0.07, S=0.25)
    assert np.allclose(r["dL"], [0, 2, 0.5, 5])
    assert np.allclose(r["B"], [0, 1.6, 0, 4.0])          # 0.5 <= 0.7: not triggered
    assert np.allclose(r["L_aug"], [10, 9.6, 9.5, 9.0])
    assert r["A"] == pytest.approx(0.25)                   # no new critical path: only the fixed cost S


def test_budget_never_exceeds_slack():
    rng = np.random.default_rng(0)
    for _ in range(100):
        L = rng.uniform(1, 20, size=rng.integers(2, 9))
        r = sasa.budget(L, n1=rng.uniform(0, 1), n2=rng.uniform(0, 0.2))
        assert np.all(r["B"] <= r["dL"] + 1e-12) and r["A"] == pytest.approx(0.0)
        assert np.all((r["B"] == 0) | (r["dL"] > 0))


def test_extra_per_head_splits_rank_budgets():
    assert list(sasa.extra_per_head([0.0, 7.9, 2.0], [2, 3, 1])) == [0, 0, 2, 2, 2, 2]


@pytest.mark.parametrize("extra", [[0, 0], [3, 0], [1, 5], [100, 100]])
def test_augmentation_nests_and_grows_L(extra):
    w = syn.workload(2, T=2, Hs=16, Ws=32, H=2, block=64)
    x = syn.make_inputs(w, seed=3)
    r = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, 0.6, 1)
    n_out, rp, ci, L_h = sasa.augment(r, extra, w.nb)
    assert np.all(n_out == np.minimum(w.nb, r.counts + np.repeat(extra, w.nb)))
    for row in range(w.rows):
        old = r.col_idx[r.row_ptr[row]:r.row_ptr[row + 1]]
        new = ci[rp[row]:rp[row + 1]]
        assert list(new[:old.size]) == list(old)            # the routed prefix is kept as is
        P = r.P[row][new]
        assert np.all(P[1:] <= P[:-1] * (1 + 1e-12))       # appended blocks follow importance order
    assert np.allclose(L_h, np.minimum(w.nb, r.counts + np.repeat(extra, w.nb)).reshape(2, -1).mean(axis=1))
