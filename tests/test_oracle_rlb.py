"""Pins for the RLB oracle: hand-worked plans, Eq. 1-2 and 5, enumeration counts."""
import numpy as np
import pytest

import oracle.rlb as rlb


def test_matching_count_is_the_involution_number():
    # disjoint pair sets on R points: 1, 1, 2, 4, 10, 26, 76, 232, 764
    assert [sum(1 for _ in rlb.matchings(R)) for R in range(9)] == [1, 1, 2, 4, 10, 26, 76, 232, 764]


def test_hand_worked_two_ranks():
    # rank 0 holds heads {0: 9, 1: 1}, rank 1 holds {2: 3, 3: 2}: L = [10, 5]
    L_h = [9.0, 1.0, 3.0, 2.0]
    owner = [0, 0, 1, 1]
    assert list(rlb.rank_loads(L_h, owner, 2)) == [10.0, 5.0]
    assert rlb.rho([10.0, 5.0]) == pytest.approx(10 / 7.5)
    (mx, var), moves, L = rlb.best_plan(L_h, owner, 2)
    # every swap raises the maximum: (0<->2) -> [4, 11], (0<->3) -> [3, 12],
    # (1<->2) -> [12, 3], (1<->3) -> [11, 4]; the empty plan keeps [10, 5]
    assert mx == 10.0 and moves == [] and list(L) == [10.0, 5.0]


def test_hand_worked_three_ranks():
    L_h = [6.0, 5.0, 1.0, 1.0, 2.0, 2.0]
    owner = [0, 0, 1, 1, 2, 2]              # L = [11, 2, 4]
    (mx, var), moves, L = rlb.best_plan(L_h, owner, 3)
    # swap head 0 (6) with a 1 on rank 1 -> [6, 7, 4]; with a 2 on rank 2 -> [7, 2, 8];
    # head 1 (5) with a 1 on rank 1 -> [7, 6, 4]; with a 2 -> [8, 2, 7]  => best max 7: [6,7,4] (var 1.556) vs
    # [7,6,4] (var 1.556): equal -- the enumeration keeps the first found
    assert mx == 7.0
    assert sorted(L) == [4.0, 6.0, 7.0]
    assert len(moves) == 2 and {m[0] for m in moves} == {0, 1}


def test_eq5_post_loads_and_one_send_one_receive():
    rng = np.random.default_rng(0)
    for _ in range(20):
        R = int(rng.integers(2, 5))
        owner = sorted(list(range(R)) * 2)
        L_h = rng.uniform(0, 10, size=len(owner))
        base = rlb.rank_loads(L_h, owner, R)
        for moves, L in rlb.plans(L_h, owner, R):
            sends = [m[0] for m in moves]
            recvs = [m[1] for m in moves]
            assert len(set(sends)) == len(sends) and len(set(recvs)) == len(recvs)
            expect = base.copy()
            for src, dst, h in moves:
                expect[src] -= L_h[h]
                expect[dst] += L_h[h]
            assert np.allclose(L, expect) and np.isclose(L.sum(), base.sum())


def test_gain_and_policy():
    K, G = rlb.gain([10.0, 5.0, 6.0], [7.0, 7.0, 7.0], c=2.0, P=1.0, C=0.5)
    assert K == 6.0 and G == 4.5
    assert [rlb.policy(x) for x in (1.0, 1.049, 1.05, 1.099, 1.10, 1.34)] == [0, 0, 1, 1, 2, 2]
