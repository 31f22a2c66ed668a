"""Host-side load-balancing planner (libbsa, no GPU) against the brute-force oracle."""
import numpy as np
import pytest

import oracle.rlb as orlb


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_top_b200 import build
    build.build()
    import block_sparse_attention_top_b200 as m
    return m


def _case(rng, R, hmin=1, hmax=3):
    owner = []
    for r in range(R):
        owner += [r] * int(rng.integers(hmin, hmax + 1))
    L_h = rng.uniform(0.5, 20.0, size=len(owner)).astype(np.float32)
    return L_h, owner


@pytest.mark.parametrize("seed", range(40))
def test_planner_matches_brute_force_objective(bsa, seed):
    rng = np.random.default_rng(seed)
    R = int(rng.integers(1, 6))
    L_h, owner = _case(rng, R)
    moves, L_new, rho_b, rho_a = bsa.bsa_rlb_plan(L_h, owner, R)
    (mx, var), _, _ = orlb.best_plan(L_h.astype(np.float64), owner, R)
    L_new = L_new.numpy().astype(np.float64)
    assert L_new.max() == pytest.approx(mx, rel=1e-5)
    assert L_new.var() == pytest.approx(var, rel=1e-4, abs=1e-4)
    # a valid plan: one send and one receive per rank, pair swaps, Eq. 5 loads
    base = orlb.rank_loads(L_h.astype(np.float64), owner, R)
    sends, recvs = [m[0] for m in moves], [m[1] for m in moves]
    assert len(set(sends)) == len(sends) and len(set(recvs)) == len(recvs) and sorted(sends) == sorted(recvs)
    expect = base.copy()
    for src, dst, h in moves:
        assert owner[h] == src
        expect[src] -= L_h[h]
        expect[dst] += L_h[h]
    assert np.allclose(L_new, expect, rtol=1e-5)
    assert rho_b == pytest.approx(orlb.rho(base), rel=1e-5) and rho_a <= rho_b * (1 + 1e-6)


def test_eight_ranks_five_heads_is_fast_and_deterministic(bsa):
    import time
    rng = np.random.default_rng(7)
    L_h = rng.gamma(2.0, 5.0, size=40).astype(np.float32)
    owner = [h // 5 for h in range(40)]
    t = time.perf_counter()
    a = bsa.bsa_rlb_plan(L_h, owner, 8)
    assert time.perf_counter() - t < 2.0
    b = bsa.bsa_rlb_plan(L_h, owner, 8)
    assert a[0] == b[0] and np.array_equal(a[1].numpy(), b[1].numpy())
    assert a[3] <= a[2]


def test_planner_errors_and_policy(bsa):
    assert bsa._lib.bsa_rlb_plan(13, 0, None, None, None, None, None, None, None) == bsa.BSA_EINVAL
    L_h = np.ones(13, dtype=np.float32)
    with pytest.raises(bsa.BsaError):
        bsa.bsa_rlb_plan(L_h, list(range(13)), 13)
    with pytest.raises(bsa.BsaError):
        bsa.bsa_rlb_plan([1.0, -1.0], [0, 1], 2)
    for rho in (1.0, 1.049, 1.05, 1.099, 1.1, 1.34):
        assert bsa.bsa_balance_policy(rho) == orlb.policy(rho)
    assert bsa.bsa_balance_policy(1.2, 1.2, 1.1) == bsa.BSA_EINVAL


def test_gain_model_matches_oracle(bsa):
    rng = np.random.default_rng(5)
    for _ in range(20):
        R = int(rng.integers(1, 9))
        L = rng.uniform(0, 20, R).astype(np.float32)
        Ln = rng.uniform(0, 20, R).astype(np.float32)
        c, P, C = (float(v) for v in rng.uniform(0, 3, 3))
        K, G = bsa.bsa_rlb_gain(L, Ln, c, P, C)
        Ko, Go = orlb.gain(L.astype(np.float64), Ln.astype(np.float64), c=c, P=P, C=C)
        assert K == pytest.approx(Ko, rel=1e-12, abs=1e-12) and G == pytest.approx(Go, rel=1e-12, abs=1e-12)
        # the joint model of Eq. 11 subtracts the augmentation cost A as well
        assert bsa.bsa_rlb_gain(L, Ln, c, P, C, A=0.25)[1] == pytest.approx(Go - 0.25, abs=1e-12)
    with pytest.raises(bsa.BsaError):
        bsa.bsa_rlb_gain([1.0, -2.0], [1.0, 1.0], 1.0)


@pytest.mark.parametrize("seed", range(10))
def test_rank_loads_match_oracle(bsa, seed):
    """Eq. 1 per-rank loads, Eq. 2 rho and head counts of a random placement."""
    rng = np.random.default_rng(100 + seed)
    R = int(rng.integers(1, 9))
    L_h, owner = _case(rng, R, hmin=0, hmax=4)
    owner = list(rng.permutation(owner))
    L_r, rho, cnt = bsa.bsa_rank_loads(L_h, owner, R)
    want = orlb.rank_loads(L_h.astype(np.float64), owner, R)
    np.testing.assert_allclose(L_r.numpy(), want, rtol=1e-6)
    if want.sum() > 0:
        assert rho == pytest.approx(orlb.rho(want), rel=1e-6)
    assert cnt.tolist() == [owner.count(r) for r in range(R)]


def test_rank_loads_errors(bsa):
    with pytest.raises(bsa.BsaError):
        bsa.bsa_rank_loads([1.0, 2.0], [0, 3], 2)          # rank outside [0, R)
    with pytest.raises(bsa.BsaError):
        bsa.bsa_rank_loads([1.0, -2.0], [0, 1], 2)         # negative workload
    L_r, rho, cnt = bsa.bsa_rank_loads([0.0, 0.0], [0, 1], 2)
    assert rho == 1.0 and cnt.tolist() == [1, 1]
