"""Pins for the routing oracle: worked example, closed forms, invariants, brute force."""
import json
import math
import os

import numpy as np
import pytest

import oracle
import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _worked_inputs(ex):
    sh = ex["shape"]
    N = sh["T"] * sh["Hs"] * sh["Ws"]
    q = np.zeros((1, N, 1, sh["d"]), np.float32)
    k = np.zeros_like(q)
    ones = np.ones(4)
    dq = 0.25 * np.array([1, 1, -1, -1])
    dk = 0.25 * np.array([1, -1, 1, -1])
    for blk, toks in enumerate(ex["hilbert_blocks_raster_tokens"]):
        c, x = ex["design"]["c"][blk], ex["design"]["x"][blk]
        q[0, toks[0], 0] = c * ones + dq
        q[0, toks[1], 0] = c * ones - dq
        k[0, toks[0], 0] = x * ones + dk
        k[0, toks[1], 0] = x * ones - dk
    return sh, q, k


def test_worked_example():
    ex = json.load(open(os.path.join(GOLDEN, "route_worked_example.json")))
    sh, q, k = _worked_inputs(ex)
    perm = oracle.token_perm(sh["T"], sh["Hs"], sh["Ws"])
    assert [list(perm[i:i + 2]) for i in range(0, 8, 2)] == ex["hilbert_blocks_raster_tokens"]
    for case in ex["cases"]:
        r = oracle.route(q, k, sh["T"], sh["Hs"], sh["Ws"], sh["block"], case["p"], case["k_floor"])
        assert list(r.ambiguous) == case["ambiguous"], case
        for i, want in enumerate(case["sets"]):
            got = list(r.col_idx[r.row_ptr[i]:r.row_ptr[i + 1]])
            if not case["ambiguous"][i]:
                assert got == want, (case, i)
                assert r.n_p[i] == case["n_p"][i]
            else:
                assert abs(len(got) - len(want)) <= 1
        if not any(case["ambiguous"]):
            assert r.L_h[0] == np.float32(case["L_h"])
        assert r.L_h[0] == np.float32(r.counts.sum()) / np.float32(4)
    # pooled means and scaled scores as derived by hand
    r = oracle.route(q, k, 1, 2, 4, 2, 0.7, 1)
    c = np.array(ex["design"]["c"])
    x = np.array(ex["design"]["x"], np.float32).astype(np.float64)
    assert np.allclose(r.qbar[0], c[:, None] * np.ones(4), atol=1e-7)
    assert np.allclose(r.scores[0], np.outer(c, 2 * x), atol=1e-6)


def test_constant_blocks_pool_to_their_value_and_tail_uses_real_count():
    T, Hs, Ws, block, d = 1, 3, 5, 4, 8          # N = 15 -> blocks of 4,4,4,3
    perm = oracle.token_perm(T, Hs, Ws)
    x = np.zeros((15, d), np.float32)
    vals = np.array([1.5, -2.0, 0.25, 7.0])
    for i in range(4):
        x[perm[i * block:(i + 1) * block]] = vals[i]
    pooled = oracle.pool_head(x, perm, block)
    assert np.array_equal(pooled, np.repeat(vals[:, None], d, axis=1))
    # tail mean over 3 real tokens: 1,2,3 -> 2
    x[perm[12:15], 0] = [1.0, 2.0, 3.0]
    assert oracle.pool_head(x, perm, block)[3, 0] == 2.0
    assert list(oracle.block_counts(15, 4)) == [4, 4, 4, 3]


def _tiny():
    w = syn.workload(1)
    return w, syn.make_inputs(w)


def test_p_one_keeps_everything():
    w, x = _tiny()
    r = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, 1.0, 0)
    assert np.all(r.counts == w.nb) and r.nnz == w.rows * w.nb
    assert np.all(r.L_h == np.float32(w.nb))
    for row in range(w.rows):
        assert sorted(r.col_idx[r.row_ptr[row]:r.row_ptr[row + 1]]) == list(range(w.nb))


@pytest.mark.parametrize("k_floor", [0, 1, 2, 5, 16, 40])
def test_floor_invariant(k_floor):
    w, x = _tiny()
    r = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, 0.3, k_floor)
    assert np.all(r.counts >= min(k_floor, w.nb)) and np.all(r.counts <= w.nb)
    assert np.all(r.counts == np.minimum(w.nb, np.maximum(k_floor, r.n_p)))


def test_monotone_and_nested_in_p():
    w, x = _tiny()
    prev = None
    for p in (0.5, 0.8, 0.9, 0.95, 0.99, 1.0):
        r = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, p, 2)
        sets = [set(r.col_idx[r.row_ptr[i]:r.row_ptr[i + 1]]) for i in range(w.rows)]
        if prev is not None:
            assert np.all(r.counts >= prev[0])
            assert all(a <= b for a, b in zip(prev[1], sets))
        prev = (r.counts, sets)


def test_uniform_row_keeps_ceil_p_nb():
    nb = 16
    for p in (0.3, 0.5, 0.9, 0.95):
        P, order, Ps, n_p, n_i, amb = oracle.route_scores(np.zeros((1, nb)), p, 0)
        assert n_p[0] == math.ceil(p * nb - 1e-9)
        assert list(order[0, :n_i[0]]) == list(range(n_i[0]))   # equal masses: ascending j
        assert amb[0] == (n_i[0] < nb)                           # ties across a cut, if any


def _featured16():
    """16 blocks of 64 tokens with the positional feature term: concentrated rows."""
    w = syn.workload(2, T=2, Hs=16, Ws=32, H=3, block=64)
    return w, syn.make_inputs(w)


@pytest.mark.parametrize("inputs", [_tiny, _featured16])
def test_brute_force_smallest_then_heaviest_subset(inputs):
    """Every kept set is a smallest subset reaching p, and a heaviest one of its size."""
    w, x = inputs()
    nb = w.nb
    subsets = ((np.arange(1 << nb)[:, None] >> np.arange(nb)[None, :]) & 1).astype(np.float64)
    size = subsets.sum(axis=1).astype(np.int64)
    for p, kf in ((0.9, 2), (0.6, 0), (0.97, 5)):
        r = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, p, kf)
        for row in range(w.rows):
            if r.ambiguous[row]:
                continue
            P = r.P[row]
            mass = subsets @ P
            kept = r.col_idx[r.row_ptr[row]:r.row_ptr[row + 1]]
            n = len(kept)
            best_of_size = mass[size == n].max()
            assert abs(P[kept].sum() - best_of_size) <= 1e-12
            reach = mass >= p
            n_min = size[reach].min() if reach.any() else nb
            assert n == min(nb, max(kf, n_min))


def test_score_temperature_and_softmax():
    """Scores are <Qbar,Kbar>/sqrt(d) and P is their row softmax (d = 64 tiny)."""
    w, x = _tiny()
    r = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, 0.9, 2)
    i, j, bh = 3, 11, 1
    s = float(np.dot(r.qbar[bh, i], r.kbar[bh, j])) / 8.0
    assert abs(r.scores[bh, i, j] - s) <= 1e-12 * max(1.0, abs(s))
    row = r.scores[bh, i]
    assert abs(r.P[bh * w.nb + i, j] - math.exp(row[j]) / np.exp(row).sum()) <= 1e-12


def test_errors():
    with pytest.raises(ValueError):
        oracle.route_scores(np.zeros((1, 4)), 0.0, 1)
    with pytest.raises(ValueError):
        oracle.route_scores(np.zeros((1, 4)), 0.5, -1)
