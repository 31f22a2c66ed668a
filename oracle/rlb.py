"""Oracle: runtime load balancing by head migration (test infrastructure only).

FVAttn review, section 3 "Stage 2: Runtime Load Balancing", Eqs. 1-6, section
3.2 and the RLB algorithm flow of section 5:

  L_r      = sum of L_h over the heads of rank r                      (Eq. 1)
  rho      = max_r L_r / mean_r L_r                                   (Eq. 2)
  K        = c * (max_r L_r - max_r L_r_new),  G = K - P - C          (Eqs. 3-4)
  L_r_new  = L_r - L_{h_r} + L_{h_sigma^-1(r)}                        (Eq. 5)
  sigma*   = argmin over S_20% of (max_r L_r_new, Var_r L_r_new)      (Eq. 6)

Reading of S_20% (the pages: one-send-one-receive, at most one local head per
rank, pair topologies enumerated for 8 GPUs): a plan is a set of disjoint rank
pairs, each pair swapping one head of each side; ranks outside every pair keep
their heads; the empty plan is allowed.  Ties in the objective are broken by
the first plan in the enumeration order of `plans()`; only the objective value
is compared against the library, which may return any optimal plan.

Also the enabling policy of section 3.3: rho < k1 -> nothing, k1 <= rho < k2 ->
SASA only, rho >= k2 -> RLB then SASA (k1 = 1.05, k2 = 1.10).
"""
from __future__ import annotations

import itertools

import numpy as np


def rank_loads(L_h, head_rank, R):
    L = np.zeros(R)
    for l, r in zip(L_h, head_rank):
        L[r] += l
    return L


def rho(L_r):
    L = np.asarray(L_r, dtype=np.float64)
    return float(L.max() / L.mean())


def matchings(R):
    """Every set of disjoint pairs over ranks 0..R-1 (the empty set included)."""
    def rec(free):
        if not free:
            yield []
            return
        first, rest = free[0], free[1:]
        yield from rec(rest)                              # `first` stays unmatched
        for i, other in enumerate(rest):
            for m in rec(rest[:i] + rest[i + 1:]):
                yield [(first, other)] + m
    yield from rec(list(range(R)))


def plans(L_h, head_rank, R):
    """All plans in S_20%: (pairs, chosen heads) with the loads after migration."""
    heads_of = [[h for h, r in enumerate(head_rank) if r == k] for k in range(R)]
    base = rank_loads(L_h, head_rank, R)
    for m in matchings(R):
        choices = [itertools.product(heads_of[a], heads_of[b]) for a, b in m]
        for pick in itertools.product(*choices):
            L = base.copy()
            moves = []
            for (a, b), (ha, hb) in zip(m, pick):
                L[a] += L_h[hb] - L_h[ha]
                L[b] += L_h[ha] - L_h[hb]
                moves += [(a, b, ha), (b, a, hb)]
            yield moves, L


def best_plan(L_h, head_rank, R):
    """Brute-force Eq. 6: lexicographic minimum of (max L_new, Var L_new)."""
    best = None
    for moves, L in plans(L_h, head_rank, R):
        key = (L.max(), L.var())
        if best is None or key < best[0]:
            best = (key, moves, L)
    return best


def gain(L_r, L_new, c, P, C):
    """Eqs. 3-4: K and G."""
    K = c * (float(np.max(L_r)) - float(np.max(L_new)))
    return K, K - P - C


def policy(rho_value, k1=1.05, k2=1.10):
    """Section 3.3 table: 0 = nothing, 1 = SASA only, 2 = RLB then SASA."""
    return 0 if rho_value < k1 else (1 if rho_value < k2 else 2)
