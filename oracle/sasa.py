"""Oracle: slack-aware sparse augmentation (test infrastructure only).

FVAttn review, section 3 "Stage 3: Slack-Aware Sparse Augmentation (SASA)",
section 3.3 and Eqs. 7-10, and the SASA algorithm flow of section 5:

  dL_r   = L_max_new - L_r_new,           L_max_new = max_r L_r_new     (Eq. 7)
  B_r    = n1 * dL_r   if dL_r > n2 * L_max_new, else 0                  (Eq. 8 + trigger)
  L_aug  = L_r_new + B_r                                                 (Eq. 9)
  A      = max(0, max_r L_aug - L_max_new) + S                           (Eq. 10)

with n1 = 0.8 and n2 = 0.07 (review, section 5 hyper-parameters), and the
augmentation itself: take the unselected blocks of the already sorted
key-block importance order, highest value first, without re-scoring.

Reading for the per-head mechanism (the pages budget per rank): a rank's
budget B_r (in units of L, mean kept blocks per query block) is spread as an
integer a_h = floor(B_r / |H_r|) extra blocks for every query block of each of
its heads, so that L_h grows by exactly a_h (Eq. 1) unless a row is already
full.  A row keeps the first min(nb, n_i + a_h) blocks of its importance order.

Pins (tests/test_oracle_sasa.py): a hand-computed Eq. 7-10 example, B_r <= dL_r,
the trigger threshold, nesting of augmented sets, and L_h growth.
"""
from __future__ import annotations

import numpy as np


def budget(L_r, n1: float = 0.8, n2: float = 0.07, S: float = 0.0):
    """Eq. 7-10 for per-rank workloads L_r; returns dict(dL, B, L_aug, A)."""
    L = np.asarray(L_r, dtype=np.float64)
    L_max = L.max()
    dL = L_max - L
    B = np.where(dL > n2 * L_max, n1 * dL, 0.0)
    L_aug = L + B
    A = max(0.0, float(L_aug.max() - L_max)) + S
    return dict(dL=dL, B=B, L_aug=L_aug, A=A)


def extra_per_head(B_r, heads_per_rank):
    """Integer extra blocks per query block for every head, rank by rank."""
    out = []
    for b, n in zip(B_r, heads_per_rank):
        out += [int(np.floor(b / n))] * int(n)
    return np.asarray(out, dtype=np.int64)


def augment(route_result, extra, nb: int):
    """Augmented CSR from an oracle RouteResult: row r of head bh keeps the
    first min(nb, n_r + extra[bh]) blocks of its importance order."""
    counts = route_result.counts
    heads = counts.size // nb
    add = np.repeat(np.maximum(np.asarray(extra, dtype=np.int64), 0), nb)
    n_out = np.minimum(nb, counts + add[:counts.size])
    row_ptr = np.zeros(counts.size + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(n_out)
    keep = np.arange(nb)[None, :] < n_out[:, None]
    col_idx = route_result.order[keep].astype(np.int64)
    L_h = n_out.reshape(heads, nb).sum(axis=1).astype(np.float32) / np.float32(nb)
    return n_out, row_ptr, col_idx, L_h
