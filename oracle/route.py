"""Oracle: FVAttn-style Top-p block routing, fp64, plain numpy (test infrastructure only).

Only tests/, the package's smoke check and the bench's CPU-baseline leg may
import this module; the product path never does.

Steps, in the order the pages give them (FVAttn review, section 3 "Stage 1:
Sparse Mask Routing" and section 3.1; alanhou.org blog, "Key Concepts",
Top-p routing with safety floor):

  1. reorder tokens along the frame-major Hilbert order (oracle.hilbert);
  2. cut the reordered sequence into blocks of `block` tokens (the last block
     holds the remainder);
  3. mean-pool Q and K over the actual tokens of each block;
  4. block scores s_ij = <Qbar_i, Kbar_j> / sqrt(d);
  5. per query block, P_ij = softmax_j(s_ij);
  6. order key blocks by P descending, equal P by ascending j;
  7. cumulative mass C_n over that order; n_p = the smallest n with C_n >= p
     ("the minimum number of blocks whose cumulative attention weight reaches
     p"), n_p = nb when p >= 1 or when no prefix reaches p;
  8. Top-k safety floor: n_i = min(nb, max(k_floor, n_p)); keep the first n_i
     blocks of the order (they are also the key-block importance order the
     review's Stage-1 output names);
  9. per-head workload L_h = mean_i sum_j M_hij (FVAttn review, Eq. 1).

Readings where the pages are silent: the score temperature is the attention
scale 1/sqrt(d); ">= p" (reached, not exceeded); the tail block is pooled over
its real tokens only and gets no re-weighting; k_floor > nb clamps to nb;
masks are per head and per query block.

Pins (tests/test_oracle_route.py): constant blocks pool to their value; p = 1
keeps every block; the floor holds; kept sets are nested and monotone in p;
a uniform row keeps ceil(p*nb) blocks; a hand-worked 4-block example
(tests/golden/route_worked_example.json); brute-force subset enumeration on
16-block rows.  The numeric values of routing on the synthetic workloads are
otherwise not printed by the pages ("parity unpinned" beyond those pins).
"""
from __future__ import annotations

import dataclasses

import numpy as np

from .hilbert import frame_hilbert_perm, identity_perm

TIE_REL = 1e-6   # relative tolerance under which two masses count as tied


def decode(x: np.ndarray) -> np.ndarray:
    """Input values as fp64: fp32 arrays as they are, uint16 arrays as bf16 bit patterns."""
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


def token_perm(T: int, Hs: int, Ws: int, order: str = "hilbert") -> np.ndarray:
    return frame_hilbert_perm(T, Hs, Ws) if order == "hilbert" else identity_perm(T, Hs, Ws)


def block_counts(N: int, block: int) -> np.ndarray:
    """m_i: the number of real tokens in each block of the reordered sequence."""
    nb = -(-N // block)
    m = np.full(nb, block, dtype=np.int64)
    m[-1] = N - (nb - 1) * block
    return m


def pool_head(x_head: np.ndarray, perm: np.ndarray, block: int) -> np.ndarray:
    """Mean over each block of one head's rows taken in reordered order.

    x_head: [N, d] (any dtype `decode` accepts); returns fp64 [nb, d].
    """
    xr = decode(x_head[perm])
    N = xr.shape[0]
    starts = np.arange(0, N, block)
    sums = np.add.reduceat(xr, starts, axis=0)
    return sums / block_counts(N, block)[:, None].astype(np.float64)


@dataclasses.dataclass
class RouteResult:
    nb: int
    counts: np.ndarray      # int64 [rows]: n_i
    n_p: np.ndarray         # int64 [rows]: Top-p count before the floor
    row_ptr: np.ndarray     # int64 [rows+1]
    col_idx: np.ndarray     # int64 [nnz], importance order within each row
    L_h: np.ndarray         # float32 [B*H]
    nnz: int
    ambiguous: np.ndarray   # bool [rows]: decision within TIE_REL of a tie / of p
    P_sorted: np.ndarray    # fp64 [rows, nb]: P in importance order
    P: np.ndarray           # fp64 [rows, nb]: P in key-block order
    order: np.ndarray       # int64 [rows, nb]: the full key-block importance order
    qbar: np.ndarray        # fp64 [B*H, nb, d]
    kbar: np.ndarray        # fp64 [B*H, nb, d]
    scores: np.ndarray      # fp64 [B*H, nb, nb]


def route_scores(scores: np.ndarray, p: float, k_floor: int):
    """Steps 5-8 on a matrix of block scores [rows, nb] (fp64)."""
    if not (p > 0.0):
        raise ValueError("p must be > 0")
    if k_floor < 0:
        raise ValueError("k_floor must be >= 0")
    rows, nb = scores.shape
    mx = scores.max(axis=1, keepdims=True)
    e = np.exp(scores - mx)
    P = e / e.sum(axis=1, keepdims=True)
    order = np.argsort(-P, axis=1, kind="stable")        # P desc, ties by ascending j
    Ps = np.take_along_axis(P, order, axis=1)
    C = np.cumsum(Ps, axis=1)
    reached = C >= p
    n_p = np.where(reached.any(axis=1), reached.argmax(axis=1) + 1, nb)
    if p >= 1.0:
        n_p = np.full(rows, nb, dtype=np.int64)
    n_i = np.minimum(nb, np.maximum(k_floor, n_p)).astype(np.int64)

    # Ambiguity: a decision the pages' arithmetic cannot pin to TIE_REL.
    amb = np.zeros(rows, dtype=bool)
    r = np.arange(rows)
    cut = n_i < nb
    a = Ps[r[cut], n_i[cut] - 1]
    b = Ps[r[cut], n_i[cut]]
    amb[cut] = np.abs(a - b) <= TIE_REL * a
    if p < 1.0:
        c_at = C[r, n_p - 1]
        c_before = np.where(n_p >= 2, C[r, np.maximum(n_p - 2, 0)], 0.0)
        amb |= (np.abs(c_at - p) <= TIE_REL * p) | (np.abs(c_before - p) <= TIE_REL * p)
    return P, order, Ps, n_p.astype(np.int64), n_i, amb


def route(q: np.ndarray, k: np.ndarray, T: int, Hs: int, Ws: int, block: int,
          p: float, k_floor: int, order: str = "hilbert") -> RouteResult:
    """Route Q, K of layout [B, N, H, d] (fp32 or bf16 bit patterns).

    Rows are numbered r = (b*H + h)*nb + i with i a block of the reordered
    sequence; columns j are blocks of the same order.
    """
    B, N, H, d = q.shape
    assert N == T * Hs * Ws and k.shape == q.shape
    perm = token_perm(T, Hs, Ws, order)
    nb = -(-N // block)
    qbar = np.empty((B * H, nb, d))
    kbar = np.empty((B * H, nb, d))
    for b in range(B):
        for h in range(H):
            qbar[b * H + h] = pool_head(q[b, :, h, :], perm, block)
            kbar[b * H + h] = pool_head(k[b, :, h, :], perm, block)
    scores = np.matmul(qbar, np.swapaxes(kbar, 1, 2)) / np.sqrt(float(d))
    P, order_idx, Ps, n_p, n_i, amb = route_scores(scores.reshape(-1, nb), p, k_floor)
    row_ptr = np.zeros(n_i.size + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(n_i)
    keep = np.arange(nb)[None, :] < n_i[:, None]
    col_idx = order_idx[keep].astype(np.int64)
    per_head = n_i.reshape(B * H, nb).sum(axis=1)
    L_h = per_head.astype(np.float32) / np.float32(nb)
    return RouteResult(nb=nb, counts=n_i, n_p=n_p, row_ptr=row_ptr, col_idx=col_idx,
                       L_h=L_h, nnz=int(row_ptr[-1]), ambiguous=amb, P_sorted=Ps, P=P, order=order_idx,
                       qbar=qbar, kbar=kbar, scores=scores)
