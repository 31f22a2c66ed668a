"""Oracle: periodic diagonal stripe block masks (test infrastructure only).

The PSA pages ("Parameterized Stripe Attention for Efficient Video
Generation": section 3.1, section 3.2 "Efficient and Flexible Kernel",
appendix C.2 "Initialization of Mask Candidates" and appendix D
"Locality-Induced Periodic Diagonal Stripes") describe per-head masks made of
periodic diagonal stripes: an inter-frame and an intra-frame part, each with
a width, an offset and a stride (six parameters), an infinite stride meaning
a single diagonal, masking done per block.  Under row-major token order the
temporal stripes repeat every frame (H*W tokens) and the column-wise ones
every row (W tokens), with half-widths set by the locality radii.

Reading used here, on blocks of the frame-major token order:
  - the inter-frame part works on latent-frame offsets, the intra-frame part
    on row offsets inside a frame (the two strides of the pages in token
    units, a frame and a row, become 1 frame and 1 row);
  - for key offset delta (key minus query), a part with half-width w, offset
    o and stride s keeps delta when |delta - o - n*s| <= w for some integer
    n (s <= 0: n = 0 only, a single stripe);
  - query block i and key block j are kept together when the inter-frame
    part keeps some frame offset f' - f (f a frame of block i, f' of block j)
    and the intra-frame part keeps some row offset y' - y, each taken over
    the range the blocks span ([min, max] of their tokens' frames and rows).
Parameters per head: (w_t, o_t, s_t, w_s, o_s, s_s).  Columns ascending.

Pins (tests/test_oracle_stripes.py): a hand-worked small case; an infinite
stride and an intra-frame width covering every row reproduce the window mask
of oracle.masks; stride 1 with width 0 keeps everything; negating both
offsets transposes the mask.
"""
from __future__ import annotations

import numpy as np

from .route import token_perm


def block_ranges(T: int, Hs: int, Ws: int, block: int, order: str = "hilbert"):
    """Per block of the token order: (min frame, max frame), (min row, max row)."""
    perm = token_perm(T, Hs, Ws, order)
    N = T * Hs * Ws
    nb = -(-N // block)
    F, Y = [], []
    for i in range(nb):
        toks = perm[i * block:min(N, (i + 1) * block)]
        t = toks // (Hs * Ws)
        y = (toks % (Hs * Ws)) // Ws
        F.append((int(t.min()), int(t.max())))
        Y.append((int(y.min()), int(y.max())))
    return F, Y


def stripe_keeps(lo: int, hi: int, w: int, o: int, s: int) -> bool:
    """Does some offset delta in [lo, hi] lie within w of a stripe centre o + n*s?"""
    for delta in range(lo, hi + 1):
        if s <= 0:
            if abs(delta - o) <= w:
                return True
            continue
        n0 = (delta - o) // s
        for n in (n0 - 1, n0, n0 + 1):
            if abs(delta - o - n * s) <= w:
                return True
    return False


def stripe_rows(T, Hs, Ws, block, params, order="hilbert"):
    """Sorted column lists of one head's query blocks for params (w_t, o_t, s_t, w_s, o_s, s_s)."""
    w_t, o_t, s_t, w_s, o_s, s_s = (int(v) for v in params)
    F, Y = block_ranges(T, Hs, Ws, block, order)
    nb = len(F)
    rows = []
    for i in range(nb):
        cols = []
        for j in range(nb):
            if (stripe_keeps(F[j][0] - F[i][1], F[j][1] - F[i][0], w_t, o_t, s_t)
                    and stripe_keeps(Y[j][0] - Y[i][1], Y[j][1] - Y[i][0], w_s, o_s, s_s)):
                cols.append(j)
        rows.append(cols)
    return rows


def stripe_csr(B, H, T, Hs, Ws, block, params, order="hilbert"):
    """CSR over rows (b*H + h)*nb + i; params: [H, 6]."""
    per_head = [stripe_rows(T, Hs, Ws, block, params[h], order) for h in range(H)]
    counts, cols = [], []
    for _ in range(B):
        for h in range(H):
            for r in per_head[h]:
                counts.append(len(r))
                cols.extend(r)
    row_ptr = np.zeros(len(counts) + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    return row_ptr, np.asarray(cols, dtype=np.int64)
