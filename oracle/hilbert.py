"""Oracle: frame-major 2-D Hilbert token order (test infrastructure only).

What it follows: the FVAttn pages reorder tokens along a Hilbert curve so that
spatially adjacent tokens fall into the same or nearby blocks (FVAttn review,
section 3 "Stage 1: Sparse Mask Routing" and section 3.1 "Sparse Routing
Frontend"; alanhou.org blog, "Core Mechanism", Layer 1: spatially and
temporally neighbouring tokens are grouped).

Reading taken (the pages name no variant): frames stay in time order; inside
each latent frame the (y, x) cells are visited in the order of the classic
2-D Hilbert curve (Hilbert 1891) over the smallest 2^m x 2^m square covering
Hs x Ws, x the column and y the row, the curve starting at (x, y) = (0, 0) and
ending at (2^m - 1, 0); cells outside the Hs x Ws grid are skipped.

This module *enumerates* the curve (curve index -> cell); the CUDA library
computes the inverse map (cell -> curve index) and sorts, so the two
constructions check each other.  Pins: 4-adjacency of consecutive cells,
aligned-quadrant locality at every scale, the end corners, and a hand-written
4x4 order (tests/golden/hilbert_4x4.txt).
"""
from __future__ import annotations

import numpy as np


def hilbert_cells(m: int) -> np.ndarray:
    """Cells of the order-m Hilbert curve in curve order: int64 [4**m, 2] of (x, y).

    Built by unfolding the curve index two bits at a time, least significant
    pair first: at scale s the pair selects one of the four s x s quadrants
    (lower-left, upper-left, upper-right, lower-right for pair values 0..3),
    and the sub-curve already built for the lower scales is reflected/
    transposed so that it enters and leaves that quadrant at the right corners.
    """
    n = 1 << m
    idx = np.arange(n * n, dtype=np.int64)
    x = np.zeros_like(idx)
    y = np.zeros_like(idx)
    t = idx.copy()
    s = 1
    while s < n:
        qx = (t >> 1) & 1            # right half?
        qy = (t ^ qx) & 1            # upper half?
        # lower quadrants: transpose; lower-right additionally reflects.
        lower = qy == 0
        refl = lower & (qx == 1)
        x = np.where(refl, s - 1 - x, x)
        y = np.where(refl, s - 1 - y, y)
        x, y = np.where(lower, y, x), np.where(lower, x, y)
        x = x + s * qx
        y = y + s * qy
        t >>= 2
        s <<= 1
    return np.stack([x, y], axis=1)


def frame_hilbert_perm(T: int, Hs: int, Ws: int) -> np.ndarray:
    """perm[n'] = raster token index (t*Hs*Ws + y*Ws + x) at reordered position n'.

    Frame-major; inside a frame, the in-grid cells of the covering Hilbert
    curve in curve order.
    """
    side = max(Hs, Ws)
    m = 0
    while (1 << m) < side:
        m += 1
    cells = hilbert_cells(m)
    keep = (cells[:, 0] < Ws) & (cells[:, 1] < Hs)
    frame = cells[keep, 1] * Ws + cells[keep, 0]
    assert frame.size == Hs * Ws
    hw = Hs * Ws
    return (np.arange(T, dtype=np.int64)[:, None] * hw + frame[None, :]).reshape(-1)


def identity_perm(T: int, Hs: int, Ws: int) -> np.ndarray:
    return np.arange(T * Hs * Ws, dtype=np.int64)
