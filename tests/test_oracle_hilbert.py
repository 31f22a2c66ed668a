"""Pins for the oracle's Hilbert order (curve properties and a hand-drawn 4x4 order)."""
import os

import numpy as np
import pytest

from oracle import frame_hilbert_perm, hilbert_cells

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_order2_matches_hand_drawn_curve():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "hilbert_4x4.txt")) if l.strip() and not l.startswith("#")]
    want = np.array(rows, dtype=np.int64)
    assert np.array_equal(hilbert_cells(2), want)


@pytest.mark.parametrize("m", range(0, 8))
def test_curve_is_adjacent_bijection(m):
    c = hilbert_cells(m)
    n = 1 << m
    assert c.shape == (n * n, 2)
    assert len({(int(x), int(y)) for x, y in c}) == n * n
    assert c.min() == 0 and c.max() == n - 1
    if m:
        assert np.all(np.abs(np.diff(c, axis=0)).sum(axis=1) == 1)
        assert tuple(c[0]) == (0, 0) and tuple(c[-1]) == (n - 1, 0)


@pytest.mark.parametrize("m", [3, 5, 6])
def test_curve_fills_aligned_squares_at_every_scale(m):
    c = hilbert_cells(m)
    for k in range(1, m + 1):
        run = 4 ** k
        blk = c.reshape(-1, run, 2) >> k                 # aligned 2^k square of each cell
        assert np.all(blk == blk[:, :1, :])


@pytest.mark.parametrize("T,Hs,Ws", [(1, 1, 1), (2, 3, 5), (4, 16, 16), (3, 45, 80), (2, 30, 52)])
def test_frame_perm(T, Hs, Ws):
    perm = frame_hilbert_perm(T, Hs, Ws)
    hw = Hs * Ws
    assert np.array_equal(np.sort(perm), np.arange(T * hw))
    assert np.all(perm.reshape(T, hw) // hw == np.arange(T)[:, None])     # frames contiguous, in order
    y, x = (perm % hw) // Ws, perm % Ws
    step = np.abs(np.diff(y.reshape(T, hw), axis=1)) + np.abs(np.diff(x.reshape(T, hw), axis=1))
    if Hs == Ws and Hs & (Hs - 1) == 0 and hw > 1:
        assert np.all(step == 1)
    # in-grid cells keep curve order: same as filtering the full square curve
    m = max(Hs, Ws).bit_length() if max(Hs, Ws) & (max(Hs, Ws) - 1) else max(Hs, Ws).bit_length() - 1
    c = hilbert_cells(m)
    keep = (c[:, 0] < Ws) & (c[:, 1] < Hs)
    assert np.array_equal(perm[:hw], c[keep, 1] * Ws + c[keep, 0])
