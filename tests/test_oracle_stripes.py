"""Pins for the stripe-mask oracle (oracle/stripes.py)."""
import numpy as np
import pytest

import oracle.masks as om
import oracle.stripes as st


def test_hand_worked_one_frame_per_block():
    # T=4 frames of 2x2 tokens, block = 4 tokens: block i is frame i, rows 0..1
    F, Y = st.block_ranges(4, 2, 2, 4)
    assert F == [(0, 0), (1, 1), (2, 2), (3, 3)] and Y == [(0, 1)] * 4
    # the next frame only (offset +1, width 0, single stripe), any row
    assert st.stripe_rows(4, 2, 2, 4, (0, 1, 0, 1, 0, 0)) == [[1], [2], [3], []]
    # every other frame: stride 2, width 0
    assert st.stripe_rows(4, 2, 2, 4, (0, 0, 2, 1, 0, 0)) == [[0, 2], [1, 3], [0, 2], [1, 3]]
    # rows: the query's own row range only (width 0) still meets every block (rows 0..1 overlap)
    assert st.stripe_rows(4, 2, 2, 4, (3, 0, 0, 0, 0, 0)) == [[0, 1, 2, 3]] * 4
    # a row offset of 5 with width 0 meets no block of a 2-row frame
    assert st.stripe_rows(4, 2, 2, 4, (3, 0, 0, 0, 5, 0)) == [[], [], [], []]


@pytest.mark.parametrize("shape", [(6, 8, 10, 64), (5, 9, 7, 32), (21, 6, 13, 128)])
@pytest.mark.parametrize("radius", [0, 1, 2])
def test_window_mask_is_a_special_case(shape, radius):
    T, Hs, Ws, block = shape
    got = st.stripe_rows(T, Hs, Ws, block, (radius, 0, 0, Hs, 0, 0))
    want = om.window_anchor_rows(T * Hs * Ws, block, Hs * Ws, radius, 0, 0)
    assert got == want


def test_stride_one_keeps_everything():
    rows = st.stripe_rows(3, 5, 6, 16, (0, 0, 1, 0, 0, 1))
    nb = len(rows)
    assert rows == [list(range(nb))] * nb


@pytest.mark.parametrize("params", [(0, 1, 0, 1, 2, 0), (1, -2, 3, 0, 1, 4), (0, 2, 5, 2, -1, 0)])
def test_negated_offsets_transpose(params):
    T, Hs, Ws, block = 6, 7, 9, 32
    w_t, o_t, s_t, w_s, o_s, s_s = params
    a = st.stripe_rows(T, Hs, Ws, block, params)
    b = st.stripe_rows(T, Hs, Ws, block, (w_t, -o_t, s_t, w_s, -o_s, s_s))
    nb = len(a)
    A = np.zeros((nb, nb), bool)
    Bm = np.zeros((nb, nb), bool)
    for i in range(nb):
        A[i, a[i]] = True
        Bm[i, b[i]] = True
    assert np.array_equal(A, Bm.T)
