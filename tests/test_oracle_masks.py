"""Pins for the fixed window + anchor mask oracle."""
import numpy as np

import oracle.masks as om
import synthetic as syn


def test_hand_counted_case():
    # 4 frames of 8 tokens, blocks of 4 tokens -> 8 blocks, 2 per frame.
    # radius 0: a block sees the blocks of its own frame; 1 anchor at step 3 -> block 3
    rows = om.window_anchor_rows(N=32, block=4, frame_tokens=8, radius=0, n_anchor=1, step=3)
    assert rows == [[0, 1, 3], [0, 1, 3], [2, 3], [2, 3], [3, 4, 5], [3, 4, 5], [3, 6, 7], [3, 6, 7]]
    # radius 1, no anchors: frames f-1..f+1
    rows = om.window_anchor_rows(N=32, block=4, frame_tokens=8, radius=1, n_anchor=0, step=0)
    assert rows[0] == [0, 1, 2, 3] and rows[3] == [0, 1, 2, 3, 4, 5] and rows[7] == [4, 5, 6, 7]


def test_blocks_straddling_frames_and_tail():
    # 3 frames of 10 tokens (N = 30), blocks of 4 -> 8 blocks; block 2 covers tokens 8..11 (frames 0 and 1)
    first, last = om.block_frames(30, 4, 10)
    assert (first[2], last[2]) == (0, 1) and (first[7], last[7]) == (2, 2)
    rows = om.window_anchor_rows(N=30, block=4, frame_tokens=10, radius=0, n_anchor=0, step=0)
    assert rows[2] == [0, 1, 2, 3, 4]          # blocks touching frame 0 or 1


def test_window_properties_on_long_shape():
    w = syn.workload(5, T=12, Hs=6, Ws=10, H=1, block=32)
    hw = w.Hs * w.Ws
    rows = om.window_anchor_rows(w.N, w.block, hw, 2, 8, 2)
    nb = w.nb
    anchors = {(2 + m * (nb // 8)) % nb for m in range(8)}
    first, last = om.block_frames(w.N, w.block, hw)
    for i, cols in enumerate(rows):
        assert cols == sorted(set(cols)) and i in cols and anchors <= set(cols)
        for j in range(nb):
            near = first[j] <= last[i] + 2 and last[j] >= first[i] - 2
            assert (j in cols) == (near or j in anchors)
            if near:
                assert i in rows[j]                   # the window part is symmetric
