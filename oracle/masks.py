"""Oracle: fixed block masks (test infrastructure only).

Window plus rotating global anchors, the structured pattern of the LVSA wiki
page ("TL;DR" and "Key points": a structured local window pattern plus global
anchor blocks that shift across diffusion timesteps).  The page gives neither
the window width nor the anchor rule; the reading used here: on the
frame-major token order, query block i keeps key block j when the latent-frame
ranges the two blocks cover come within `radius` frames of each other, plus
`n_anchor` anchor blocks {(step + m * floor(nb / n_anchor)) mod nb : m <
n_anchor} for every row.  Columns ascending, unique; identical for every head.

Pins (tests/test_oracle_masks.py): a hand-counted small case, symmetry of the
window part, every row containing its own block and the anchors, and the
window being exactly the frame-distance predicate evaluated pair by pair.
"""
from __future__ import annotations

import numpy as np


def block_frames(N: int, block: int, frame_tokens: int):
    """(first, last) latent frame covered by each block of a frame-major order."""
    nb = -(-N // block)
    first = [(i * block) // frame_tokens for i in range(nb)]
    last = [(min(N, (i + 1) * block) - 1) // frame_tokens for i in range(nb)]
    return first, last


def window_anchor_rows(N: int, block: int, frame_tokens: int, radius: int, n_anchor: int, step: int):
    """List of sorted column lists, one per query block (one head)."""
    nb = -(-N // block)
    first, last = block_frames(N, block, frame_tokens)
    anchors = {(step + m * (nb // n_anchor)) % nb for m in range(n_anchor)} if n_anchor > 0 else set()
    rows = []
    for i in range(nb):
        cols = set(anchors)
        for j in range(nb):
            if first[j] <= last[i] + radius and last[j] >= first[i] - radius:
                cols.add(j)
        rows.append(sorted(cols))
    return rows


def window_anchor_csr(B: int, H: int, N: int, block: int, frame_tokens: int, radius: int, n_anchor: int,
                      step: int):
    """CSR (row_ptr int64 [B*H*nb+1], col_idx int64 [nnz]) with rows (b*H + h)*nb + i."""
    rows = window_anchor_rows(N, block, frame_tokens, radius, n_anchor, step)
    counts = [len(r) for r in rows] * (B * H)
    row_ptr = np.zeros(len(counts) + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    col_idx = np.array([c for _ in range(B * H) for r in rows for c in r], dtype=np.int64)
    return row_ptr, col_idx
