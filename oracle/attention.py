"""Oracle: attention restricted to the retained key blocks, fp64 (test infrastructure only).

Only tests/, the package's smoke check and the bench's CPU-baseline leg may
import this module; the product path never does.

What it computes (FVAttn review, section 3 "Block-Sparse Attention Execution";
alanhou.org blog, "Core Mechanism", Layer 1): for a query token in block i of
the reordered sequence, ordinary softmax attention whose keys are exactly the
real tokens of the key blocks listed for row (b, h, i) of the CSR mask, scale
1/sqrt(d), no causal mask, output returned for the original token position.
Padding never enters: blocks are cut from the N real tokens only.

The inputs are the values the CUDA path sees: bf16 Q, K, V (uint16 bit
patterns), widened exactly to fp64.

Pins (tests/test_oracle_attention.py): with every block kept the result equals
dense softmax attention, checked against torch's float64
scaled_dot_product_attention on CPU; constant V gives that constant; one key
block of identical keys gives the mean of V over that block; a one-block-per-
row mask reduces to attention inside that block.
"""
from __future__ import annotations

import numpy as np

from .route import decode, token_perm


def _softmax_rows(s: np.ndarray) -> np.ndarray:
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def attend_block(q, k, v, perm, block, row_ptr, col_idx, H, b, h, i, rows=None):
    """Outputs of query block i of head (b, h), fp64 [len(rows), d].

    `rows` selects positions inside the block (0..m_i-1), default all; the
    returned rows belong to tokens perm[i*block + rows].
    """
    B, N, _, d = q.shape
    nb = -(-N // block)
    r = (b * H + h) * nb + i
    lo = i * block
    hi = min(N, lo + block)
    pos = np.arange(lo, hi) if rows is None else lo + np.asarray(rows)
    qi = decode(q[b, perm[pos], h, :])
    keys = []
    for j in col_idx[row_ptr[r]:row_ptr[r + 1]]:
        keys.append(np.arange(j * block, min(N, (j + 1) * block)))
    kp = perm[np.concatenate(keys)]
    kj = decode(k[b, kp, h, :])
    vj = decode(v[b, kp, h, :])
    P = _softmax_rows(qi @ kj.T / np.sqrt(float(d)))
    return P @ vj


def sparse_attention(q, k, v, T, Hs, Ws, block, row_ptr, col_idx, order="hilbert"):
    """Full output [B, N, H, d] fp64, original token order.  Small inputs only."""
    B, N, H, d = q.shape
    perm = token_perm(T, Hs, Ws, order)
    nb = -(-N // block)
    out = np.zeros((B, N, H, d))
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                lo, hi = i * block, min(N, (i + 1) * block)
                out[b, perm[lo:hi], h, :] = attend_block(q, k, v, perm, block, row_ptr,
                                                         col_idx, H, b, h, i)
    return out


def dense_attention(q, k, v):
    """softmax(Q K^T / sqrt(d)) V over all N keys, per (b, h); fp64 [B, N, H, d]."""
    B, N, H, d = q.shape
    out = np.zeros((B, N, H, d))
    for b in range(B):
        for h in range(H):
            qq, kk, vv = (decode(x[b, :, h, :]) for x in (q, k, v))
            out[b, :, h, :] = _softmax_rows(qq @ kk.T / np.sqrt(float(d))) @ vv
    return out
