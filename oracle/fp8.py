"""Oracle: attention with an FP8 (e4m3) P.V product (test infrastructure only).

Only tests/ may import this module; the product path never does.

The FVAttn review (section 3 "Block-Sparse Attention Execution" and section
3.4) quantizes V before attention, overlapped with the CPU plan search, and
does not state the format.  Reading used here (the plainest one the rest of
the pages support, in the style of 8-bit attention kernels): Q, K and Q.K^T stay bf16; V of each head
is quantized per channel, Vq[:, c] = e4m3(V[:, c] / sigma_c) with sigma_c =
amax over the head's N tokens of |V[:, c]| / 448 (1 for an all-zero
channel); the probabilities, taken relative to the row maximum (so P <= 1),
enter the product as e4m3(16 P), which keeps them in e4m3's normal range down
to P = 2^-10; the products are summed in fp32 and the output column c is
O = sigma_c / 16 * sum_j e4m3(16 P_j) Vq_j[c] / sum_j P_j, the denominator
from the unrounded probabilities.  (A kernel that lets its running maximum
lag the true one by up to 2^4 rounds 16 P 2^delta instead, 0 <= delta < 4:
other individual roundings, the same error bound.)

e4m3 here is the OCP FP8 E4M3 format: 1 sign, 4 exponent bits (bias 7), 3
mantissa bits, subnormals below 2^-6, largest finite value 448, no
infinities; rounding to nearest, ties to even, saturating at +-448.

Pins (tests/test_oracle_fp8.py): the rounding equals the nearest of the 256
codes enumerated from the format definition (ties to the even code) and
torch's float8_e4m3fn conversion; values already on the grid are fixed
points; equal scores with V = sigma times grid values give plain attention
exactly; on a small workload the result stays within the stated error bound
(mean relative error <= 6e-2) of the exact oracle, and is not exact.
"""
from __future__ import annotations

import numpy as np

from .route import decode

E4M3_MAX = 448.0


def e4m3_table() -> np.ndarray:
    """The values of the 256 e4m3 codes (NaN for the two NaN codes), code order."""
    vals = np.empty(256)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = sign * (m / 8.0) * 2.0 ** -6
        else:
            vals[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


def round_e4m3(x) -> np.ndarray:
    """Round to the nearest e4m3 value, ties to even, saturating at +-448 (fp64 in, fp64 out)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)                     # subnormal spacing below 2^-6
    quantum = np.exp2(e - 3.0)                  # 3 mantissa bits
    r = np.rint(a / quantum) * quantum          # numpy rounds halves to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def channel_scales(v_head: np.ndarray) -> np.ndarray:
    """sigma_c = amax over tokens of |V[:, c]| / 448 for one head's [N, d] V (1 where all zero)."""
    amax = np.max(np.abs(v_head), axis=0)
    return np.where(amax > 0, amax / E4M3_MAX, 1.0)


P_SCALE = 16.0   # probabilities enter the product as e4m3(16 P)


def attend_block_fp8v(q, k, v, perm, block, row_ptr, col_idx, H, b, h, i, sigma=None):
    """Outputs of query block i of head (b, h) with the e4m3 P.V product, fp64 [m_i, d]."""
    B, N, _, d = q.shape
    nb = -(-N // block)
    r = (b * H + h) * nb + i
    lo, hi = i * block, min(N, (i + 1) * block)
    if sigma is None:
        sigma = channel_scales(decode(v[b, :, h, :]))
    qi = decode(q[b, perm[np.arange(lo, hi)], h, :])
    cols = list(col_idx[row_ptr[r]:row_ptr[r + 1]])
    toks = np.concatenate([perm[np.arange(j * block, min(N, (j + 1) * block))] for j in cols])
    S = qi @ decode(k[b, toks, h, :]).T / np.sqrt(float(d))
    P = np.exp(S - S.max(axis=1, keepdims=True))
    vq = round_e4m3(decode(v[b, toks, h, :]) / sigma)
    num = round_e4m3(P_SCALE * P) @ vq
    return num * (sigma / P_SCALE) / P.sum(axis=1, keepdims=True)


def sparse_attention_fp8v(q, k, v, T, Hs, Ws, block, row_ptr, col_idx, order="hilbert"):
    """Full output [B, N, H, d] fp64, original token order (rows with no key block: 0).  Small inputs only."""
    from .route import token_perm
    B, N, H, d = q.shape
    perm = token_perm(T, Hs, Ws, order)
    nb = -(-N // block)
    out = np.zeros((B, N, H, d))
    for b in range(B):
        for h in range(H):
            sigma = channel_scales(decode(v[b, :, h, :]))
            for i in range(nb):
                lo, hi = i * block, min(N, (i + 1) * block)
                r = (b * H + h) * nb + i
                if row_ptr[r + 1] == row_ptr[r]:
                    continue
                out[b, perm[lo:hi], h, :] = attend_block_fp8v(q, k, v, perm, block, row_ptr, col_idx,
                                                              H, b, h, i, sigma)
    return out
