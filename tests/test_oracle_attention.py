"""Pins for the attention oracle: library routine, closed forms, special cases."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn


def _small(T=2, Hs=5, Ws=7, H=2, d=16, block=16, seed=7):
    w = syn.workload(2, T=T, Hs=Hs, Ws=Ws, H=H, d=d, block=block)
    x = syn.make_inputs(w, seed=seed)
    return w, x


def _dense_mask(w):
    nb = w.nb
    row_ptr = np.arange(w.rows + 1, dtype=np.int64) * nb
    col_idx = np.tile(np.arange(nb), w.rows)
    return row_ptr, col_idx


def _sdpa(q, k, v):
    """torch float64 scaled_dot_product_attention over [B,N,H,d] inputs."""
    t = [torch.from_numpy(oracle.decode(a)).permute(0, 2, 1, 3) for a in (q, k, v)]
    return torch.nn.functional.scaled_dot_product_attention(*t).permute(0, 2, 1, 3).numpy()


def test_all_blocks_equals_sdpa():
    w, x = _small()
    rp, ci = _dense_mask(w)
    out = oracle.sparse_attention(x["q"], x["k"], x["v"], w.T, w.Hs, w.Ws, w.block, rp, ci)
    assert np.abs(out - _sdpa(x["q"], x["k"], x["v"])).max() < 1e-12
    assert np.abs(oracle.dense_attention(x["q"], x["k"], x["v"]) - out).max() < 1e-12


def test_routed_with_p_one_equals_sdpa():
    w, x = _small(T=1, Hs=8, Ws=8, d=32, block=16)
    r = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, 1.0, 0)
    out = oracle.sparse_attention(x["q"], x["k"], x["v"], w.T, w.Hs, w.Ws, w.block, r.row_ptr, r.col_idx)
    assert np.abs(out - _sdpa(x["q"], x["k"], x["v"])).max() < 1e-12


def test_constant_v_gives_constant():
    w, x = _small()
    v = np.full_like(x["v"], syn.f32_to_bf16_bits(np.float32(0.375)))
    r = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, 0.7, 1)
    out = oracle.sparse_attention(x["q"], x["k"], v, w.T, w.Hs, w.Ws, w.block, r.row_ptr, r.col_idx)
    assert np.abs(out - 0.375).max() < 1e-14


def test_identical_keys_give_block_mean_of_v():
    w, x = _small()
    perm = oracle.token_perm(w.T, w.Hs, w.Ws)
    k = x["k"].copy()
    k[:] = k[:, :1]                                   # every key equals token 0's key
    j0 = 1
    row_ptr = np.arange(w.rows + 1, dtype=np.int64)
    col_idx = np.full(w.rows, j0, dtype=np.int64)
    out = oracle.sparse_attention(x["q"], k, x["v"], w.T, w.Hs, w.Ws, w.block, row_ptr, col_idx)
    toks = perm[j0 * w.block:(j0 + 1) * w.block]
    mean_v = oracle.decode(x["v"][:, toks]).mean(axis=1)          # [B, H, d]
    assert np.abs(out - mean_v[:, None]).max() < 1e-12


def test_diagonal_mask_is_block_local_attention():
    w, x = _small()
    perm = oracle.token_perm(w.T, w.Hs, w.Ws)
    nb = w.nb
    row_ptr = np.arange(w.rows + 1, dtype=np.int64)
    col_idx = np.tile(np.arange(nb), w.rows)
    out = oracle.sparse_attention(x["q"], x["k"], x["v"], w.T, w.Hs, w.Ws, w.block, row_ptr, col_idx)
    for i in range(nb):
        toks = perm[i * w.block:min(w.N, (i + 1) * w.block)]
        ref = _sdpa(x["q"][:, toks], x["k"][:, toks], x["v"][:, toks])
        assert np.abs(out[:, toks] - ref).max() < 1e-12


def test_attend_block_row_subset_matches_full_block():
    w, x = _small()
    perm = oracle.token_perm(w.T, w.Hs, w.Ws)
    r = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, 0.8, 2)
    full = oracle.attend_block(x["q"], x["k"], x["v"], perm, w.block, r.row_ptr, r.col_idx, w.H, 0, 1, w.nb - 1)
    part = oracle.attend_block(x["q"], x["k"], x["v"], perm, w.block, r.row_ptr, r.col_idx, w.H, 0, 1, w.nb - 1,
                               rows=[0, full.shape[0] - 1])
    assert np.array_equal(part, full[[0, -1]])
