"""The library's host stripe-mask producer against the oracle (no GPU)."""
import numpy as np
import pytest

import oracle.stripes as st


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_top_b200 import build
    build.build()
    import block_sparse_attention_top_b200 as m
    return m


@pytest.mark.parametrize("shape", [(4, 2, 2, 64, 1, 1), (6, 8, 10, 64, 1, 3), (5, 9, 7, 128, 2, 2),
                                   (21, 30, 52, 128, 1, 2)])
@pytest.mark.parametrize("order", [0, 1])
def test_matches_oracle_exactly(bsa, shape, order):
    T, Hs, Ws, block, B, H = shape
    rng = np.random.default_rng(T * 100 + Hs + order)
    params = []
    for h in range(H):
        params.append((int(rng.integers(0, 3)), int(rng.integers(-3, 4)), int(rng.integers(-1, 6)),
                       int(rng.integers(0, 4)), int(rng.integers(-4, 5)), int(rng.integers(-1, 8))))
    rp, ci = bsa.bsa_mask_stripes(B, H, T, Hs, Ws, block, params, order)
    want_rp, want_ci = st.stripe_csr(B, H, T, Hs, Ws, block, np.array(params),
                                     order="hilbert" if order == 0 else "identity")
    np.testing.assert_array_equal(rp.numpy(), want_rp)
    np.testing.assert_array_equal(ci.numpy(), want_ci)


def test_capacity_and_errors(bsa):
    import ctypes
    import torch
    T, Hs, Ws, block = 6, 8, 10, 64
    nb = -(-(T * Hs * Ws) // block)
    params = torch.tensor([0, 0, 0, 8, 0, 0], dtype=torch.int32)     # frame diagonal, every row
    row_ptr = torch.empty(nb + 1, dtype=torch.int32)
    col_idx = torch.empty(3, dtype=torch.int32)
    nnz = ctypes.c_int64()
    rc = bsa._lib.bsa_mask_stripes(1, 1, T, Hs, Ws, block, 0, params.data_ptr(), row_ptr.data_ptr(),
                                   col_idx.data_ptr(), 3, ctypes.byref(nnz))
    assert rc == bsa.BSA_ECAPACITY and nnz.value > 3 and int(row_ptr[-1]) == nnz.value
    bad = torch.tensor([-1, 0, 0, 0, 0, 0], dtype=torch.int32)                 # negative width
    assert bsa._lib.bsa_mask_stripes(1, 1, T, Hs, Ws, block, 0, bad.data_ptr(), row_ptr.data_ptr(),
                                     col_idx.data_ptr(), 3, ctypes.byref(nnz)) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_mask_stripes(1, 1, T, Hs, Ws, 96, 0, params.data_ptr(), row_ptr.data_ptr(),
                                     col_idx.data_ptr(), 3, ctypes.byref(nnz)) == bsa.BSA_EINVAL
    with pytest.raises(ValueError):
        bsa.bsa_mask_stripes(1, 2, T, Hs, Ws, block, [(0, 0, 0, 0, 0, 0)])


def test_window_special_case_through_the_library(bsa):
    import oracle.masks as om
    T, Hs, Ws, block = 21, 30, 52, 128
    rp, ci = bsa.bsa_mask_stripes(1, 1, T, Hs, Ws, block, [(2, 0, 0, Hs, 0, 0)])
    want_rp, want_ci = om.window_anchor_csr(1, 1, T * Hs * Ws, block, Hs * Ws, 2, 0, 0)
    np.testing.assert_array_equal(rp.numpy(), want_rp)
    np.testing.assert_array_equal(ci.numpy(), want_ci)
