"""The C-ABI library loads, exports every declared symbol, and validates
arguments on the host (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsa.h")


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_top_b200 import build
    build.build()
    import block_sparse_attention_top_b200 as m
    return m


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z0-9_]+)\s*\(", text)))


def test_header_symbols_exported(bsa):
    names = declared_symbols()
    assert "bsa_route" in names and "bsa_sparse_attn" in names
    out = subprocess.run(["nm", "-D", "--defined-only", bsa.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (bsa_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(bsa.LIB_PATH)
    for n in names:
        getattr(lib, n)
    assert set(names) == set(bsa.EXPORTED)


def test_strerror(bsa):
    assert bsa.bsa_strerror(0) == "ok"
    for code in range(-6, 0):
        assert bsa.bsa_strerror(code) not in ("", "unknown status")
    assert bsa.bsa_strerror(-99) == "unknown status"


@pytest.mark.parametrize("T,Hs,Ws", [(1, 1, 1), (2, 3, 5), (4, 16, 16), (21, 30, 52), (2, 45, 80), (1, 64, 64)])
def test_library_token_order_matches_oracle(bsa, T, Hs, Ws):
    """The library computes cell -> curve index and sorts; the oracle enumerates
    the curve.  Two constructions of the same order must agree exactly."""
    import oracle
    got = bsa.bsa_token_order(T, Hs, Ws).numpy().astype(np.int64)
    assert np.array_equal(got, oracle.frame_hilbert_perm(T, Hs, Ws))
    ident = bsa.bsa_token_order(T, Hs, Ws, bsa.BSA_ORDER_IDENTITY).numpy()
    assert np.array_equal(ident, np.arange(T * Hs * Ws))


def test_token_order_rejects_bad_args(bsa):
    out = torch.empty(16, dtype=torch.int32)
    assert bsa._lib.bsa_token_order(0, 4, 4, 0, out.data_ptr()) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_token_order(1, 4, 4, 7, out.data_ptr()) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_token_order(1, 4, 4, 0, None) == bsa.BSA_EINVAL


@pytest.mark.parametrize("args,code", [
    ((0, 2, 1, 4, 4, 64, 64, 0), -1),
    ((1, 2, 1, 4, 4, 64, 64, 5), -1),
    ((1, 2, 1, 4, 4, 96, 64, 0), -2),
    ((1, 2, 1, 4, 4, 64, 32, 0), -2),
    ((1, 2, 1, -4, 4, 64, 64, 0), -1),
])
def test_plan_create_validates_before_cuda(bsa, args, code):
    h = ctypes.c_void_p(123)
    assert bsa._lib.bsa_plan_create(ctypes.byref(h), *args) == code
    assert h.value is None


def test_null_plan_calls(bsa):
    assert bsa._lib.bsa_workspace_size(None, 0) == 0
    assert bsa._lib.bsa_route(None, None, None, 0, 0.9, 1, None, None, 0, None, None, None, 0, None) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_sparse_attn(None, None, None, None, None, None, None, None, 0, None) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_sparse_attn_fp8v(None, None, None, None, None, None, None, None, 0, None) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_attn_prepare_fp8v(None, None, None, None, None, None, 0, None) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_attn_run_fp8v(None, None, None, None, None, 0, None) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_attn_prepare(None, None, None, None, None, None, 0, None) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_attn_run(None, None, None, None, None, 0, None) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_augment(None, None, None, None, None, None, 0, None, None, None, 0, None) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_mask_window_anchor(None, 2, 8, 0, None, None, 0, None, None, 0, None) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_last_device_error(None, None) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_plan_info(None, None, None, None) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_plan_set_schedule(None, 0) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_plan_set_wait_limit(None, 0) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_mask_stripes_device(None, None, None, None, 0, None, None, 0, None) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_schedule_balance(None, None, None, None, None, None) == bsa.BSA_EINVAL
    assert bsa._lib.bsa_attn_intermediates(None, None, None, None, None) == bsa.BSA_EINVAL


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_plan_create_without_gpu_reports_cuda_error(bsa):
    h = ctypes.c_void_p()
    assert bsa._lib.bsa_plan_create(ctypes.byref(h), 1, 2, 4, 16, 16, 64, 64, 0) == bsa.BSA_ECUDA
    with pytest.raises(bsa.BsaError):
        bsa.Plan(1, 2, 4, 16, 16, 64, 64)


def test_sasa_budget_host_matches_oracle(bsa):
    """bsa_sasa_budget is host-only: Eqs. 7-10 against the oracle, and the per-head split."""
    import numpy as np
    import oracle.sasa as sasa
    rng = np.random.default_rng(4)
    for _ in range(50):
        R = int(rng.integers(1, 9))
        L = rng.uniform(1, 30, size=R).astype(np.float32)
        n1, n2, S = float(rng.uniform(0, 1)), float(rng.uniform(0, 0.2)), float(rng.uniform(0, 1))
        heads = rng.integers(1, 6, size=R)
        B, La, A, ex = bsa.bsa_sasa_budget(L, n1, n2, S, heads)
        ref = sasa.budget(L.astype(np.float64), np.float32(n1), np.float32(n2), np.float32(S))
        assert np.allclose(B.numpy(), ref["B"], rtol=1e-5, atol=1e-5)
        assert np.allclose(La.numpy(), ref["L_aug"], rtol=1e-5, atol=1e-5)
        assert abs(A - ref["A"]) < 1e-4
        assert list(ex.numpy()) == list(sasa.extra_per_head(B.numpy().astype(np.float64), heads))
    assert bsa._lib.bsa_sasa_budget(0, None, 0.8, 0.07, 0.0, None, None, None, None, None) == bsa.BSA_EINVAL
