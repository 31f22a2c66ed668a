"""The attention kernels' bounded waits: a wait limit of 0 makes the first wait
that is not already satisfied run out, the call reports BSA_EDEVICE through the
plan's error word (no trap, no hang), and the next call with the default limit
computes the right answer on the same plan and device."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from _gpu import bf16_to_f64, to_dev
from _parity import check_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_top_b200 import build
    build.build()
    import block_sparse_attention_top_b200 as m
    return m


@pytest.mark.parametrize("block,fp8", [(128, False), (128, True), (64, False)])
def test_expired_wait_reported_then_recovers(bsa, block, fp8):
    w = syn.workload(2, T=3, Hs=16, Ws=16, H=2, d=128, block=block)
    x = syn.make_inputs(w, seed=17)
    m = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, 0.8, 2)
    plan = bsa.Plan(w.B, w.H, w.T, w.Hs, w.Ws, w.d, w.block)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    rp = torch.from_numpy(m.row_ptr.astype(np.int32)).cuda()
    ci = torch.from_numpy(m.col_idx.astype(np.int32)).cuda()
    ws = plan.workspace(bsa.BSA_OP_ATTN)
    o = torch.zeros_like(q)
    call = bsa.bsa_sparse_attn_fp8v if fp8 else bsa.bsa_sparse_attn
    plan.set_wait_limit(0)
    assert call(plan, q, k, v, rp, ci, o, ws) == bsa.BSA_OK          # launched
    assert bsa.bsa_last_device_error(plan) == bsa.BSA_EDEVICE          # and gave up, recorded
    assert bsa.bsa_last_device_error(plan) == bsa.BSA_OK               # reading clears the word
    plan.set_wait_limit(4_000_000_000)
    o = torch.full_like(q, float("nan"))
    assert call(plan, q, k, v, rp, ci, o, ws) == bsa.BSA_OK
    assert bsa.bsa_last_device_error(plan) == bsa.BSA_OK
    got = bf16_to_f64(o)
    assert np.isfinite(got).all()
    if not fp8:
        ref = oracle.sparse_attention(x["q"], x["k"], x["v"], w.T, w.Hs, w.Ws, w.block, m.row_ptr, m.col_idx)
        check_attention(got, ref)
