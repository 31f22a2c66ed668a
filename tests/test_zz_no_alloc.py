"""The allocation-free routing entry point (bsa_route_static).

Some callers cannot allocate device memory when they route -- their device
memory belongs to their own arena.  bsa_route_static serves them from a fixed device
array owned by the library.  These tests call it through the C ABI twice in a
row, on different inputs, and require the same masks, L_h and nnz as
bsa_route with a caller workspace (bit-exact, the routing tolerance).  The
file sorts last so that a stop-at-first-failure run has done everything else.
"""
import numpy as np
import pytest
import torch

import synthetic as syn
from _gpu import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_top_b200 import build
    build.build()
    import block_sparse_attention_top_b200 as m
    return m


def _outputs(plan):
    dev = "cuda"
    return (torch.full((plan.rows + 1,), -7, dtype=torch.int32, device=dev),
            torch.full((plan.rows * plan.nb,), -7, dtype=torch.int32, device=dev),
            torch.full((plan.B * plan.H,), -7.0, dtype=torch.float32, device=dev),
            torch.full((1,), -7, dtype=torch.int64, device=dev))


def _host(rp, ci, L, nnz):
    n = int(nnz.item())
    return rp.cpu().numpy(), ci[:n].cpu().numpy(), L.cpu().numpy(), n


@pytest.mark.parametrize("cid", [2, 1])
def test_static_scratch_matches_workspace_twice(bsa, cid):
    w = syn.workload(cid)
    plan = bsa.Plan(w.B, w.H, w.T, w.Hs, w.Ws, w.d, w.block)
    dtype = bsa.BSA_BF16 if w.dtype == "bf16" else bsa.BSA_F32
    ws = plan.workspace(bsa.BSA_OP_ROUTE)
    for call, seed in enumerate((syn.seed_for(cid), syn.seed_for(cid) + 17)):
        x = syn.make_inputs(w, seed=seed)
        q, k = to_dev(x["q"]), to_dev(x["k"])
        ref = _outputs(plan)
        assert bsa.bsa_route(plan, q, k, dtype, w.ps[0], w.k_floor, ref[0], ref[1], ref[1].numel(), ref[2], ref[3],
                             ws) == 0
        got = _outputs(plan)
        assert bsa.bsa_route_static(plan, q, k, dtype, w.ps[0], w.k_floor, got[0], got[1], got[1].numel(), got[2],
                                    got[3]) == 0
        assert bsa.bsa_last_device_error(plan) == 0
        a, b = _host(*ref), _host(*got)
        assert a[3] == b[3], f"call {call}: nnz differs"
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2]), call


def test_static_scratch_rejects_large_shapes(bsa):
    w = syn.workload(3)                                  # 720p: route scratch ~190 MB > 32 MiB
    plan = bsa.Plan(w.B, w.H, w.T, w.Hs, w.Ws, w.d, w.block)
    assert plan.workspace_size(bsa.BSA_OP_ROUTE) > 32 << 20
    rp, ci, L, nnz = (torch.empty(16, dtype=t, device="cuda") for t in (torch.int32, torch.int32, torch.float32,
                                                                         torch.int64))
    q = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    assert bsa.bsa_route_static(plan, q, q, bsa.BSA_BF16, 0.9, 4, rp, ci, ci.numel(), L, nnz) == bsa.BSA_EWORKSPACE
