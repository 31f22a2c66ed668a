"""Work-list schedules of the attention kernel (bsa_plan_set_schedule): the list
is a permutation of the rows in the stated order, the outputs do not depend on
it, and bsa_schedule_balance follows the kernels' static CTA assignment."""
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


def work_list(bsa, plan, ws):
    wptr, _, _ = bsa.bsa_attn_intermediates(plan, ws)
    off = wptr - ws.data_ptr()
    return ws[off:off + 4 * plan.rows].view(torch.int32).cpu().numpy()


def prepared_list(bsa, w, row_ptr, schedule):
    plan = bsa.Plan(w.B, w.H, w.T, w.Hs, w.Ws, w.d, w.block)
    plan.set_schedule(schedule)
    q = torch.zeros((w.B, w.N, w.H, w.d), dtype=torch.bfloat16, device="cuda")
    ws = plan.workspace(bsa.BSA_OP_ATTN)
    rp = torch.from_numpy(np.asarray(row_ptr, dtype=np.int32)).cuda()
    assert bsa.bsa_attn_prepare(plan, q, q, q, rp, ws) == 0
    assert bsa.bsa_last_device_error(plan) == 0
    return plan, work_list(bsa, plan, ws)


def heads_per_group(w):
    """The stated grouping rule: as many heads as fit 40 % of L2 with their K and V tiles."""
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    head_bytes = 2.0 * w.nb * w.block * w.d * 2.0
    return int(min(w.B * w.H, max(1, int(0.4 * l2 / head_bytes))))


@pytest.mark.parametrize("shape", [
    dict(T=21, Hs=45, Ws=80, H=5, block=128),          # 720p geometry: one head per group
    dict(T=4, Hs=30, Ws=52, H=6, block=128),           # small heads: one group
])
def test_work_list_orders(bsa, shape):
    w = syn.workload(3, **shape)
    rng = np.random.default_rng(7)
    counts = rng.integers(0, w.nb + 1, size=w.rows)
    counts[w.nb:2 * w.nb] = w.nb                        # one dense head
    row_ptr = np.concatenate([[0], np.cumsum(counts)])
    # in order
    _, wk = prepared_list(bsa, w, row_ptr, bsa.BSA_SCHED_IN_ORDER)
    assert np.array_equal(wk, np.arange(w.rows))
    # heaviest first: a permutation with non-increasing counts
    _, wk = prepared_list(bsa, w, row_ptr, bsa.BSA_SCHED_HEAVIEST_FIRST)
    assert np.array_equal(np.sort(wk), np.arange(w.rows))
    assert np.all(np.diff(counts[wk]) <= 0)
    # head groups: contiguous runs per group, groups by descending work, items by descending count
    _, wk = prepared_list(bsa, w, row_ptr, bsa.BSA_SCHED_L2_HEADS)
    assert np.array_equal(np.sort(wk), np.arange(w.rows))
    G = heads_per_group(w)
    grp = (wk // w.nb) // G
    runs = [grp[0]] + [g for a, g in zip(grp[:-1], grp[1:]) if g != a]
    n_groups = -(-w.B * w.H // G)
    assert sorted(runs) == list(range(n_groups)), "each group is one contiguous run"
    gw = np.array([counts[g * G * w.nb:(g + 1) * G * w.nb].sum() for g in range(n_groups)])
    want = sorted(range(n_groups), key=lambda g: (-gw[g], g))
    assert runs == want
    for g in range(n_groups):
        assert np.all(np.diff(counts[wk[grp == g]]) <= 0)
    if G == 1 and n_groups > 1:
        assert runs[0] == 1                             # the dense head goes first


def test_balance_follows_the_kernels_assignment(bsa):
    w = syn.workload(3, T=21, Hs=45, Ws=80, H=3, block=128)
    rng = np.random.default_rng(3)
    counts = rng.integers(1, w.nb + 1, size=w.rows)
    row_ptr = np.concatenate([[0], np.cumsum(counts)])
    plan, wk = prepared_list(bsa, w, row_ptr, bsa.BSA_SCHED_HEAVIEST_FIRST)
    rho, mx, mean = bsa.bsa_schedule_balance(plan, row_ptr, wk)
    grid = min(torch.cuda.get_device_properties(0).multi_processor_count, w.rows)
    load = np.zeros(grid, dtype=np.int64)
    for idx, r in enumerate(wk):
        k, c = divmod(idx, grid)
        load[grid - 1 - c if k & 1 else c] += counts[r]
    assert mx == load.max() and mean == pytest.approx(load.mean())
    assert rho == pytest.approx(load.max() / load.mean())
    with pytest.raises(bsa.BsaError):
        bsa.bsa_schedule_balance(plan, row_ptr, np.full(w.rows, w.rows, dtype=np.int32))


def test_outputs_do_not_depend_on_the_schedule(bsa):
    w = syn.workload(2, T=4, Hs=30, Ws=52, H=3, d=128, block=128)
    x = syn.make_inputs(w, seed=44)
    m = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, 0.7, 2)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    rp = torch.from_numpy(m.row_ptr.astype(np.int32)).cuda()
    ci = torch.from_numpy(m.col_idx.astype(np.int32)).cuda()
    outs = []
    for sched in (0, 1, 2):
        plan = bsa.Plan(w.B, w.H, w.T, w.Hs, w.Ws, w.d, w.block)
        plan.set_schedule(sched)
        ws = plan.workspace(bsa.BSA_OP_ATTN)
        o = torch.full_like(q, float("nan"))
        assert bsa.bsa_sparse_attn(plan, q, k, v, rp, ci, o, ws) == 0
        assert bsa.bsa_last_device_error(plan) == 0
        outs.append(o)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    ref = oracle.sparse_attention(x["q"], x["k"], x["v"], w.T, w.Hs, w.Ws, w.block, m.row_ptr, m.col_idx)
    check_attention(bf16_to_f64(outs[0]), ref)


def test_set_schedule_rejects_unknown(bsa):
    plan = bsa.Plan(1, 1, 1, 16, 16, 64, 64)
    with pytest.raises(bsa.BsaError):
        plan.set_schedule(3)
