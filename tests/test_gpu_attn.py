"""GPU block-sparse attention (bsa_sparse_attn and the SIMT cross-check)
against the oracle, on masks the oracle produced (or the fixed window mask)."""
import numpy as np
import pytest
import torch

import oracle
import oracle.masks as om
import synthetic as syn
from _gpu import bf16_to_f64, to_dev
from _parity import check_attention, sample_blocks

pytestmark = pytest.mark.gpu

KERNELS = ["tc", "simt"]


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_top_b200 import build
    build.build()
    import block_sparse_attention_top_b200 as m
    return m


def as_bf16_bits(x):
    return x if x.dtype == np.uint16 else syn.f32_to_bf16_bits(x)


def gpu_attn(bsa, w, qb, kb, vb, row_ptr, col_idx, kernel, order=0):
    plan = bsa.Plan(w.B, w.H, w.T, w.Hs, w.Ws, w.d, w.block, order)
    q, k, v = to_dev(qb), to_dev(kb), to_dev(vb)
    rp = torch.from_numpy(np.asarray(row_ptr, dtype=np.int32)).cuda()
    ci = torch.from_numpy(np.asarray(col_idx, dtype=np.int32).reshape(-1)).cuda()
    if ci.numel() == 0:
        ci = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = plan.workspace(bsa.BSA_OP_ATTN)
    o = torch.full_like(q, float("nan"))
    if kernel == "tc":
        assert bsa.bsa_sparse_attn(plan, q, k, v, rp, ci, o, ws) == 0
    else:
        assert bsa.bsa_attn_prepare(plan, q, k, v, rp, ws) == 0
        assert bsa.bsa_attn_run_simt(plan, rp, ci, o, ws) == 0
    status = bsa.bsa_last_device_error(plan)
    return o, status


def oracle_rows(w, qb, kb, vb, row_ptr, col_idx, rows, order="hilbert"):
    """Oracle outputs for sampled query blocks: list of (token ids, head, values)."""
    perm = oracle.token_perm(w.T, w.Hs, w.Ws, order)
    res = []
    for r in rows:
        bh, i = divmod(int(r), w.nb)
        b, h = divmod(bh, w.H)
        vals = oracle.attend_block(qb, kb, vb, perm, w.block, row_ptr, col_idx, w.H, b, h, i)
        toks = perm[i * w.block:min(w.N, (i + 1) * w.block)]
        res.append((b, toks, h, vals))
    return res


def compare_rows(o, ref_rows):
    got, want = [], []
    on = None
    for b, toks, h, vals in ref_rows:
        got.append(bf16_to_f64(o[b, torch.from_numpy(toks).cuda(), h, :]))
        want.append(vals)
    return check_attention(np.concatenate(got), np.concatenate(want))


@pytest.mark.parametrize("kernel", KERNELS)
def test_tiny_full(bsa, kernel):
    w = syn.workload(1)
    x = syn.make_inputs(w, seed=syn.seed_for(1))
    ref_mask = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, 0.9, 2)
    qb, kb, vb = (as_bf16_bits(x[n]) for n in "qkv")
    o, status = gpu_attn(bsa, w, qb, kb, vb, ref_mask.row_ptr, ref_mask.col_idx, kernel)
    assert status == 0
    ref = oracle.sparse_attention(qb, kb, vb, w.T, w.Hs, w.Ws, w.block, ref_mask.row_ptr, ref_mask.col_idx)
    print(check_attention(bf16_to_f64(o), ref))


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("shape", [
    dict(T=1, Hs=5, Ws=7, H=3, d=64, block=64),
    dict(T=3, Hs=7, Ws=9, H=2, d=128, block=64),
    dict(T=2, Hs=33, Ws=17, H=2, d=64, block=128),
    dict(T=3, Hs=16, Ws=16, H=2, d=128, block=128),
    dict(T=4, Hs=30, Ws=52, H=2, d=128, block=128),
])
@pytest.mark.parametrize("p", [0.6, 1.0])
def test_small_shapes_full(bsa, kernel, shape, p):
    w = syn.workload(2, **shape)
    x = syn.make_inputs(w, seed=21)
    m = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, p, 1)
    o, status = gpu_attn(bsa, w, x["q"], x["k"], x["v"], m.row_ptr, m.col_idx, kernel)
    assert status == 0
    ref = oracle.sparse_attention(x["q"], x["k"], x["v"], w.T, w.Hs, w.Ws, w.block, m.row_ptr, m.col_idx)
    check_attention(bf16_to_f64(o), ref)
    if p == 1.0:
        check_attention(bf16_to_f64(o), oracle.dense_attention(x["q"], x["k"], x["v"]))


@pytest.mark.parametrize("kernel", KERNELS)
def test_identity_order_and_user_mask(bsa, kernel):
    """Arbitrary column order, a row with no key block (zeros), identity token order."""
    w = syn.workload(2, T=2, Hs=20, Ws=24, H=2, block=128)
    x = syn.make_inputs(w, seed=8)
    rng = np.random.default_rng(1)
    rows, nb = w.rows, w.nb
    counts = rng.integers(1, nb + 1, size=rows)
    counts[3] = 0
    cols = [rng.permutation(nb)[:c] for c in counts]
    row_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    col_idx = np.concatenate(cols).astype(np.int64)
    o, status = gpu_attn(bsa, w, x["q"], x["k"], x["v"], row_ptr, col_idx, kernel, order=1)
    assert status == 0
    keep = [r for r in range(rows) if counts[r] > 0]
    ref_rows = oracle_rows(w, x["q"], x["k"], x["v"], row_ptr, col_idx, keep, order="identity")
    compare_rows(o, ref_rows)
    # row 3 = (b0, h0, block 3) has no keys: zeros
    toks = np.arange(3 * w.block, min(w.N, 4 * w.block))
    assert torch.all(o[0, torch.from_numpy(toks).cuda(), 0, :] == 0)


@pytest.mark.parametrize("kernel", KERNELS)
def test_stripe_mask(bsa, kernel):
    """A PSA stripe mask from the host producer (every-other-frame stripes of
    half-width 1 frame, rows within 4 of the query's) through the attention."""
    w = syn.workload(2, T=6, Hs=12, Ws=16, H=2, block=128)
    x = syn.make_inputs(w, seed=9)
    params = [(1, 0, 2, 4, 0, 0), (0, 1, 0, w.Hs, 0, 0)]
    rp, ci = bsa.bsa_mask_stripes(w.B, w.H, w.T, w.Hs, w.Ws, w.block, params)
    row_ptr, col_idx = rp.numpy().astype(np.int64), ci.numpy().astype(np.int64)
    o, status = gpu_attn(bsa, w, x["q"], x["k"], x["v"], row_ptr, col_idx, kernel)
    assert status == 0
    counts = np.diff(row_ptr)
    keep = [r for r in range(w.rows) if counts[r] > 0]
    compare_rows(o, oracle_rows(w, x["q"], x["k"], x["v"], row_ptr, col_idx, keep))
    for r in range(w.rows):                      # rows without a key block are zeros
        if counts[r] == 0:
            bh, i = divmod(r, w.nb)
            b, h = divmod(bh, w.H)
            toks = oracle.token_perm(w.T, w.Hs, w.Ws)[i * w.block:min(w.N, (i + 1) * w.block)]
            assert torch.all(o[b, torch.from_numpy(toks).cuda(), h, :] == 0)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("block", [64, 128])
def test_malformed_mask_reported(bsa, kernel, block):
    w = syn.workload(2, T=1, Hs=16, Ws=block // 4, H=1, block=block)        # four query blocks
    x = syn.make_inputs(w, seed=2)
    nb = w.nb
    row_ptr = np.array([0, 2, 4, 5, 6], dtype=np.int64)
    col_idx = np.array([0, 1, 2, nb + 5, 3, -1], dtype=np.int64)     # two bad columns
    o, status = gpu_attn(bsa, w, x["q"], x["k"], x["v"], row_ptr, col_idx, kernel)
    assert status == bsa.BSA_EDEVICE
    # rows 0 and 2 are well-formed and still computed
    ref_rows = oracle_rows(w, x["q"], x["k"], x["v"], row_ptr, col_idx, [0, 2])
    compare_rows(o, ref_rows)


@pytest.mark.parametrize("kernel", ["tc"])
@pytest.mark.parametrize("cid,p_index", [(2, 0), (3, 0), (3, 1), (3, 2), (4, 0)])
def test_full_size_routed_sampled(bsa, kernel, cid, p_index):
    w = syn.workload(cid)
    x = syn.make_inputs(w, seed=syn.seed_for(cid, p_index))
    m = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, w.ps[p_index], w.k_floor)
    o, status = gpu_attn(bsa, w, x["q"], x["k"], x["v"], m.row_ptr, m.col_idx, kernel)
    assert status == 0
    rows = sample_blocks(m.counts, w.B * w.H, w.nb, n=64, seed=cid)
    print(compare_rows(o, oracle_rows(w, x["q"], x["k"], x["v"], m.row_ptr, m.col_idx, rows)))


@pytest.mark.parametrize("kernel", ["tc"])
@pytest.mark.parametrize("step", [0, 1, 2])
def test_long_fixed_mask_sampled(bsa, kernel, step):
    w = syn.workload(5)
    x = syn.make_inputs(w, seed=syn.seed_for(5))
    row_ptr, col_idx = om.window_anchor_csr(w.B, w.H, w.N, w.block, w.Hs * w.Ws, 2, 8, step)
    o, status = gpu_attn(bsa, w, x["q"], x["k"], x["v"], row_ptr, col_idx, kernel)
    assert status == 0
    counts = np.diff(row_ptr)
    rows = sample_blocks(counts, w.B * w.H, w.nb, n=48, seed=step)
    print(compare_rows(o, oracle_rows(w, x["q"], x["k"], x["v"], row_ptr, col_idx, rows)))
