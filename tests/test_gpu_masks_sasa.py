"""Device fixed-mask producer and the SASA augmentation against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import oracle.masks as om
import oracle.sasa as osasa
import synthetic as syn
from _gpu import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_top_b200 import build
    build.build()
    import block_sparse_attention_top_b200 as m
    return m


def gpu_mask(bsa, w, radius, n_anchor, step, col_cap=None):
    plan = bsa.Plan(w.B, w.H, w.T, w.Hs, w.Ws, w.d, w.block)
    cap = plan.rows * plan.nb if col_cap is None else col_cap
    rp = torch.empty(plan.rows + 1, dtype=torch.int32, device="cuda")
    ci = torch.full((max(cap, 1),), -1, dtype=torch.int32, device="cuda")
    nnz = torch.empty(1, dtype=torch.int64, device="cuda")
    ws = plan.workspace(bsa.BSA_OP_MASK)
    rc = bsa.bsa_mask_window_anchor(plan, radius, n_anchor, step, rp, ci, cap, nnz, ws)
    return rc, rp.cpu().numpy(), ci.cpu().numpy(), int(nnz.item()), bsa.bsa_last_device_error(plan)


@pytest.mark.parametrize("step", [0, 1, 2])
def test_long_horizon_mask_exact(bsa, step):
    w = syn.workload(5)
    rc, rp, ci, nnz, st = gpu_mask(bsa, w, 2, 8, step)
    assert rc == 0 and st == 0
    orp, oci = om.window_anchor_csr(w.B, w.H, w.N, w.block, w.Hs * w.Ws, 2, 8, step)
    assert np.array_equal(rp, orp) and nnz == oci.size and np.array_equal(ci[:nnz], oci)


@pytest.mark.parametrize("shape,radius,n_anchor,step", [
    (dict(T=5, Hs=7, Ws=9, H=2, block=64), 0, 0, 0),        # blocks straddle frames, ragged tail
    (dict(T=5, Hs=7, Ws=9, H=2, block=64), 1, 3, 7),
    (dict(T=3, Hs=4, Ws=4, H=1, block=64), 0, 8, 1),        # nb = 1 < n_anchor: anchors coincide
    (dict(T=12, Hs=6, Ws=10, H=3, block=128), 50, 4, 5),    # window covers everything
    (dict(T=40, Hs=3, Ws=5, H=1, block=64), 3, 64, 9),      # many anchors
])
def test_small_masks_exact(bsa, shape, radius, n_anchor, step):
    w = syn.workload(5, **shape)
    rc, rp, ci, nnz, st = gpu_mask(bsa, w, radius, n_anchor, step)
    assert rc == 0 and st == 0
    orp, oci = om.window_anchor_csr(w.B, w.H, w.N, w.block, w.Hs * w.Ws, radius, n_anchor, step)
    assert np.array_equal(rp, orp) and np.array_equal(ci[:nnz], oci)


def test_mask_errors(bsa):
    w = syn.workload(5, T=6, Hs=6, Ws=10, H=1, block=64)
    assert gpu_mask(bsa, w, 2, 65, 0)[0] == bsa.BSA_EINVAL
    assert gpu_mask(bsa, w, -1, 8, 0)[0] == bsa.BSA_EINVAL
    rc, rp, ci, nnz, st = gpu_mask(bsa, w, 2, 8, 0, col_cap=5)
    assert rc == 0 and st == bsa.BSA_ECAPACITY and nnz > 5


def _route_with_order(bsa, w, x, p, kf):
    plan = bsa.Plan(w.B, w.H, w.T, w.Hs, w.Ws, w.d, w.block)
    q, k = to_dev(x["q"]), to_dev(x["k"])
    ws = plan.workspace(bsa.BSA_OP_ROUTE)
    rp, ci, L, nnz = bsa.route(plan, q, k, p, kf, workspace=ws)
    optr = bsa.bsa_route_order(plan, ws)
    off = optr - ws.data_ptr()
    order = ws[off:off + 2 * plan.rows * plan.nb].view(torch.int16)       # uint16 indices < 8192
    return plan, ws, rp, order


@pytest.mark.parametrize("cid,extras", [(1, [0, 3]), (2, None)])
def test_augment_matches_oracle(bsa, cid, extras):
    w = syn.workload(cid)
    x = syn.make_inputs(w, seed=syn.seed_for(cid))
    p, kf = w.ps[0] - (0.3 if cid == 1 else 0.2), w.k_floor
    plan, ws, rp, order = _route_with_order(bsa, w, x, p, kf)
    heads = w.B * w.H
    extra = np.array(extras if extras is not None else [(3 * h) % 17 for h in range(heads)], dtype=np.int32)
    ex_d = torch.from_numpy(extra).cuda()
    rp_o = torch.empty(plan.rows + 1, dtype=torch.int32, device="cuda")
    ci_o = torch.empty(plan.rows * plan.nb, dtype=torch.int32, device="cuda")
    L_o = torch.empty(heads, dtype=torch.float32, device="cuda")
    nnz_o = torch.empty(1, dtype=torch.int64, device="cuda")
    wsa = plan.workspace(bsa.BSA_OP_AUGMENT)
    assert bsa.bsa_augment(plan, rp, order, ex_d, rp_o, ci_o, ci_o.numel(), L_o, nnz_o, wsa) == 0
    assert bsa.bsa_last_device_error(plan) == 0

    ref = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, p, kf)
    n_ref, rp_ref, ci_ref, L_ref = osasa.augment(ref, extra, w.nb)
    g_rp = rp_o.cpu().numpy().astype(np.int64)
    g_ci = ci_o.cpu().numpy()
    g_n = np.diff(g_rp)
    nb = w.nb
    # the full importance order: a permutation, non-increasing under the oracle's P (ties allowed)
    g_order = order.cpu().numpy().astype(np.int64).reshape(plan.rows, nb)
    for r in range(plan.rows):
        assert sorted(g_order[r]) == list(range(nb))
        P = ref.P[r][g_order[r]]
        assert np.all(P[1:] <= P[:-1] * (1 + 1e-6) + 1e-300)
    # augmented rows: exact unless the routed cut or the new cut sits on a tie
    Ps = ref.P_sorted
    checked = 0
    skip = ref.ambiguous.copy()
    for r in range(plan.rows):
        n = n_ref[r]
        skip[r] |= bool(n < nb and abs(Ps[r, n - 1] - Ps[r, n]) <= 1e-6 * Ps[r, n - 1])
        if skip[r]:
            continue
        checked += 1
        assert g_n[r] == n, r
        assert set(g_ci[g_rp[r]:g_rp[r + 1]]) == set(ci_ref[rp_ref[r]:rp_ref[r + 1]]), r
    assert checked > 0.9 * plan.rows
    heads_ok = ~skip.reshape(heads, nb).any(axis=1)
    assert np.allclose(L_o.cpu().numpy()[heads_ok], L_ref[heads_ok], rtol=0, atol=1e-6)


def _stripe_params(rng, H):
    return [(int(rng.integers(0, 3)), int(rng.integers(-3, 4)), int(rng.integers(-1, 6)),
             int(rng.integers(0, 4)), int(rng.integers(-4, 5)), int(rng.integers(-1, 8))) for _ in range(H)]


def gpu_stripes(bsa, w, params, order=0, col_cap=None):
    plan = bsa.Plan(w.B, w.H, w.T, w.Hs, w.Ws, w.d, w.block, order)
    cap = plan.rows * plan.nb if col_cap is None else col_cap
    rp = torch.empty(plan.rows + 1, dtype=torch.int32, device="cuda")
    ci = torch.full((max(cap, 1),), -1, dtype=torch.int32, device="cuda")
    nnz = torch.empty(1, dtype=torch.int64, device="cuda")
    ws = plan.workspace(bsa.BSA_OP_MASK)
    rc = bsa.bsa_mask_stripes_device(plan, params, rp, ci, cap, nnz, ws)
    return rc, rp.cpu().numpy(), ci.cpu().numpy(), int(nnz.item()), bsa.bsa_last_device_error(plan)


@pytest.mark.parametrize("shape", [(4, 2, 2, 64, 1, 1), (6, 8, 10, 64, 1, 3), (5, 9, 7, 128, 2, 2),
                                   (21, 30, 52, 128, 1, 12)])
@pytest.mark.parametrize("order", [0, 1])
def test_stripes_device_matches_oracle(bsa, shape, order):
    """PSA stripe masks made on the device equal the oracle's CSR exactly (the last
    shape is the 480p workload with twelve random heads)."""
    import oracle.stripes as ostr
    T, Hs, Ws, block, B, H = shape
    w = syn.workload(2, T=T, Hs=Hs, Ws=Ws, block=block, B=B, H=H)
    params = _stripe_params(np.random.default_rng(T * 100 + Hs + order), H)
    rc, rp, ci, nnz, st = gpu_stripes(bsa, w, params, order)
    assert rc == 0 and st == 0
    want_rp, want_ci = ostr.stripe_csr(B, H, T, Hs, Ws, block, np.array(params),
                                       order="hilbert" if order == 0 else "identity")
    np.testing.assert_array_equal(rp, want_rp)
    assert nnz == want_ci.size
    np.testing.assert_array_equal(ci[:nnz], want_ci)


def test_stripes_device_capacity_and_errors(bsa):
    w = syn.workload(2, T=6, Hs=8, Ws=10, block=64, H=1)
    rc, rp, ci, nnz, st = gpu_stripes(bsa, w, [(0, 0, 0, 8, 0, 0)], col_cap=3)
    assert rc == 0 and st == bsa.BSA_ECAPACITY and nnz > 3 and rp[-1] == nnz
    assert gpu_stripes(bsa, w, [(-1, 0, 0, 0, 0, 0)])[0] == bsa.BSA_EINVAL
    w2 = syn.workload(2, T=1, Hs=8, Ws=8, block=64, H=161)
    assert gpu_stripes(bsa, w2, [(0, 0, 0, 0, 0, 0)] * 161)[0] == bsa.BSA_EUNSUPPORTED
