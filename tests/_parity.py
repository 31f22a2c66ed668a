"""Comparison rules shared by the GPU parity tests.

Masks: bit-exact outside the oracle's ambiguity set (decisions within 1e-6
relative of a tie or of p).  Attention: max |O - O_ref| <= 2e-2 and
sum|O - O_ref| / sum|O_ref| <= 5e-3 (bf16 output against the fp64 oracle).
"""
import numpy as np

ATOL_MAX = 2e-2
MEAN_REL = 5e-3
TIE = 1e-6


def check_route(gpu_row_ptr, gpu_col_idx, gpu_L_h, gpu_nnz, ref, H_total):
    """Compare a GPU routing result (numpy arrays) with an oracle RouteResult."""
    rows = ref.counts.size
    nb = ref.nb
    assert gpu_row_ptr.shape == (rows + 1,) and gpu_row_ptr[0] == 0
    counts = np.diff(gpu_row_ptr.astype(np.int64))
    assert np.all(counts >= 1) and np.all(counts <= nb)
    assert int(gpu_nnz) == int(gpu_row_ptr[-1])
    amb = ref.ambiguous
    bad = np.nonzero((counts != ref.counts) & ~amb)[0]
    assert bad.size == 0, f"{bad.size} unambiguous rows differ in count, e.g. row {bad[:5]}"
    assert np.all(np.abs(counts - ref.counts)[amb] <= 1)
    mism = []
    for r in range(rows):
        g = gpu_col_idx[gpu_row_ptr[r]:gpu_row_ptr[r + 1]].astype(np.int64)
        assert np.unique(g).size == g.size and g.min() >= 0 and g.max() < nb, r
        P = ref.P[r]
        Pg = P[g]
        # importance order: non-increasing under the oracle's P, up to ties
        assert np.all(Pg[1:] <= Pg[:-1] * (1 + TIE) + 1e-300), r
        if not amb[r]:
            o = ref.col_idx[ref.row_ptr[r]:ref.row_ptr[r + 1]]
            if set(g.tolist()) != set(o.tolist()):
                mism.append(r)
        else:
            rest = np.setdiff1d(np.arange(nb), g)
            if rest.size:
                assert Pg.min() >= P[rest].max() * (1 - TIE), r
    assert not mism, f"{len(mism)} unambiguous rows differ in kept set, e.g. {mism[:5]}"
    heads_amb = amb.reshape(H_total, nb).any(axis=1)
    ok = ~heads_amb
    assert np.array_equal(gpu_L_h[ok], ref.L_h[ok])
    return float(amb.mean())


def check_attention(out, ref):
    """out, ref: arrays of the same shape (any float dtypes)."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(out - ref)
    max_abs = float(err.max()) if err.size else 0.0
    mean_rel = float(err.sum() / max(np.abs(ref).sum(), 1e-30))
    assert max_abs <= ATOL_MAX, f"max abs err {max_abs}"
    assert mean_rel <= MEAN_REL, f"mean rel err {mean_rel}"
    return max_abs, mean_rel


def sample_blocks(ref_counts, H_total, nb, n=96, seed=0):
    """Stratified query-block sample: 8 heaviest, 8 lightest, every tail block
    (last block of each head), the rest uniform with a fixed seed."""
    rows = ref_counts.size
    order = np.argsort(-ref_counts, kind="stable")
    pick = set(order[:8].tolist()) | set(order[-8:].tolist())
    pick |= {bh * nb + nb - 1 for bh in range(H_total)}
    rng = np.random.default_rng(seed)
    rest = rng.permutation(rows)
    for r in rest:
        if len(pick) >= max(n, len(pick)):
            break
        pick.add(int(r))
    return np.array(sorted(pick), dtype=np.int64)
