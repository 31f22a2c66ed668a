"""Python binding of libbsa: Top-p block routing + block-sparse attention on B200.

Argument marshalling only: every step of the path runs in the CUDA kernels of
libbsa.so (csrc/).  PyTorch supplies device memory and streams.  If the
library is missing the import fails loudly; there is no CPU path.

The functions keep the C names (bsa_route, bsa_sparse_attn, ...) and take
torch tensors where the C call takes device pointers; `Plan` wraps
bsa_plan_create / bsa_plan_destroy.  `route`, `sparse_attn` and
`sparse_attn_fp8v` are thin conveniences that allocate the outputs and the
workspace with torch.

    import torch, block_sparse_attention_top_b200 as bsa
    # q, k, v: bf16 [B, N, H, d] on cuda, N = T * Hs * Ws latent tokens
    plan = bsa.Plan(B, H, T, Hs, Ws, d, 128)             # frame-major Hilbert order
    row_ptr, col_idx, L_h, nnz = bsa.route(plan, q, k, 0.9, 4)   # Top-p 0.9, floor 4
    o = bsa.sparse_attn(plan, q, k, v, row_ptr, col_idx)        # bf16 [B, N, H, d]
    o8 = bsa.sparse_attn_fp8v(plan, q, k, v, row_ptr, col_idx)  # e4m3 P.V product
    assert bsa.bsa_last_device_error(plan) == bsa.BSA_OK
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

LIB_PATH = _build.LIB
if _build.stale():
    # missing or older than its sources: build it now, or fail loudly (there is no CPU path)
    try:
        _build.build()
    except Exception as exc:  # noqa: BLE001
        raise ImportError(f"libbsa.so at {LIB_PATH} is missing or stale and could not be built: {exc}") from exc
_lib = ctypes.CDLL(LIB_PATH)

BSA_OK, BSA_EINVAL, BSA_EUNSUPPORTED, BSA_ECAPACITY, BSA_EWORKSPACE, BSA_ECUDA, BSA_EDEVICE = 0, -1, -2, -3, -4, -5, -6
BSA_ORDER_HILBERT2D_FRAME, BSA_ORDER_IDENTITY = 0, 1
BSA_BF16, BSA_F32 = 0, 1
BSA_OP_ROUTE, BSA_OP_ATTN, BSA_OP_MASK, BSA_OP_AUGMENT = 0, 1, 2, 3
BSA_SCHED_L2_HEADS, BSA_SCHED_HEAVIEST_FIRST, BSA_SCHED_IN_ORDER = 0, 1, 2

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t

_SIGS = {
    "bsa_plan_create": (_I, [ctypes.POINTER(_P), _I, _I, _I, _I, _I, _I, _I, _I]),
    "bsa_plan_destroy": (None, [_P]),
    "bsa_plan_info": (_I, [_P, ctypes.POINTER(_I64), ctypes.POINTER(_I64), ctypes.POINTER(_I64)]),
    "bsa_plan_set_schedule": (_I, [_P, _I]),
    "bsa_plan_set_wait_limit": (_I, [_P, ctypes.c_uint64]),
    "bsa_schedule_balance": (_I, [_P, _P, _P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I64),
                                  ctypes.POINTER(ctypes.c_double)]),
    "bsa_attn_intermediates": (_I, [_P, _P, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_P)]),
    "bsa_token_order": (_I, [_I, _I, _I, _I, _P]),
    "bsa_workspace_size": (_SZ, [_P, _I]),
    "bsa_route": (_I, [_P, _P, _P, _I, ctypes.c_float, _I, _P, _P, _I64, _P, _P, _P, _SZ, _P]),
    "bsa_route_static": (_I, [_P, _P, _P, _I, ctypes.c_float, _I, _P, _P, _I64, _P, _P, _P]),
    "bsa_route_intermediates": (_I, [_P, _P, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_P)]),
    "bsa_mask_window_anchor": (_I, [_P, _I, _I, _I, _P, _P, _I64, _P, _P, _SZ, _P]),
    "bsa_route_order": (_I, [_P, _P, ctypes.POINTER(_P)]),
    "bsa_augment": (_I, [_P, _P, _P, _P, _P, _P, _I64, _P, _P, _P, _SZ, _P]),
    "bsa_sasa_budget": (_I, [_I, _P, ctypes.c_float, ctypes.c_float, ctypes.c_float, _P, _P, _P, _P, _P]),
    "bsa_rlb_plan": (_I, [_I, _I, _P, _P, _P, ctypes.POINTER(_I), _P, _P, _P]),
    "bsa_rank_loads": (_I, [_I, _I, _P, _P, _P, _P, _P]),
    "bsa_rlb_gain": (_I, [_I, _P, _P, ctypes.c_double, ctypes.c_double, ctypes.c_double, ctypes.c_double,
                          _P, _P]),
    "bsa_mask_stripes": (_I, [_I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _I64, _P]),
    "bsa_mask_stripes_device": (_I, [_P, _P, _P, _P, _I64, _P, _P, _SZ, _P]),
    "bsa_balance_policy": (_I, [ctypes.c_float, ctypes.c_float, ctypes.c_float]),
    "bsa_sparse_attn": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "bsa_attn_prepare": (_I, [_P, _P, _P, _P, _P, _P, _SZ, _P]),
    "bsa_attn_run": (_I, [_P, _P, _P, _P, _P, _SZ, _P]),
    "bsa_attn_run_simt": (_I, [_P, _P, _P, _P, _P, _SZ, _P]),
    "bsa_sparse_attn_fp8v": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "bsa_attn_prepare_fp8v": (_I, [_P, _P, _P, _P, _P, _P, _SZ, _P]),
    "bsa_attn_run_fp8v": (_I, [_P, _P, _P, _P, _P, _SZ, _P]),
    "bsa_last_device_error": (_I, [_P, _P]),
    "bsa_strerror": (ctypes.c_char_p, [_I]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


class BsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {bsa_strerror(status)} ({status})")
        self.status = status


def bsa_strerror(status: int) -> str:
    return _lib.bsa_strerror(status).decode()


def _check(status: int, where: str) -> None:
    if status != BSA_OK:
        raise BsaError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class Plan:
    """Owns a bsa_plan for one (B, H, T, Hs, Ws, head_dim, block, order) shape."""

    def __init__(self, B, H, T, Hs, Ws, head_dim, block, order=BSA_ORDER_HILBERT2D_FRAME):
        h = _P()
        _check(_lib.bsa_plan_create(ctypes.byref(h), B, H, T, Hs, Ws, head_dim, block, order), "bsa_plan_create")
        self.handle = h
        self.B, self.H, self.T, self.Hs, self.Ws, self.d, self.block, self.order = B, H, T, Hs, Ws, head_dim, block, order
        n, nb, rows = _I64(), _I64(), _I64()
        _check(_lib.bsa_plan_info(h, ctypes.byref(n), ctypes.byref(nb), ctypes.byref(rows)), "bsa_plan_info")
        self.N, self.nb, self.rows = n.value, nb.value, rows.value

    def set_schedule(self, schedule: int) -> None:
        _check(_lib.bsa_plan_set_schedule(self.handle, int(schedule)), "bsa_plan_set_schedule")

    def set_wait_limit(self, ns: int) -> None:
        _check(_lib.bsa_plan_set_wait_limit(self.handle, int(ns)), "bsa_plan_set_wait_limit")

    def workspace_size(self, op: int) -> int:
        return int(_lib.bsa_workspace_size(self.handle, op))

    def workspace(self, op: int, device="cuda") -> torch.Tensor:
        return torch.empty(self.workspace_size(op), dtype=torch.uint8, device=device)

    def close(self):
        if getattr(self, "handle", None):
            _lib.bsa_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def bsa_schedule_balance(plan, row_ptr, work):
    """Per-CTA load balance of a work list (host tensors or arrays): (rho, max blocks, mean blocks)."""
    rp = torch.as_tensor(row_ptr, dtype=torch.int32).cpu().contiguous()
    wk = torch.as_tensor(work, dtype=torch.int32).cpu().contiguous()
    if rp.numel() != plan.rows + 1 or wk.numel() != plan.rows:
        raise ValueError("row_ptr must hold rows + 1 entries and work rows entries")
    rho, mx, mean = ctypes.c_double(), _I64(), ctypes.c_double()
    _check(_lib.bsa_schedule_balance(plan.handle, rp.data_ptr(), wk.data_ptr(), ctypes.byref(rho), ctypes.byref(mx),
                                     ctypes.byref(mean)), "bsa_schedule_balance")
    return rho.value, mx.value, mean.value


def bsa_attn_intermediates(plan, workspace):
    """Device addresses of (work list, e4m3 V tiles, V scales) in a prepared attention workspace."""
    a, b, c = _P(), _P(), _P()
    _check(_lib.bsa_attn_intermediates(plan.handle, _ptr(workspace), ctypes.byref(a), ctypes.byref(b),
                                       ctypes.byref(c)), "bsa_attn_intermediates")
    return a.value, b.value, c.value


def bsa_token_order(T: int, Hs: int, Ws: int, order: int = BSA_ORDER_HILBERT2D_FRAME):
    """Host-only token permutation (int32 CPU tensor)."""
    out = torch.empty(T * Hs * Ws, dtype=torch.int32)
    _check(_lib.bsa_token_order(T, Hs, Ws, order, out.data_ptr()), "bsa_token_order")
    return out


def bsa_route(plan, q, k, dtype, p, k_floor, row_ptr, col_idx, col_cap, L_h, nnz, workspace, stream=None):
    return _lib.bsa_route(plan.handle, _ptr(q), _ptr(k), dtype, float(p), int(k_floor), _ptr(row_ptr),
                          _ptr(col_idx), int(col_cap), _ptr(L_h), _ptr(nnz), _ptr(workspace),
                          workspace.numel() if workspace is not None else 0, _stream(stream))


def bsa_route_static(plan, q, k, dtype, p, k_floor, row_ptr, col_idx, col_cap, L_h, nnz, stream=None):
    """bsa_route with the library's fixed device scratch instead of a caller workspace
    (for callers that cannot allocate when they route)."""
    return _lib.bsa_route_static(plan.handle, _ptr(q), _ptr(k), dtype, float(p), int(k_floor), _ptr(row_ptr),
                                 _ptr(col_idx), int(col_cap), _ptr(L_h), _ptr(nnz), _stream(stream))


def bsa_mask_window_anchor(plan, radius_frames, n_anchor, step, row_ptr, col_idx, col_cap, nnz, workspace,
                           stream=None):
    return _lib.bsa_mask_window_anchor(plan.handle, int(radius_frames), int(n_anchor), int(step), _ptr(row_ptr),
                                       _ptr(col_idx), int(col_cap), _ptr(nnz), _ptr(workspace),
                                       workspace.numel() if workspace is not None else 0, _stream(stream))


def bsa_route_order(plan, workspace):
    """Device address of the full importance order (uint16 [rows, nb]) in a route workspace."""
    out = _P()
    _check(_lib.bsa_route_order(plan.handle, _ptr(workspace), ctypes.byref(out)), "bsa_route_order")
    return out.value


def bsa_augment(plan, row_ptr, order, extra, row_ptr_out, col_idx_out, col_cap, L_h_out, nnz_out, workspace,
                stream=None):
    return _lib.bsa_augment(plan.handle, _ptr(row_ptr), _ptr(order), _ptr(extra), _ptr(row_ptr_out),
                            _ptr(col_idx_out), int(col_cap), _ptr(L_h_out), _ptr(nnz_out), _ptr(workspace),
                            workspace.numel() if workspace is not None else 0, _stream(stream))


def bsa_sasa_budget(L_r, n1=0.8, n2=0.07, S=0.0, heads_per_rank=None):
    """Host-only SASA budget (Eqs. 7-10).  Returns (B_r, L_aug, A, extra_per_head or None)."""
    R = len(L_r)
    L = torch.tensor(list(L_r), dtype=torch.float32)
    B = torch.empty(R, dtype=torch.float32)
    La = torch.empty(R, dtype=torch.float32)
    A = torch.empty(1, dtype=torch.float32)
    hp = ex = None
    if heads_per_rank is not None:
        hp = torch.tensor(list(heads_per_rank), dtype=torch.int32)
        ex = torch.empty(int(hp.sum()), dtype=torch.int32)
    _check(_lib.bsa_sasa_budget(R, L.data_ptr(), float(n1), float(n2), float(S), B.data_ptr(), La.data_ptr(),
                                A.data_ptr(), _ptr(hp), _ptr(ex)), "bsa_sasa_budget")
    return B, La, float(A[0]), ex


def bsa_rlb_plan(L_h, head_rank, R):
    """Host-only load-balancing plan: (moves [(src, dst, head)], L_r_new, rho_before, rho_after)."""
    Lh = torch.tensor(list(L_h), dtype=torch.float32)
    hr = torch.tensor(list(head_rank), dtype=torch.int32)
    moves = torch.empty(3 * R, dtype=torch.int32)
    n = _I()
    Ln = torch.empty(R, dtype=torch.float32)
    rb, ra = torch.empty(1), torch.empty(1)
    _check(_lib.bsa_rlb_plan(R, Lh.numel(), hr.data_ptr(), Lh.data_ptr(), moves.data_ptr(), ctypes.byref(n),
                             Ln.data_ptr(), rb.data_ptr(), ra.data_ptr()), "bsa_rlb_plan")
    mv = moves[:3 * n.value].view(-1, 3).tolist()
    return [tuple(m) for m in mv], Ln, float(rb[0]), float(ra[0])


def bsa_rank_loads(L_h, head_rank, R):
    """Host-only per-rank loads (Eq. 1), imbalance factor rho (Eq. 2) and head counts of a placement:
    returns (L_r float32 [R], rho, heads_per_rank int32 [R])."""
    Lh = torch.tensor([float(v) for v in L_h], dtype=torch.float32)
    hr = torch.tensor([int(v) for v in head_rank], dtype=torch.int32)
    if Lh.shape != hr.shape:
        raise ValueError("L_h and head_rank must have the same length")
    L_r = torch.empty(R, dtype=torch.float32)
    cnt = torch.empty(R, dtype=torch.int32)
    rho = ctypes.c_float()
    _check(_lib.bsa_rank_loads(int(R), Lh.numel(), hr.data_ptr(), Lh.data_ptr(), L_r.data_ptr(), ctypes.byref(rho),
                               cnt.data_ptr()), "bsa_rank_loads")
    return L_r, rho.value, cnt


def bsa_rlb_gain(L_r, L_r_new, c, P=0.0, C=0.0, A=0.0):
    """(K, G) of the review's gain model (Eqs. 3-4, 11) for rank loads before and after a plan."""
    a = torch.tensor([float(v) for v in L_r], dtype=torch.float32)
    b = torch.tensor([float(v) for v in L_r_new], dtype=torch.float32)
    if a.shape != b.shape:
        raise ValueError("L_r and L_r_new must have the same length")
    K, G = ctypes.c_double(), ctypes.c_double()
    _check(_lib.bsa_rlb_gain(a.numel(), a.data_ptr(), b.data_ptr(), float(c), float(P), float(C), float(A),
                             ctypes.byref(K), ctypes.byref(G)), "bsa_rlb_gain")
    return K.value, G.value


def bsa_mask_stripes(B, H, T, Hs, Ws, block, params, order=0):
    """Host stripe-mask CSR (row_ptr, col_idx) as int32 CPU tensors; params: H rows of
    (w_t, o_t, s_t, w_s, o_s, s_s)."""
    pr = torch.tensor([[int(v) for v in row] for row in params], dtype=torch.int32).reshape(-1)
    if pr.numel() != 6 * H:
        raise ValueError("params must hold 6 values per head")
    nb = -(-(T * Hs * Ws) // block)
    rows = B * H * nb
    row_ptr = torch.empty(rows + 1, dtype=torch.int32)
    nnz = ctypes.c_int64()
    cap = rows * nb                                   # every block kept: cannot overflow
    col_idx = torch.empty(max(cap, 1), dtype=torch.int32)
    _check(_lib.bsa_mask_stripes(B, H, T, Hs, Ws, block, order, pr.data_ptr(), row_ptr.data_ptr(),
                                 col_idx.data_ptr(), cap, ctypes.byref(nnz)), "bsa_mask_stripes")
    return row_ptr, col_idx[:nnz.value].clone()


def bsa_mask_stripes_device(plan, params, row_ptr, col_idx, col_cap, nnz, workspace, stream=None):
    """Device stripe-mask CSR into device row_ptr / col_idx / nnz; params: H rows of
    (w_t, o_t, s_t, w_s, o_s, s_s) (host)."""
    pr = torch.tensor([[int(v) for v in row] for row in params], dtype=torch.int32).reshape(-1)
    if pr.numel() != 6 * plan.H:
        raise ValueError("params must hold 6 values per head")
    return _lib.bsa_mask_stripes_device(plan.handle, pr.data_ptr(), _ptr(row_ptr), _ptr(col_idx), int(col_cap),
                                        _ptr(nnz), _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                        _stream(stream))


def bsa_balance_policy(rho, k1=1.05, k2=1.10) -> int:
    return _lib.bsa_balance_policy(float(rho), float(k1), float(k2))


def migrate_heads(x, local_heads, moves, rank, group=None):
    """Carry out a plan's head moves with torch.distributed point-to-point sends.

    x: [B, N, H_local, d] tensor holding the heads listed in `local_heads`
    (global ids, same order); moves: [(src, dst, head)] from bsa_rlb_plan.
    Returns (x_new, local_heads_new): sent heads removed, received heads
    appended in move order.  Plumbing only: the data leaves and arrives as is.
    """
    import torch.distributed as dist
    keep = list(range(len(local_heads)))
    recv_bufs, recv_ids, reqs = [], [], []
    for src, dst, h in moves:
        if src == rank:
            i = local_heads.index(h)
            keep.remove(i)
            reqs.append(dist.isend(x[:, :, i].contiguous(), dst, group=group))
        elif dst == rank:
            buf = torch.empty_like(x[:, :, 0])
            reqs.append(dist.irecv(buf, src, group=group))
            recv_bufs.append(buf)
            recv_ids.append(h)
    for q in reqs:
        q.wait()
    parts = [x[:, :, i] for i in keep] + recv_bufs
    heads = [local_heads[i] for i in keep] + recv_ids
    return torch.stack(parts, dim=2) if parts else x[:, :, :0], heads


def balance_step(L_h_local, local_heads, tensors, rank, world, group=None, k1=1.05, k2=1.10, n1=0.8, n2=0.07):
    """One step of the pages' runtime balancing across ranks (FVAttn review, section 3 "Stage 2" and
    "Stage 3", section 3.3): all-gather the per-head workloads L_h (Eq. 1), take rho (Eq. 2) and the
    enabling policy; at policy 2 every rank computes the same pair-swap plan (Eqs. 5-6, bsa_rlb_plan)
    and the planned heads move with point-to-point sends; at policy >= 1 the slack-augmentation budget
    (Eqs. 7-10, bsa_sasa_budget) becomes a_h extra blocks for every query block of each local head.

    L_h_local: workloads of `local_heads` (global head ids, same order); tensors: [B, N, H_local, d]
    tensors holding those heads (all migrated alike).  Host plumbing over the library's host calls and
    torch.distributed; nothing here computes on the device.
    Returns dict(policy, rho_before, rho_after, moves, L_r, L_r_new, tensors, local_heads, extra).
    """
    import torch.distributed as dist
    mine = (list(local_heads), [float(v) for v in L_h_local])
    every = [None] * world
    dist.all_gather_object(every, mine, group=group)
    n_heads = sum(len(hs) for hs, _ in every)
    owner, L_h = [0] * n_heads, [0.0] * n_heads
    for r, (hs, ls) in enumerate(every):
        for h, l in zip(hs, ls):
            owner[h], L_h[h] = r, l
    L_r, rho, _ = bsa_rank_loads(L_h, owner, world)
    L_r = L_r.tolist()
    policy = bsa_balance_policy(rho, k1, k2)
    moves, L_r_new, rho_after = [], list(L_r), rho
    heads = list(local_heads)
    new_owner = list(owner)
    if policy == 2:
        moves, L_new, _, rho_after = bsa_rlb_plan(L_h, owner, world)
        L_r_new = L_new.tolist()
        for src, dst, h in moves:
            new_owner[h] = dst
        out = []
        for x in tensors:
            x_new, heads_new = migrate_heads(x, list(local_heads), moves, rank, group)
            out.append(x_new)
        tensors = out
        if tensors:
            heads = heads_new
        else:                                             # no payload: the head list still follows the plan
            heads = [h for h in local_heads if not any(m[2] == h and m[0] == rank for m in moves)]
            heads += [m[2] for m in moves if m[1] == rank]
    extra = [0] * len(heads)
    if policy >= 1:
        # heads each rank holds after the migration, in the order bsa_sasa_budget lists them
        _, _, counts = bsa_rank_loads(L_h, new_owner, world)
        counts = counts.tolist()
        if counts[rank] != len(heads):
            raise RuntimeError("head bookkeeping disagrees with the plan")
        _, _, _, ex = bsa_sasa_budget(L_r_new, n1, n2, heads_per_rank=counts)
        lo = sum(counts[:rank])
        extra = ex[lo:lo + counts[rank]].tolist()
    return dict(policy=policy, rho_before=rho, rho_after=rho_after, moves=moves, L_r=L_r, L_r_new=L_r_new,
                tensors=tensors, local_heads=heads, extra=extra)


def return_heads(out, heads, home_heads, moves, rank, group=None):
    """The reverse of migrate_heads: send every migrated head's output back to the rank it came from
    and return this rank's outputs in its original head order (FVAttn review, section 3 "Block-Sparse
    Attention Execution": the outputs of migrated heads go back and head order is restored).

    out: [B, N, H_now, d] outputs of the heads listed in `heads` (the order balance_step / migrate_heads
    returned); home_heads: this rank's heads before the migration, in their original order; moves: the
    plan's [(src, dst, head)].  Returns [B, N, len(home_heads), d].  Plumbing only."""
    import torch.distributed as dist
    home_of = {h: src for src, dst, h in moves}            # heads that moved: where they live
    reqs, kept, got = [], {}, {}
    for i, h in enumerate(heads):
        if h in home_of and home_of[h] != rank:            # computed here for another rank: send it home
            reqs.append(dist.isend(out[:, :, i].contiguous(), home_of[h], group=group))
        else:
            kept[h] = out[:, :, i]
    for src, dst, h in moves:
        if src == rank:                                    # ours, computed elsewhere: receive it
            buf = torch.empty_like(out[:, :, 0]) if out.shape[2] else torch.empty(
                out.shape[:2] + out.shape[3:], dtype=out.dtype, device=out.device)
            reqs.append(dist.irecv(buf, dst, group=group))
            got[h] = buf
    for q in reqs:
        q.wait()
    parts = []
    for h in home_heads:
        if h in kept:
            parts.append(kept[h])
        elif h in got:
            parts.append(got[h])
        else:
            raise RuntimeError(f"head {h} is neither kept nor received on rank {rank}")
    return torch.stack(parts, dim=2) if parts else out[:, :, :0]


def local_attention(q, k, v, T, Hs, Ws, block, p, k_floor, extra=None):
    """Route and attend over the heads a rank holds: bf16 [B, N, H_local, d] on its device; extra: SASA
    blocks per local head (bsa_augment), or None.  Returns (o, L_h) device tensors."""
    B, N, H, d = q.shape
    plan = Plan(B, H, T, Hs, Ws, d, block)
    ws = plan.workspace(BSA_OP_ROUTE, q.device)
    row_ptr, col_idx, L_h, _ = route(plan, q, k, p, k_floor, workspace=ws)
    if extra is not None and any(int(e) > 0 for e in extra):
        ex = torch.tensor([int(e) for e in extra], dtype=torch.int32, device=q.device)
        rp2 = torch.empty_like(row_ptr)
        ci2 = torch.empty(plan.rows * plan.nb, dtype=torch.int32, device=q.device)
        L2 = torch.empty_like(L_h)
        nnz2 = torch.empty(1, dtype=torch.int64, device=q.device)
        ws_aug = plan.workspace(BSA_OP_AUGMENT, q.device)
        _check(bsa_augment(plan, row_ptr, bsa_route_order(plan, ws), ex, rp2, ci2, ci2.numel(), L2, nnz2, ws_aug),
               "bsa_augment")
        row_ptr, col_idx, L_h = rp2, ci2, L2
    o = sparse_attn(plan, q, k, v, row_ptr, col_idx)
    _check(bsa_last_device_error(plan), "device error")
    return o, L_h


def balanced_attention(q, k, v, L_h_local, local_heads, rank, world, compute, group=None, **policy):
    """One balanced attention step over the ranks (FVAttn review, section 3): balance_step moves the
    planned heads' Q, K, V and decides the augmentation, `compute(q, k, v, heads, extra)` runs the
    rank-local route + attention over the heads the rank now holds (e.g. local_attention), and
    return_heads sends the migrated heads' outputs home in the original head order.
    Returns (o [B, N, H_local, d] in `local_heads` order, the balance_step record)."""
    st = balance_step(L_h_local, local_heads, [q, k, v], rank, world, group=group, **policy)
    q2, k2, v2 = st["tensors"]
    o2 = compute(q2, k2, v2, st["local_heads"], st["extra"])
    return return_heads(o2, st["local_heads"], list(local_heads), st["moves"], rank, group), st


def bsa_route_intermediates(plan, workspace):
    a, b, c = _P(), _P(), _P()
    _check(_lib.bsa_route_intermediates(plan.handle, _ptr(workspace), ctypes.byref(a), ctypes.byref(b),
                                        ctypes.byref(c)), "bsa_route_intermediates")
    return a.value, b.value, c.value


def bsa_sparse_attn(plan, q, k, v, row_ptr, col_idx, o, workspace, stream=None):
    return _lib.bsa_sparse_attn(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr), _ptr(col_idx), _ptr(o),
                                _ptr(workspace), workspace.numel(), _stream(stream))


def bsa_attn_prepare(plan, q, k, v, row_ptr, workspace, stream=None):
    return _lib.bsa_attn_prepare(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr), _ptr(workspace),
                                 workspace.numel(), _stream(stream))


def bsa_attn_run(plan, row_ptr, col_idx, o, workspace, stream=None):
    return _lib.bsa_attn_run(plan.handle, _ptr(row_ptr), _ptr(col_idx), _ptr(o), _ptr(workspace),
                             workspace.numel(), _stream(stream))


def bsa_attn_run_simt(plan, row_ptr, col_idx, o, workspace, stream=None):
    return _lib.bsa_attn_run_simt(plan.handle, _ptr(row_ptr), _ptr(col_idx), _ptr(o), _ptr(workspace),
                                  workspace.numel(), _stream(stream))


def bsa_sparse_attn_fp8v(plan, q, k, v, row_ptr, col_idx, o, workspace, stream=None):
    return _lib.bsa_sparse_attn_fp8v(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr), _ptr(col_idx),
                                     _ptr(o), _ptr(workspace), workspace.numel(), _stream(stream))


def bsa_attn_prepare_fp8v(plan, q, k, v, row_ptr, workspace, stream=None):
    return _lib.bsa_attn_prepare_fp8v(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr), _ptr(workspace),
                                      workspace.numel(), _stream(stream))


def bsa_attn_run_fp8v(plan, row_ptr, col_idx, o, workspace, stream=None):
    return _lib.bsa_attn_run_fp8v(plan.handle, _ptr(row_ptr), _ptr(col_idx), _ptr(o), _ptr(workspace),
                                  workspace.numel(), _stream(stream))


def bsa_last_device_error(plan, stream=None) -> int:
    return _lib.bsa_last_device_error(plan.handle, _stream(stream))


# ---- conveniences (allocate outputs with torch, raise on error) ----

def route(plan: Plan, q: torch.Tensor, k: torch.Tensor, p: float, k_floor: int, workspace=None,
          col_cap: int | None = None, stream=None):
    """Returns (row_ptr, col_idx[:col_cap], L_h, nnz) device tensors; nnz stays on device."""
    dev = q.device
    dtype = BSA_BF16 if q.dtype == torch.bfloat16 else BSA_F32
    if col_cap is None:
        col_cap = plan.rows * plan.nb
    row_ptr = torch.empty(plan.rows + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(max(col_cap, 1), dtype=torch.int32, device=dev)
    L_h = torch.empty(plan.B * plan.H, dtype=torch.float32, device=dev)
    nnz = torch.empty(1, dtype=torch.int64, device=dev)
    if workspace is None:
        workspace = plan.workspace(BSA_OP_ROUTE, dev)
    _check(bsa_route(plan, q, k, dtype, p, k_floor, row_ptr, col_idx, col_cap, L_h, nnz, workspace, stream),
           "bsa_route")
    return row_ptr, col_idx, L_h, nnz


def sparse_attn(plan: Plan, q, k, v, row_ptr, col_idx, workspace=None, out=None, stream=None):
    """O = block-sparse attention of bf16 [B,N,H,d] inputs under the CSR mask."""
    if workspace is None:
        workspace = plan.workspace(BSA_OP_ATTN, q.device)
    o = torch.empty_like(q) if out is None else out
    _check(bsa_sparse_attn(plan, q, k, v, row_ptr, col_idx, o, workspace, stream), "bsa_sparse_attn")
    return o


def sparse_attn_fp8v(plan: Plan, q, k, v, row_ptr, col_idx, workspace=None, out=None, stream=None):
    """As sparse_attn, with the e4m3 P.V product (block 128 only)."""
    if workspace is None:
        workspace = plan.workspace(BSA_OP_ATTN, q.device)
    o = torch.empty_like(q) if out is None else out
    _check(bsa_sparse_attn_fp8v(plan, q, k, v, row_ptr, col_idx, o, workspace, stream), "bsa_sparse_attn_fp8v")
    return o
