"""The load-balancing flow across ranks, on CPU with gloo: every rank all-gathers
the head workloads, plans independently and gets the same plan (no solve-and-
broadcast), then the planned heads move by point-to-point sends."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, hpr, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import block_sparse_attention_top_b200 as bsa
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_heads = list(range(rank * hpr, (rank + 1) * hpr))
        g = torch.Generator().manual_seed(100 + rank)
        L_local = torch.rand(hpr, generator=g) * 10 + (8.0 if rank == 0 else 0.0)     # rank 0 overloaded
        gathered = [torch.empty(hpr) for _ in range(world)]
        dist.all_gather(gathered, L_local)
        L_h = torch.cat(gathered)
        owner = [h // hpr for h in range(world * hpr)]
        moves, L_new, rho_b, rho_a = bsa.bsa_rlb_plan(L_h.tolist(), owner, world)
        # per-head payload [B=1, N=3, H_local, d=2] whose values name the head
        x = torch.stack([torch.full((1, 3, 2), float(h)) for h in local_heads], dim=2)
        x2, heads2 = bsa.migrate_heads(x, local_heads, moves, rank)
        ok = all(float(x2[0, 0, i, 0]) == float(h) for i, h in enumerate(heads2))
        q.put((rank, moves, [round(v, 5) for v in L_new.tolist()], heads2, ok, rho_b, rho_a))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,hpr", [(2, 3), (4, 5)])
def test_all_ranks_plan_alike_and_heads_move(world, hpr):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, hpr, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {r[0]: r[1:] for r in (q.get(timeout=120) for _ in range(world))}
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    plans = [res[r][0] for r in range(world)]
    assert all(p == plans[0] for p in plans)                      # identical, independently computed
    assert all(res[r][1] == res[0][1] for r in range(world))
    assert all(res[r][3] for r in range(world))                   # payloads arrived intact
    # the heads each rank holds afterwards follow the plan
    owner = {h: h // hpr for h in range(world * hpr)}
    for src, dst, h in plans[0]:
        owner[h] = dst
    for r in range(world):
        assert sorted(res[r][2]) == sorted(h for h, o in owner.items() if o == r)
    assert res[0][5] <= res[0][4]                                 # rho does not grow


def _step_worker(rank, world, port, hpr, skew, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import block_sparse_attention_top_b200 as bsa
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        heads = list(range(rank * hpr, (rank + 1) * hpr))
        g = torch.Generator().manual_seed(7 + rank)
        L = (torch.rand(hpr, generator=g) * 4 + 10 + (skew if rank == 0 else 0.0)).tolist()
        x = torch.stack([torch.full((1, 2, 3), float(h)) for h in heads], dim=2)
        res = bsa.balance_step(L, heads, [x], rank, world)
        xs = res["tensors"][0]
        intact = all(float(xs[0, 0, i, 0]) == float(h) for i, h in enumerate(res["local_heads"]))
        q.put((rank, res["policy"], res["moves"], res["local_heads"], res["extra"], res["L_r_new"], intact,
               res["rho_before"], res["rho_after"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,hpr,skew,policy", [(2, 3, 30.0, 2), (4, 2, 40.0, 2), (4, 2, 0.0, None)])
def test_balance_step(world, hpr, skew, policy):
    """The whole runtime flow: every rank reaches the same decision; heads and payloads follow the
    plan; the augmentation extras are the oracle's for the post-migration loads."""
    import oracle.rlb as orlb
    import oracle.sasa as osasa
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_step_worker, args=(r, world, port, hpr, skew, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {r[0]: r[1:] for r in (q.get(timeout=120) for _ in range(world))}
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    pol, moves = res[0][0], res[0][1]
    assert all(res[r][0] == pol and res[r][1] == moves for r in range(world))
    assert pol == orlb.policy(res[0][6])
    if policy is not None:
        assert pol == policy and moves and res[0][7] < res[0][6]
    assert all(res[r][5] for r in range(world))                  # payloads intact
    owner = {h: h // hpr for h in range(world * hpr)}
    for src, dst, h in moves:
        owner[h] = dst
    for r in range(world):
        assert sorted(res[r][2]) == sorted(h for h, o in owner.items() if o == r)
    if pol >= 1:
        B = osasa.budget(res[0][4])["B"]
        want = osasa.extra_per_head(B, [hpr] * world)
        got = [e for r in range(world) for e in res[r][3]]
        assert got == list(want)
    else:
        assert all(all(e == 0 for e in res[r][3]) for r in range(world))


def _exec_worker(rank, world, port, hpr, skew, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import block_sparse_attention_top_b200 as bsa
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        heads = list(range(rank * hpr, (rank + 1) * hpr))
        g = torch.Generator().manual_seed(11 + rank)
        L = (torch.rand(hpr, generator=g) * 4 + 10 + (skew if rank == 0 else 0.0)).tolist()
        # Q, K, V of a head hold its id in every element (K = 2 id, V = 3 id)
        qx = torch.stack([torch.full((1, 4, 2), float(h)) for h in heads], dim=2)
        kx, vx = 2 * qx, 3 * qx

        def compute(q2, k2, v2, heads_now, extra):
            # the stand-in for route + attention on this rank: output of head h = 1000 h + its extra
            # blocks + a check that its Q, K, V arrived together (h, 2h, 3h)
            out = torch.empty_like(q2)
            for i, h in enumerate(heads_now):
                same = bool(torch.all(q2[:, :, i] == h) and torch.all(k2[:, :, i] == 2 * h)
                            and torch.all(v2[:, :, i] == 3 * h))
                out[:, :, i] = 1000.0 * h + extra[i] + (0.0 if same else 0.5)
            return out

        o, st = bsa.balanced_attention(qx, kx, vx, L, heads, rank, world, compute)
        q.put((rank, o[0, 0, :, 0].tolist(), st["moves"], st["local_heads"], st["extra"], st["policy"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,hpr,skew", [(2, 3, 30.0), (4, 2, 40.0), (4, 3, 0.0)])
def test_balanced_attention_restores_head_order(world, hpr, skew):
    """Rank-local execution after the migration, then the reverse migration: each rank gets back the
    outputs of its own heads, in its original head order, computed from that head's Q, K and V and
    with the augmentation the plan gave the rank that computed it."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_exec_worker, args=(r, world, port, hpr, skew, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {r[0]: r[1:] for r in (q.get(timeout=120) for _ in range(world))}
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    moves = res[0][1]
    if skew > 0:
        assert moves                                          # something moved
    extra_of = {}
    for r in range(world):
        for h, e in zip(res[r][2], res[r][3]):
            extra_of[h] = e                                   # extra of the rank that computed h
    for r in range(world):
        home = list(range(r * hpr, (r + 1) * hpr))
        assert res[r][0] == [1000.0 * h + extra_of[h] for h in home]
