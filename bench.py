"""Benchmark: Top-p block routing + block-sparse attention on B200.

One step = one pass of the whole hot path over the 480p Wan2.1-shaped workload
(B1 H12 d128, 21x30x52 = 32760 tokens, block 128, p = 0.9, k_floor = 4):
bsa_route (gather + mean-pool, block scores, row routing, CSR) then
bsa_attn_prepare (heaviest-first work list, reordered Q/K/V tiles) then
bsa_attn_run (persistent tcgen05 attention, output scattered to token order).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  `value` is effective TFLOP/s over the whole
step: retained-block attention FLOPs (sum over kept (row, block) pairs of
4 * m_i * m_j * d with the real token counts) of all ranks / max-over-ranks step
time.  N > 1 (torchrun) runs one independent replica per GPU (weak scaling, no
collective on the data path).  `--impl reference` times the fp64 CPU oracle on a
bounded sample of the same workload and extrapolates to the same unit.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as syn  # noqa: E402

CID = 2
P_INDEX = 0
METRIC = "block-sparse attn ms/call & effective TFLOP/s (% bf16 peak); routing GB/s"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNELS_PER_STEP = 10   # route: 5, prepare: 4 (hist, bins, scatter, permute), run: 1


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK), "fallback"


def workload_desc(w):
    return (f"{w.name} (config {w.cid}): B{w.B} H{w.H} d{w.d} T{w.T}x{w.Hs}x{w.Ws}={w.N} tokens, "
            f"block {w.block}, p={w.ps[P_INDEX]}, k_floor={w.k_floor}")


def attention_flops(row_ptr, col_idx, w):
    counts = np.diff(row_ptr.astype(np.int64))
    m = np.full(w.nb, w.block, dtype=np.int64)
    m[-1] = w.N - (w.nb - 1) * w.block
    rows = np.repeat(np.arange(counts.size), counts)
    cols = col_idx[: counts.sum()].astype(np.int64)
    return 4.0 * w.d * float(np.sum(m[rows % w.nb] * m[cols]))


def reduce_over_ranks(times_ms, work, world, device):
    """Whole-job view of a replicated run: the max over ranks of each timing and
    the sum over ranks of the work.  Every rank takes the same two collectives."""
    import torch
    stats = torch.tensor(list(times_ms), dtype=torch.float64, device=device)
    total = torch.tensor([float(work)], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(stats, op=torch.distributed.ReduceOp.MAX)
        torch.distributed.all_reduce(total, op=torch.distributed.ReduceOp.SUM)
    return [float(x) for x in stats.tolist()], float(total[0])


def route_bytes(w, nnz, in_bytes):
    return 2 * in_bytes + (w.rows + 1) * 4 + nnz * 4 + w.B * w.H * 4 + 8


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        busy = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- ours
def run_ours(args, rank, world, local_rank):
    import torch
    import block_sparse_attention_top_b200 as bsa

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = syn.workload(CID)
    p = w.ps[P_INDEX]
    x = syn.make_inputs(w, seed=syn.seed_for(CID, P_INDEX) + 7919 * rank)

    def to_dev(a):
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)

    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    plan = bsa.Plan(w.B, w.H, w.T, w.Hs, w.Ws, w.d, w.block)
    col_cap = plan.rows * plan.nb
    row_ptr = torch.empty(plan.rows + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(col_cap, dtype=torch.int32, device=dev)
    L_h = torch.empty(w.B * w.H, dtype=torch.float32, device=dev)
    nnz = torch.empty(1, dtype=torch.int64, device=dev)
    ws_route = plan.workspace(bsa.BSA_OP_ROUTE, dev)
    ws_attn = plan.workspace(bsa.BSA_OP_ATTN, dev)
    o = torch.empty_like(q)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)     # > 126 MB L2
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        rc = bsa.bsa_route(plan, q, k, bsa.BSA_BF16, p, w.k_floor, row_ptr, col_idx, col_cap, L_h, nnz, ws_route,
                           stream)
        if ev:
            ev[1].record(stream)
        rc |= bsa.bsa_attn_prepare(plan, q, k, v, row_ptr, ws_attn, stream)
        if ev:
            ev[2].record(stream)
        rc |= bsa.bsa_attn_run(plan, row_ptr, col_idx, o, ws_attn, stream)
        if ev:
            ev[3].record(stream)
        if rc:
            raise RuntimeError(f"bsa call failed: {rc}")

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if bsa.bsa_last_device_error(plan) != 0:
        raise RuntimeError("device error during warm-up")
    flops = attention_flops(row_ptr.cpu().numpy(), col_idx.cpu().numpy(), w)
    nnz_v = int(nnz.item())
    rbytes = route_bytes(w, nnz_v, q.numel() * 2)

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank) if rank == 0 else None
    for i in range(args.steps):
        flush.zero_()
        step(events[i])
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop() if clocks else None
    if bsa.bsa_last_device_error(plan) != 0:
        raise RuntimeError("device error during timing")
    step_ms = [e[0].elapsed_time(e[3]) for e in events]
    route_ms = [e[0].elapsed_time(e[1]) for e in events]
    prep_ms = [e[1].elapsed_time(e[2]) for e in events]
    attn_ms = [e[2].elapsed_time(e[3]) for e in events]
    total_ms = sum(step_ms)

    # the FP8 P.V variant on the same inputs and mask (reported beside the bf16 headline)
    fp8_steps = max(3, min(args.steps, 50))
    fp8_prep, fp8_run = [], []
    for i in range(fp8_steps + 2):
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        rc = bsa.bsa_attn_prepare_fp8v(plan, q, k, v, row_ptr, ws_attn, stream)
        ev[1].record(stream)
        rc |= bsa.bsa_attn_run_fp8v(plan, row_ptr, col_idx, o, ws_attn, stream)
        ev[2].record(stream)
        if rc:
            raise RuntimeError(f"fp8 attention call failed: {rc}")
        if i >= 2:
            fp8_prep.append(ev)
    torch.cuda.synchronize()
    if bsa.bsa_last_device_error(plan) != 0:
        raise RuntimeError("device error in the fp8 variant")
    fp8_prep_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in fp8_prep)
    fp8_run_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in fp8_prep)

    # end to end through the public API with pinned host buffers
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_step():
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        rp, ci, lh, nz = bsa.route(plan, qd, kd, p, w.k_floor, workspace=ws_route, col_cap=col_cap)
        bsa.sparse_attn(plan, qd, kd, vd, rp, ci, workspace=ws_attn, out=o)
        oh.copy_(o, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    (total_ms_max, e2e_ms_max, _, _), flops_sum = reduce_over_ranks(
        [total_ms, e2e_ms, max(attn_ms), max(route_ms)], flops, world, dev)
    if rank != 0:
        return None

    pk, pk_kind = peaks()
    attn_avg = statistics.mean(attn_ms)
    achieved = flops / (attn_avg * 1e-3) / 1e12
    traffic = load_traffic()
    ms_per_step = total_ms_max / args.steps
    value = flops_sum / (ms_per_step * 1e-3) / 1e12
    route_avg = statistics.mean(route_ms)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) + sinusoidal (t,y,x) features, Wan2.1-480p-shaped; no weights)",
        "config": {"workload": workload_desc(w), "global_batch": w.B * world, "seq_len": w.N,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "flushed before every timed step (256 MB write, untimed)",
                   "density": round(float(nnz_v) / (w.rows * w.nb), 4)},
        "attn_ms_per_call": round(attn_avg, 4),
        "attn_tflops": round(achieved, 2),
        "attn_frac_of_bf16_burst": round(achieved / pk["bf16_tflops"], 4),
        "route_ms_per_call": round(route_avg, 4),
        "route_gbs": round(rbytes / (route_avg * 1e-3) / 1e9, 1),
        "route_frac_of_hbm": round(rbytes / (route_avg * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
        "prepare_ms_per_call": round(statistics.mean(prep_ms), 4),
        # the attention kernel is timed inside a ~1 s loop of steps under the power cap:
        # the sustained bf16 peak is its denominator (the burst one is reported beside it)
        "roofline": {"bound": "tensor", "kernel": ATTN_KERNEL, "achieved": round(achieved, 2),
                     "peak": pk["bf16_tflops_sustained"],
                     "peak_kind": f"bf16 dense sustained (cuBLAS 8192^3 for 4 s), {pk_kind}", "unit": "TFLOP/s",
                     "frac": round(achieved / pk["bf16_tflops_sustained"], 4),
                     "frac_of_burst": round(achieved / pk["bf16_tflops"], 4),
                     "traffic": traffic},
        "e2e": {"value": round(flops_sum / (e2e_ms_max * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms_max, 3),
                "h2d_bytes_per_step": 3 * q.numel() * 2, "d2h_bytes_per_step": o.numel() * 2},
        "attn_fp8v": {"kernel": ATTN_KERNEL + "<F8>", "calls": fp8_steps, "attn_ms_per_call": round(fp8_run_ms, 4),
                      "tflops": round(flops / (fp8_run_ms * 1e-3) / 1e12, 2),
                      "prepare_ms_per_call": round(fp8_prep_ms, 4),
                      "note": "Q.K^T bf16, P.V e4m3 (per-channel V scales); same FLOP count as the bf16 path"},
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "clocks": clk,
    }
    if world == 1:
        line["cpu_baseline"] = cpu_baseline(x, w, p, flops)
    return line


ATTN_KERNEL = "k_attn_pp"        # the attention kernel bsa_attn_run launches for block 128
ATTN_SOURCES = ("attn_pp.cu", "tc_common.cuh")
ATTN_PROFILE = "k_attn_pp_wan21_480p.md"


def sources_sha256(names):
    import hashlib
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(ROOT, "block_sparse_attention_top_b200", "csrc", n), "rb").read())
    return h.hexdigest()


def load_traffic():
    """DRAM bytes per launch of the attention kernel, from the committed ncu summary
    (profiles/k_attn_pp_wan21_480p.md), or None if that summary was taken on
    different kernel sources than the ones built here."""
    path = os.path.join(ROOT, "profiles", ATTN_PROFILE)
    try:
        fields = {}
        for line in open(path):
            if ":" in line and line.startswith("- "):
                key, val = line[2:].split(":", 1)
                fields[key.strip()] = val.strip().strip("`")
        if fields.get("sources sha256") != sources_sha256(ATTN_SOURCES):
            return None
        return int(fields["dram bytes per launch"].replace(",", ""))
    except Exception:
        return None


# --------------------------------------------------------------------------- oracle (CPU)
def oracle_step(x, w, p, sample_blocks, rng):
    """One bounded oracle step: full routing, attention on `sample_blocks` query blocks.
    Returns (route_s, attn_s, sample_flops)."""
    import oracle
    t0 = time.perf_counter()
    r = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, p, w.k_floor)
    t1 = time.perf_counter()
    perm = oracle.token_perm(w.T, w.Hs, w.Ws)
    m = oracle.block_counts(w.N, w.block)
    rows = rng.choice(w.rows, size=sample_blocks, replace=False)
    fl = 0.0
    for row in rows:
        bh, i = divmod(int(row), w.nb)
        b, h = divmod(bh, w.H)
        oracle.attend_block(x["q"], x["k"], x["v"], perm, w.block, r.row_ptr, r.col_idx, w.H, b, h, i)
        cols = r.col_idx[r.row_ptr[row]:r.row_ptr[row + 1]]
        fl += 4.0 * w.d * m[i] * float(m[cols].sum())
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1, fl


def cpu_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([d.get("num_threads", 1) for d in info] or [os.cpu_count() or 1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(x, w, p, full_flops, sample_blocks=32, seed=0):
    rng = np.random.default_rng(seed)
    rs, as_, fl = oracle_step(x, w, p, sample_blocks, rng)
    est = rs + as_ * full_flops / fl
    return {"value": round(full_flops / est / 1e12, 6), "unit": "TFLOP/s", "cores": cpu_threads(),
            "kind": "oracle",
            "sample": f"full routing of the workload ({rs:.2f} s) + attention on {sample_blocks} random query "
                      f"blocks ({as_:.2f} s, {fl / 1e9:.1f} GFLOP), attention time extrapolated linearly to the "
                      f"full {full_flops / 1e12:.2f} TFLOP step"}


def reference_step(x, w, p, full_flops, rng):
    """One bounded oracle step: routing of one random head, attention on one
    random query block of it; both extrapolated to the full step."""
    import oracle
    h = int(rng.integers(w.H))
    xh = {n: x[n][:, :, h:h + 1, :] for n in "qkv"}
    t0 = time.perf_counter()
    r = oracle.route(xh["q"], xh["k"], w.T, w.Hs, w.Ws, w.block, p, w.k_floor)
    t1 = time.perf_counter()
    perm = oracle.token_perm(w.T, w.Hs, w.Ws)
    m = oracle.block_counts(w.N, w.block)
    i = int(rng.integers(w.nb))
    oracle.attend_block(xh["q"], xh["k"], xh["v"], perm, w.block, r.row_ptr, r.col_idx, 1, 0, 0, i)
    t2 = time.perf_counter()
    cols = r.col_idx[r.row_ptr[i]:r.row_ptr[i + 1]]
    fl = 4.0 * w.d * m[i] * float(m[cols].sum())
    return (t1 - t0) * w.B * w.H + (t2 - t1) * full_flops / fl


def run_reference(args, world=1):
    """The fp64 CPU oracle on bounded samples of the same workload (the reference arm)."""
    w = syn.workload(CID)
    p = w.ps[P_INDEX]
    x = syn.make_inputs(w, seed=syn.seed_for(CID, P_INDEX))
    import oracle
    r = oracle.route(x["q"], x["k"], w.T, w.Hs, w.Ws, w.block, p, w.k_floor)
    full_flops = attention_flops(r.row_ptr, r.col_idx, w)
    rng = np.random.default_rng(1)
    for _ in range(args.warmup):
        reference_step(x, w, p, full_flops, rng)
    est = [reference_step(x, w, p, full_flops, rng) for _ in range(args.steps)]
    ms = float(np.mean(est)) * 1e3
    value = full_flops / (ms * 1e-3) / 1e12
    sample = (f"each step: oracle routing of 1 random head (of {w.H}) and attention on 1 random query block of "
              f"it, timed and extrapolated linearly to the full step ({w.H} heads, {full_flops / 1e12:.2f} TFLOP)")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(w), "global_batch": w.B, "seq_len": w.N,
                       "parallelism": "CPU oracle (numpy fp64)"},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
