"""Benchmark: block-sparse 3D-video attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--partition heads|batch] [--impl reference] [--no-extra]

One step is one pass of the whole path over one batch of synthetic input,
through the C ABI: rebuild the plan's tile map and kv-tile lists, permute
q, k, v into tile-major order, run the block-sparse attention forward, and
restore the output order.  Inputs (natural-order q, k, v) are resident in HBM
when the timed region starts; they are larger than L2, so no flush is needed
between steps.  Each step is timed with CUDA events on the launching stream;
the attention kernel is also timed alone inside every step.

Throughput is effective TFLOP/s over executed tiles: 4 * d * Bq * Bk FLOPs per
full or boundary (q tile, kv tile) pair of the map, per head and batch.

e2e: the same step from pinned host buffers through the host-buffer entry
point (vsa_pipeline_run: per chunk of heads, the host-to-device copies of
q, k, v, the step's kernels and the device-to-host copies of o and lse on
three streams, overlapped), timed with CUDA events on the caller's stream.
Routed workloads time it with the copies and the step in series.

N > 1 (torchrun), --partition heads (default): rank r takes the contiguous
heads [floor(r H / N), floor((r+1) H / N)) of the same batch element, builds
its own plan for them and runs the unchanged path (strong scaling: the whole
job's work is fixed; heads are independent, so there is no data-path
collective).  --partition batch: every rank runs all heads of its own batch
element (weak scaling).  Step times are the max over ranks.

At N = 1 the line also carries ``workloads``: the attention kernel alone on
the other workloads (STA HunyuanVideo, the stripe heads, the dense and
spatial scaling grids T = 5..33 with their scaling efficiency, and the
q-tile x kv-tile sweep at T = 21), a few timed launches each.

--impl reference: the CPU oracle (fp64, all host cores), each step a bounded
sample of query rows of the same workload, reported in the same unit.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "sparse attn fwd ms & effective TFLOPS (kept tiles) vs B200 bf16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# kernels launched per ABI call (claimed launch count inside the timed region)
LAUNCHES = {"plan_build": 6, "plan_build_stripe": 7, "permute": 1, "unpermute": 1, "fwd": 1,
            "route": 3, "apply": 1}
ROUTE_FRAC = 0.01      # sampled share of the tokens for SVG routing
E2E_CHUNK_HEADS = 1    # heads per chunk of the copy-overlapped host-buffer path

WORKLOADS = {
    "svg_wan720p": W.svg_wan720p,
    "svg_wan720p_temporal_f0": lambda: W.svg_wan720p(temporal_layout=1),
    "svg_wan720p_rounded": lambda: W.svg_wan720p(tile_round=1),
    "svg_wan720p_temporal_f0_rounded": lambda: W.svg_wan720p(temporal_layout=1, tile_round=1),
    "svg_wan720p_routing": W.svg_wan720p_routing,
    "svg_wan720p_routing_f0": lambda: W.svg_wan720p_routing(temporal_layout=1),
    "tiny": W.tiny,
    "sta_hunyuan720p": W.sta_hunyuan720p,
    "stripe_wan720p": W.stripe_wan720p,
}
for _T in W.SCALING_T:
    for _m in ("full", "spatial"):
        WORKLOADS[f"scaling_{_m}_T{_T}"] = (lambda T=_T, m=_m: W.scaling(T, m))
for _q in W.SWEEP_Q:
    for _k in W.SWEEP_KV:
        WORKLOADS[f"sweep_q{_q}_k{_k}"] = (lambda q=_q, k=_k: W.scaling(21, "spatial", q, k))


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------


def exec_flops(w, counts) -> float:
    """Executed-tile FLOPs per batch element: 4*d*Bq*Bk per full or boundary tile."""
    executed = int(counts[:, 1].sum() + counts[:, 2].sum())
    return 4.0 * w.D * w.q_tile * w.kv_tile * executed


def rank_workload(w, rank: int):
    """--partition batch: the workload rank `rank` processes is the same shape
    and masks with its own batch element (independent seeds), so per-GPU work
    is fixed as ranks are added."""
    from dataclasses import replace
    return replace(w, seeds=tuple(s + 1000 * rank for s in w.seeds))


def head_range(heads: int, rank: int, world: int):
    """--partition heads: rank r's contiguous heads [floor(r H / G), floor((r+1) H / G))."""
    if world > heads:
        raise ValueError(f"{world} ranks for {heads} heads: some rank would hold no head")
    return rank * heads // world, (rank + 1) * heads // world


def rank_shard(w, rank: int, world: int, partition: str):
    """The workload one rank runs: its head range (heads) or its batch element (batch)."""
    if partition == "heads":
        lo, hi = head_range(w.heads, rank, world)
        return w.head_shard(lo, hi) if (lo, hi) != (0, w.heads) else w
    return rank_workload(w, rank)


def aggregate_tflops(flops_per_rank_step: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's executed FLOPs over the slowest rank's step time."""
    return flops_per_rank_step * world / (ms_max * 1e-3) / 1e12


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        backend = "nccl" if os.environ.get("VSA_BENCH_BACKEND", "nccl") == "nccl" else "gloo"
        dist.init_process_group(backend, timeout=timedelta(seconds=300))
    return world, rank, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def oracle_groups(w, max_groups: int = 8):
    """Heads that stand for the workload in an oracle sample: one per distinct
    mask, with the number of heads sharing it as its weight; with more than
    ``max_groups`` distinct masks (the stripe workload's 40), ``max_groups``
    heads spread evenly over the workload, each weighing heads / max_groups."""
    groups = []
    for h, s in enumerate(w.specs):
        for g in groups:
            if w.specs[g[0]] == s:
                g[1] += 1
                break
        else:
            groups.append([h, 1])
    if len(groups) > max_groups:
        pick = np.linspace(0, w.heads - 1, max_groups).round().astype(int)
        groups = [[int(h), w.heads / max_groups] for h in pick]
    return [(h, float(c)) for h, c in groups]


_ORACLE_INPUTS = {}


def oracle_sample_step(w, R: int, seed: int, threads: int):
    """One bounded sample of the oracle on workload ``w``, timed on host cores.

    For each head standing for the workload (``oracle_groups``): one call with
    no query rows, which costs what every call costs once (widening the head's
    k and v to fp64, starting the threads), and one call with R uniform random
    query rows (each exact over all N keys; a row's cost depends on how many
    keys its mask keeps, so rows are drawn uniformly, not stratified).
    Returns (estimated seconds of the oracle over the whole workload: every
    head pays the fixed cost once and N rows at its mask's per-row cost;
    wall seconds of this sample; rows timed)."""
    import oracle
    grid = (w.T, w.H, w.W)
    est, wall, nrows = 0.0, 0.0, 0
    for h, weight in oracle_groups(w):
        key = (w.name, w.head_offset, h)
        if key not in _ORACLE_INPUTS:
            if len(_ORACLE_INPUTS) >= 8:
                _ORACLE_INPUTS.clear()
            _ORACLE_INPUTS[key] = tuple(W.head_tensor(w, x, 0, h) for x in "qkv")
        q, k, v = _ORACLE_INPUTS[key]
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, h])))
        rows = np.sort(g.choice(w.N, size=min(R, w.N), replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        oracle.attention_rows(w.specs[h], grid, w.unit, w.D, w.scale, q, k, v, rows[:0], threads)
        t1 = time.perf_counter()
        oracle.attention_rows(w.specs[h], grid, w.unit, w.D, w.scale, q, k, v, rows, threads)
        t2 = time.perf_counter()
        fixed = t1 - t0
        per_row = max(0.0, (t2 - t1) - fixed) / len(rows)
        est += weight * w.B * (fixed + w.N * per_row)
        wall += t2 - t0
        nrows += len(rows)
    return est, wall, nrows


def oracle_rate(w, flops_step: float, steps: int, R: int, threads: int, seed0: int = 0):
    """The oracle's throughput in the bench's unit from ``steps`` samples:
    executed-tile FLOPs of one whole step over the mean estimated time of the
    oracle on it.  Both the GPU arm's cpu_baseline and --impl reference call
    this, so they measure the same thing the same way."""
    ests, walls, rows = [], [], 0
    for i in range(steps):
        e, wl, n = oracle_sample_step(w, R, seed0 + i, threads)
        ests.append(e)
        walls.append(wl)
        rows += n
    est = statistics.mean(ests)
    groups = oracle_groups(w)
    sample = (f"per step, for heads {[h for h, _ in groups]} (weights {[c for _, c in groups]}; one head per "
              f"distinct mask, or spread evenly): a call with no rows (the per-call fixed cost: widening k, v "
              f"to fp64, thread start) and a call with {R} uniform random query rows exact over all {w.N} keys; "
              f"whole-step time estimated as every head's fixed cost + {w.N} rows at its mask's per-row cost "
              f"= {est:.1f} s (mean of {steps} samples, {rows} rows timed in all)")
    return flops_step / est / 1e12, est, statistics.mean(walls), sample


def oracle_exec_flops(w, threads: int, max_full: int = 4, n_qtiles: int = 64):
    """Executed-tile FLOPs of one step of ``w`` from the oracle's own tile
    classes: every q tile of every distinct mask when the workload has at most
    ``max_full`` distinct masks (exact), else ``n_qtiles`` evenly spaced q-tile
    rows per distinct mask (extrapolated).  Returns (FLOPs, how)."""
    import oracle
    grid = (w.T, w.H, w.W)
    L = max(128, w.q_tile, w.kv_tile)        # the tile-major slots: padded grid in whole tiles
    n_slots = -(-oracle.padded_tokens(grid, w.unit) // L) * L
    nq = n_slots // w.q_tile
    distinct = {tuple(sorted(s.items())) for s in w.specs}
    exact = len(distinct) <= max_full
    sample_q = np.arange(nq) if exact else np.unique(np.linspace(0, nq - 1, n_qtiles).round().astype(np.int64))
    counts, done = np.zeros((w.heads, 3)), {}
    for h in range(w.heads):
        key = tuple(sorted(w.specs[h].items()))
        if key not in done:
            fn = oracle.rounded_tile_map if w.specs[h].get("tile_round", 0) else oracle.tile_map
            cls = fn(w.specs[h], grid, w.unit, n_slots, w.q_tile, w.kv_tile, sample_q, threads)
            done[key] = [(cls == c).sum() * nq / len(sample_q) for c in range(3)]
        counts[h] = done[key]
    how = ("from the oracle's classes of every q tile of each distinct mask" if exact else
           f"from the oracle's classes on {len(sample_q)} evenly spaced q-tile rows per distinct mask")
    return exec_flops(w, counts) * w.B, how


def bench_config(w, world: int, partition: str):
    par = (f"heads{world} (contiguous head ranges per rank, no collective)" if partition == "heads"
           else f"dp{world} (independent batch per rank)")
    mb = 3 * w.B * w.heads * w.N * w.D * 2 / 1e6
    l2 = (f"inputs larger than L2 (natural q,k,v = {mb:.0f} MB), no flush" if mb > 126
          else f"inputs fit in L2 (natural q,k,v = {mb:.1f} MB): warm-cache timing")
    return dict(w.describe(), parallelism=par, l2=l2)


def run_reference(args, w, world, rank):
    """The CPU oracle, timed on bounded samples of the same workload."""
    if rank != 0:
        return
    import oracle
    threads = oracle.default_threads()
    flops, how = oracle_exec_flops(w, threads)
    R = 512          # the same sample size as the GPU arm's cpu_baseline
    for i in range(args.warmup):              # untimed: page in inputs, warm the caches
        oracle_sample_step(w, 16, 10_000 + i, threads)
    value, est, wall, sample = oracle_rate(w, flops, args.steps, R, threads)
    sample += f"; executed tiles {how}; ms_per_step is the wall time of one sample step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": wall * 1e3, "higher_is_better": True,
        "scaling": "strong" if args.partition == "heads" else "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w, args.gpus, args.partition),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample, "est_step_s": est},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


EXTRA_WARMUP, EXTRA_TIMED = 3, 5


def extra_entries():
    """(key, workload) pairs timed for the line's ``workloads`` key."""
    out = [("sta_hunyuan720p", W.sta_hunyuan720p()), ("stripe_wan720p", W.stripe_wan720p())]
    for T in W.SCALING_T:
        for m in ("full", "spatial"):
            out.append((f"scaling_{m}_T{T}", W.scaling(T, m)))
    for q in W.SWEEP_Q:
        for k in W.SWEEP_KV:
            if (q, k) != (128, 128):
                out.append((f"sweep_q{q}_k{k}", W.scaling(21, "spatial", q, k)))
    return out


def time_attention(w, dev, stream, peak: float) -> dict:
    """The attention kernel alone on workload ``w``: plan, permuted N(0,1)
    bf16 inputs drawn on the device from a fixed seed, EXTRA_WARMUP untimed and
    EXTRA_TIMED timed launches (CUDA events on the launching stream)."""
    import torch
    import block_sparse_attention_mask_b200 as vsa
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234)
    with torch.cuda.stream(stream):
        plan = vsa.Plan(list(w.specs), (w.T, w.H, w.W), w.unit, w.q_tile, w.kv_tile, stream=stream)
        try:
            S = plan.n_slots
            nat = [torch.randn((w.B, w.heads, w.N, w.D), generator=gen, device=dev).to(torch.bfloat16)
                   for _ in range(3)]
            qp = torch.empty((w.B, w.heads, S, w.D), dtype=torch.bfloat16, device=dev)
            kp, vp, op = torch.empty_like(qp), torch.empty_like(qp), torch.empty_like(qp)
            lse = torch.empty((w.B, w.heads, S), dtype=torch.float32, device=dev)
            h, sh = plan.handle, stream.cuda_stream
            vsa.vsa_permute_qkv(h, nat[0], nat[1], nat[2], qp, kp, vp, w.B, w.D, sh)
            del nat
            for _ in range(EXTRA_WARMUP):
                vsa.vsa_sparse_attn_fwd(qp, kp, vp, op, lse, h, w.B, w.D, w.scale, sh)
            ev = []
            for _ in range(EXTRA_TIMED):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                vsa.vsa_sparse_attn_fwd(qp, kp, vp, op, lse, h, w.B, w.D, w.scale, sh)
                e1.record(stream)
                ev.append((e0, e1))
            stream.synchronize()
            plan.check(stream)
            counts = plan.tile_counts(stream)
            steps = int(plan.exec_steps(stream).sum())
        finally:
            plan.close()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    flops = exec_flops(w, counts) * w.B
    tf = flops / (ms * 1e-3) / 1e12
    full, bnd, empty = (int(counts[:, c].sum()) for c in (2, 1, 0))
    return {"fwd_ms": round(ms, 4), "tflops": round(tf, 1), "frac": round(tf / peak, 4),
            "exec_tflop": round(flops / 1e12, 4), "tiles": {"full": full, "boundary": bnd, "empty": empty},
            "boundary_share": round(bnd / max(1, full + bnd), 4),
            "executed_fraction": round((full + bnd) / max(1, full + bnd + empty), 4), "exec_steps": steps,
            "q_tile": w.q_tile, "kv_tile": w.kv_tile}


def extra_workloads(dev, stream, peak: float, smi_id: str) -> dict:
    """Attention-only numbers for the other workloads, and the scaling
    efficiency (t_spatial / t_dense) / (executed spatial / executed dense)
    per T: 1 means the wall time follows the executed-tile fraction."""
    smi = ClockSampler(smi_id)
    smi.start()
    out = {}
    for key, w in extra_entries():
        out[key] = time_attention(w, dev, stream, peak)
    clk = smi.stop()
    eff = {}
    for T in W.SCALING_T:
        d, sp = out[f"scaling_full_T{T}"], out[f"scaling_spatial_T{T}"]
        eff[f"T{T}"] = round((sp["fwd_ms"] / d["fwd_ms"]) / (sp["exec_tflop"] / d["exec_tflop"]), 4)
    out["scaling_efficiency"] = eff
    out["timing"] = (f"attention kernel alone, {EXTRA_TIMED} launches after {EXTRA_WARMUP} warm-ups, CUDA events; "
                     f"frac of the measured burst bf16 peak {peak}")
    out["clocks"] = clk
    return out


def run_gpu(args, w, world, rank, local):
    import torch
    import block_sparse_attention_mask_b200 as vsa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)
    grid = (w.T, w.H, w.W)
    B = w.B

    # this rank's share: its head range (default) or its own batch element
    wg = w
    w = rank_shard(w, rank, world, args.partition)
    host = [W.full_tensor(w, x) for x in "qkv"]
    pinned = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in host]
    del host
    with torch.cuda.stream(stream):
        q, k, v = (p.to(dev, non_blocking=True) for p in pinned)
        plan = vsa.Plan(list(w.specs), grid, w.unit, w.q_tile, w.kv_tile, stream=stream)
        S = plan.n_slots
        qp = torch.empty((B, w.heads, S, w.D), dtype=torch.bfloat16, device=dev)
        kp, vp, op = torch.empty_like(qp), torch.empty_like(qp), torch.empty_like(qp)
        lse = torch.empty((B, w.heads, S), dtype=torch.float32, device=dev)
        o = torch.empty_like(q)
    stream.synchronize()
    h = plan.handle
    sh = stream.cuda_stream
    has_stripe = any(s["kind"] == W.MASK_KINDS["stripe"] for s in w.specs)
    per_step_launches = (LAUNCHES["plan_build_stripe"] if has_stripe else LAUNCHES["plan_build"]) \
        + LAUNCHES["permute"] + LAUNCHES["fwd"] + LAUNCHES["unpermute"]

    # SVG routing before the plan build: sampled-query profiling, then the
    # per-head switch (which rebuilds the plan on the device)
    routed = bool(w.route_specs)
    route_events = []
    if routed:
        plan.set_route_candidates([a for a, _ in w.route_specs], [b for _, b in w.route_specs], stream)
        rows_np = W.route_rows(w.N, ROUTE_FRAC).astype(np.int32)
        with torch.cuda.stream(stream):
            rows_d = torch.from_numpy(rows_np).to(dev)
            ws = torch.empty(vsa.vsa_svg_route_workspace_size(h, B, w.D, len(rows_np)),
                             dtype=torch.uint8, device=dev)
            r_err = torch.empty((w.heads, 2), dtype=torch.float32, device=dev)
            r_flags = torch.empty((w.heads,), dtype=torch.int32, device=dev)
        stream.synchronize()
        per_step_launches += LAUNCHES["route"] + LAUNCHES["apply"]

    def plan_step(qn, kn, vn, record: bool):
        if not routed:
            vsa.vsa_plan_build(h, sh)
            return
        if record:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        vsa.vsa_svg_route(h, qn, kn, vn, B, w.D, rows_d, len(rows_np), w.scale, r_err, r_flags, ws,
                          ws.numel(), sh)
        if record:
            e1.record(stream)
            route_events.append((e0, e1))
        vsa.vsa_plan_apply_route(h, r_flags, sh)

    fwd_events = []

    def step(record_fwd: bool):
        plan_step(q, k, v, record_fwd)
        vsa.vsa_permute_qkv(h, q, k, v, qp, kp, vp, B, w.D, sh)
        if record_fwd:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        vsa.vsa_sparse_attn_fwd(qp, kp, vp, op, lse, h, B, w.D, w.scale, sh)
        if record_fwd:
            e1.record(stream)
            fwd_events.append((e0, e1))
        vsa.vsa_unpermute(h, op, o, B, w.D, sh)

    for _ in range(args.warmup):
        step(False)
    stream.synchronize()
    plan.check(stream)
    counts = plan.tile_counts(stream)
    steps_exec = plan.exec_steps(stream)
    flops_b = exec_flops(w, counts)          # per batch element
    flops_step = flops_b * B

    # ---- device-resident timed region ----
    props = torch.cuda.get_device_properties(dev)
    try:
        smi_id = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
    except AttributeError:
        smi_id = str(local)
    clocks = ClockSampler(smi_id)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    step_events = []
    for _ in range(args.steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step(True)
        e1.record(stream)
        step_events.append((e0, e1))
    stream.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    plan.check(stream)
    ms_steps = [a.elapsed_time(b) for a, b in step_events]
    ms_fwd = [a.elapsed_time(b) for a, b in fwd_events]
    ms_route = max_over_ranks(statistics.mean([a.elapsed_time(b) for a, b in route_events]), world, dev) \
        if routed else None
    ms_step = max_over_ranks(statistics.mean(ms_steps), world, dev)
    ms_fwd_mean = max_over_ranks(statistics.mean(ms_fwd), world, dev)
    # whole-job executed FLOPs: every rank's own (head ranges differ in work)
    flops_job = sum_over_ranks(flops_step, world, dev)
    value = flops_job / (ms_step * 1e-3) / 1e12

    # ---- end to end through the public API with host buffers ----
    o_host = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()
    lse_host = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    pipe = None
    if not routed:
        # the host-buffer entry point: copies overlapped with compute, one
        # chunk of heads at a time (vsa_pipeline_run)
        pipe = vsa.Pipeline(list(w.specs), grid, w.unit, w.q_tile, w.kv_tile, B=B, D=w.D,
                            chunk_heads=E2E_CHUNK_HEADS)

    def e2e_step():
        if pipe is not None:
            pipe.run(pinned[0], pinned[1], pinned[2], o_host, lse_host, w.scale, sh)
            return
        qd.copy_(pinned[0], non_blocking=True)
        kd.copy_(pinned[1], non_blocking=True)
        vd.copy_(pinned[2], non_blocking=True)
        plan_step(qd, kd, vd, False)
        vsa.vsa_permute_qkv(h, qd, kd, vd, qp, kp, vp, B, w.D, sh)
        vsa.vsa_sparse_attn_fwd(qp, kp, vp, op, lse, h, B, w.D, w.scale, sh)
        vsa.vsa_unpermute(h, op, o, B, w.D, sh)
        o_host.copy_(o, non_blocking=True)
        lse_host.copy_(lse, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 10))
    with torch.cuda.stream(stream):
        for _ in range(2):
            e2e_step()
        stream.synchronize()
        barrier(world)
        ev = []
        for _ in range(e2e_steps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            e2e_step()
            e1.record(stream)
            ev.append((e0, e1))
        stream.synchronize()
    barrier(world)
    ms_e2e = max_over_ranks(statistics.mean([a.elapsed_time(b) for a, b in ev]), world, dev)
    plan.check(stream)
    if pipe is not None:
        pipe.check(stream)
        pipe.close()
    h2d = 3 * q.numel() * 2
    d2h = o.numel() * 2 + lse.numel() * 4

    pk, how = peaks()
    peak = float(pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    # the dominant kernel on this rank: its executed FLOPs over its own mean launch time
    achieved = flops_b * B / (statistics.mean(ms_fwd) * 1e-3) / 1e12
    traffic = None
    prof = os.path.join(ROOT, "profiles", "attn_fwd_svg_wan720p_traffic.txt")
    if os.path.exists(prof):
        try:
            with open(prof) as f:
                tj = json.load(f)
            if tj.get("workload") == w.name and tj.get("kernel_rev") == kernel_rev():
                traffic = tj.get("bytes_per_launch")
        except Exception:
            traffic = None

    kept = plan.kept_pairs(stream)
    useful = sum_over_ranks(4.0 * w.D * float(kept.sum()) * B, world, dev)
    tiles = [sum_over_ranks(float(counts[:, c].sum()), world, dev) for c in range(3)]
    extra = None
    if world == 1 and not args.no_extra:
        extra = extra_workloads(dev, stream, float(peaks()[0].get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])),
                                smi_id)
    result = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            threads = oracle.default_threads()
            cval, est, _, sample = oracle_rate(w, flops_step, 4, 512, threads, seed0=100)
            cpu = {"value": cval, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                   "sample": sample, "est_step_s": est}
        heads_job = wg.heads if args.partition == "heads" else wg.heads * world
        result = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "strong" if args.partition == "heads" else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": bench_config(wg, world, args.partition),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "kernel": "attn_fwd_kernel<128,128>",
                         "peak_source": f"{how} bf16_tflops (burst)"},
            "fwd_ms": ms_fwd_mean,
            "exec_tflop_per_step": flops_job / 1e12,
            "useful_tflop_per_step": useful / 1e12,
            "useful_tflops_fwd": useful / (ms_fwd_mean * 1e-3) / 1e12,
            "kept_pair_fraction": useful / (4.0 * w.D * B) / (heads_job * w.N ** 2),
            "tiles": {"full": int(tiles[2]), "boundary": int(tiles[1]), "empty": int(tiles[0]),
                      "boundary_share_of_executed": tiles[1] / max(1.0, tiles[1] + tiles[2])},
            "exec_steps": int(steps_exec.sum()),
            "cpu_baseline": cpu,
            "route": None if not routed else {
                "ms": ms_route, "rows": int(len(rows_np)),
                "flags": [int(x) for x in r_flags.cpu().numpy()],
                # four R x N x D products (QK^T and three PV) over the sampled rows
                "tflops": 8.0 * B * w.heads * len(rows_np) * w.N * w.D / (ms_route * 1e-3) / 1e12,
                "frac": 8.0 * B * w.heads * len(rows_np) * w.N * w.D / (ms_route * 1e-3) / 1e12 / peak},
            "e2e": {"value": flops_job / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d * world,
                    "d2h_bytes_per_step": d2h * world},
            "clocks": clk,
            "gpu_launches": per_step_launches * args.steps * world,
        }
        if extra is not None:
            result["workloads"] = extra
    plan.close()
    return result


_REV = None


def kernel_rev() -> str:
    """Hash of the attention kernel's sources and of the plan code that orders
    its kv lists (the order moves DRAM traffic), to tie stored ncu counters to them."""
    global _REV
    if _REV is None:
        import hashlib
        h = hashlib.sha256()
        for f in ("vsa_attn.cu", "vsa_sm100.cuh", "vsa_plan.cu"):
            with open(os.path.join(ROOT, "block_sparse_attention_mask_b200", "csrc", f), "rb") as fh:
                h.update(fh.read())
        _REV = h.hexdigest()[:16]
    return _REV


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="svg_wan720p", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="vsa", choices=["vsa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads' attention timings")
    ap.add_argument("--partition", default="heads", choices=["heads", "batch"],
                    help="N > 1: split the heads across ranks (default) or give each rank a batch element")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    w = WORKLOADS[args.workload]()
    if args.impl == "reference":
        # the CPU oracle runs on rank 0 only; no process group is needed
        run_reference(args, w, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_init()
    try:
        res = run_gpu(args, w, world, rank, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
