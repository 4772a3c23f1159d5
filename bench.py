"""Benchmark: block-sparse 3D-video attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

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

N > 1 (torchrun): each rank runs the same workload on its own GPU and its own
batch element (weak scaling; heads and batches are independent, so there is
no data-path collective).  Step times are the max over ranks.

--impl reference: the CPU oracle (fp64, all host cores) on a bounded sample of
query rows of the same workload per step, reported in the same unit.
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
LAUNCHES = {"plan_build": 3, "plan_build_stripe": 4, "permute": 1, "unpermute": 1, "fwd": 1,
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
    """The workload rank `rank` processes: same shape and masks, its own batch
    element (independent seeds), so per-GPU work is fixed as ranks are added."""
    from dataclasses import replace
    return replace(w, seeds=tuple(s + 1000 * rank for s in w.seeds))


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


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_baseline(w, seconds_target: float = 12.0):
    """Time the oracle as it stands on sampled rows of up to four heads with
    distinct masks and extrapolate linearly (its cost per row does not depend
    on the row: every row visits all N keys)."""
    import oracle
    heads, seen = [], []
    for h, s in enumerate(w.specs):
        if s not in seen:
            seen.append(s)
            heads.append(h)
    heads = heads[:4]
    grid = (w.T, w.H, w.W)
    threads = oracle.default_threads()
    spent_all, rows_all = 0.0, 0
    budget = seconds_target / len(heads)
    for h in heads:
        q, k, v = (W.head_tensor(w, x, 0, h) for x in "qkv")
        R, spent = 64, 0.0
        while spent < budget and R <= w.N:
            rows = W.sample_rows(w, h, R, seed=1000 + R)
            t0 = time.perf_counter()
            oracle.attention_rows(w.specs[h], grid, w.unit, w.D, w.scale, q, k, v, rows, threads)
            spent += time.perf_counter() - t0
            rows_all += len(rows)
            R *= 2
        spent_all += spent
    per_row = spent_all / rows_all
    est = per_row * w.N * w.heads * w.B
    return est, threads, spent_all, rows_all, heads


def run_reference(args, w, world, rank):
    """The CPU oracle, timed on bounded samples of the same workload."""
    if rank != 0:
        return
    import oracle
    grid = (w.T, w.H, w.W)
    threads = oracle.default_threads()
    # the tile-major layout holds the padded grid rounded up to whole tiles
    L = max(128, w.q_tile, w.kv_tile)
    n_slots = -(-oracle.padded_tokens(grid, w.unit) // L) * L
    # executed tiles of the workload, from the oracle's own tile classes on sampled q tiles
    counts = np.zeros((w.heads, 3))
    nq = n_slots // w.q_tile
    sample_q = np.unique(np.linspace(0, nq - 1, 8).astype(np.int64))
    for h in range(w.heads):
        same = [g for g in range(h) if w.specs[g] == w.specs[h]]
        if same:
            counts[h] = counts[same[0]]
            continue
        cls = oracle.tile_map(w.specs[h], grid, w.unit, n_slots, w.q_tile, w.kv_tile,
                              sample_q, threads)
        for c in range(3):
            counts[h, c] = (cls == c).sum() * nq / len(sample_q)
    flops = exec_flops(w, counts) * w.B
    h0 = 0
    q, k, v = (W.head_tensor(w, x, 0, h0) for x in "qkv")
    R = 256
    times = []
    for step in range(args.warmup + args.steps):
        rows = W.sample_rows(w, h0, R, seed=step)
        t0 = time.perf_counter()
        oracle.attention_rows(w.specs[h0], grid, w.unit, w.D, w.scale, q, k, v, rows, threads)
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            times.append(dt)
    per_row = statistics.mean(times) / R
    full_time = per_row * w.N * w.heads * w.B
    value = flops / full_time / 1e12
    sample = (f"{R} sampled query rows of head {h0} per step (exact over all {w.N} keys), "
              f"extrapolated linearly to {w.heads} heads x {w.N} rows; executed tiles from the "
              f"oracle's classes on {len(sample_q)} sampled q-tile rows per distinct head")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": full_time * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(w.describe(), parallelism="cpu oracle"),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_gpu(args, w, world, rank, local):
    import torch
    import block_sparse_attention_mask_b200 as vsa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)
    grid = (w.T, w.H, w.W)
    B = w.B

    # inputs: rank r draws its own batch element (weak scaling)
    wr = rank_workload(w, rank)
    host = [W.full_tensor(wr, x) for x in "qkv"]
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
    value = aggregate_tflops(flops_step, world, ms_step)

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
    achieved = flops_b * B / (ms_fwd_mean * 1e-3) / 1e12
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

    result = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            est, cores, spent, nrows, heads = cpu_baseline(w)
            cpu = {"value": flops_step / est / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                   "sample": (f"{nrows} stratified query rows of heads {heads} (one per distinct mask, "
                              f"exact over all {w.N} keys, {spent:.1f} s), extrapolated linearly to "
                              f"{w.heads} heads x {w.N} rows = {est:.0f} s for one step")}
        kept = plan.kept_pairs(stream)
        useful = 4.0 * w.D * float(kept.sum()) * B
        result = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": dict(w.describe(), parallelism=f"dp{world} (independent batch per rank)",
                           l2="inputs larger than L2 (natural q,k,v = "
                              f"{3 * q.numel() * 2 / 1e6:.0f} MB), no flush"),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "kernel": "attn_fwd_kernel<128,128>",
                         "peak_source": f"{how} bf16_tflops (burst)"},
            "fwd_ms": ms_fwd_mean,
            "exec_tflop_per_step": flops_step / 1e12,
            "useful_tflop_per_step": useful / 1e12,
            "useful_tflops_fwd": useful / (ms_fwd_mean * 1e-3) / 1e12,
            "kept_pair_fraction": float(kept.sum()) / (w.heads * w.N ** 2),
            "tiles": {"full": int(counts[:, 2].sum()), "boundary": int(counts[:, 1].sum()),
                      "empty": int(counts[:, 0].sum()),
                      "boundary_share_of_executed": float(counts[:, 1].sum() / max(1, counts[:, 1:].sum()))},
            "exec_steps": int(steps_exec.sum()),
            "cpu_baseline": cpu,
            "route": None if not routed else {
                "ms": ms_route, "rows": int(len(rows_np)),
                "flags": [int(x) for x in r_flags.cpu().numpy()],
                # four R x N x D products (QK^T and three PV) over the sampled rows
                "tflops": 8.0 * B * w.heads * len(rows_np) * w.N * w.D / (ms_route * 1e-3) / 1e12,
                "frac": 8.0 * B * w.heads * len(rows_np) * w.N * w.D / (ms_route * 1e-3) / 1e12 / peak},
            "e2e": {"value": aggregate_tflops(flops_step, world, ms_e2e), "unit": "TFLOP/s",
                    "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "clocks": clk,
            "gpu_launches": per_step_launches * args.steps,
        }
    plan.close()
    return result


_REV = None


def kernel_rev() -> str:
    """Hash of the attention kernel's sources, to tie stored ncu counters to them."""
    global _REV
    if _REV is None:
        import hashlib
        h = hashlib.sha256()
        for f in ("vsa_attn.cu", "vsa_sm100.cuh"):
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
