"""Benchmark of the performer unit step on B200.

One step = one full 640x368 unit of the performer: append the thinker's
conditioning slice, then for each of the 4 flow-matching Euler steps run the 40
layers' block-causal attention over the 64-unit history (each call first writes
the current latent tokens' K/V into the cache), then the Euler update of the
unit latent; finally commit the unit's latent K/V.  Inputs are seeded synthetic
N(0,1) bf16 tensors resident in HBM before the timed region; the 50.9 GB cache
and the per-call inputs are far larger than L2, so no flush is needed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Under torchrun (N > 1) every rank runs an
independent replica (the unit step has no cross-GPU exchange on one GPU's
work), the step time is the max over ranks and ``value`` aggregates all ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "block-causal unit-attention TFLOP/s & ms per 640×368 unit on 1 B200 (% of bf16 peak)"
UNIT = "TFLOP/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "unit_attention_traffic.txt")
# sources of the benchmark's attention kernel (the single-SM kernel)
KERNEL_SOURCES = ["kv_cache_serving_ws_b200/csrc/attention.cu", "kv_cache_serving_ws_b200/csrc/attn_common.cuh",
                  "kv_cache_serving_ws_b200/csrc/sm100.cuh", "kv_cache_serving_ws_b200/csrc/kernels.cuh",
                  "kv_cache_serving_ws_b200/csrc/tmem_ldst.cuh"]


# ------------------------------------------------------------ multi-rank --

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity when there is one rank)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device_index=None):
    if world <= 1:
        return
    import torch.distributed as dist
    if device_index is not None and dist.get_backend() == "nccl":
        dist.barrier(device_ids=[device_index])
    else:
        dist.barrier()


def aggregate(per_rank_flops: float, world: int, step_s_max: float, steps: int) -> float:
    """Whole-job TFLOP/s: every rank's work over the slowest rank's time."""
    return per_rank_flops * world * steps / step_s_max / 1e12 / steps if step_s_max > 0 else 0.0


# ---------------------------------------------------------------- helpers --

def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {"hbm": p["hbm_gbs"], "bf16": p["bf16_tflops"], "bf16_sustained": p["bf16_tflops_sustained"],
                "source": "measured"}
    except Exception:
        return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    try:
        kv = {}
        with open(TRAFFIC_FILE) as f:
            for line in f:
                if "=" in line and not line.startswith("#"):
                    k, v = line.strip().split("=", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("source_sha") != kernel_source_sha():
            return None
        return float(kv["traffic_bytes_per_full_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = max(smax, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax or None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- our arm --

def run_ours(args, rank, local_rank, world):
    import torch

    from kv_cache_serving_ws_b200 import native as ws
    from kv_cache_serving_ws_b200 import synth
    from kv_cache_serving_ws_b200.workloads import FULL, GpuSession, key

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = FULL
    L, S = w.n_layers, w.steps
    g = GpuSession(w, device=dev)
    stream = torch.cuda.current_stream()

    # ---- resident inputs: one unit's worth, reused by every timed unit
    qs = (w.n_query, w.n_heads, w.head_dim)
    n_lat = w.n_query * w.n_heads * w.head_dim
    bf = torch.bfloat16
    q_all = torch.empty((S, L) + qs, dtype=bf, device=dev)
    kn_all, vn_all = torch.empty_like(q_all), torch.empty_like(q_all)
    for s in range(S):
        for l in range(L):
            g.fill(q_all[s, l], key(w, synth.KIND_Q, w.unit, l, s))
            g.fill(kn_all[s, l], key(w, synth.KIND_K_NEW, w.unit, l, s))
            g.fill(vn_all[s, l], key(w, synth.KIND_V_NEW, w.unit, l, s))
    vel = torch.empty((S, n_lat), dtype=bf, device=dev)
    for s in range(S):
        g.fill(vel[s], key(w, synth.KIND_VEL, w.unit, 0, s))
    x0 = torch.empty(n_lat, dtype=bf, device=dev)
    g.fill(x0, key(w, synth.KIND_X, w.unit))
    x = x0.clone()
    out = torch.empty(qs, dtype=bf, device=dev)
    cond_k = torch.empty_like(g.cond_k)
    cond_v = torch.empty_like(g.cond_v)
    g.fill(cond_k, key(w, synth.KIND_COND_K, w.unit))
    g.fill(cond_v, key(w, synth.KIND_COND_V, w.unit))
    commit_k, commit_v = g.commit_buffers()

    # ---- steady-state history: 64 committed units, each with its own data
    for u in range(0, w.unit):
        g.append_cond(u)
        g.commit(u)
    g.fill(commit_k, key(w, synth.KIND_COMMIT_K, w.unit))
    g.fill(commit_v, key(w, synth.KIND_COMMIT_V, w.unit))
    torch.cuda.synchronize()

    h = g.h
    next_unit = [w.unit]

    def unit_step(x_dev, inputs=None, after_call=None, vel_of=None, cond=None):
        """One unit: conditioning append, S x L attention calls with Euler updates, commit."""
        u = next_unit[0]
        ck, cv = (cond_k, cond_v) if cond is None else cond
        ws.ws_cache_append(h, u, ws.WS_SEG_COND, ck, cv)
        for s in range(S):
            for l in range(L):
                q, kn, vn = (q_all[s, l], kn_all[s, l], vn_all[s, l]) if inputs is None else inputs(s, l)
                ws.ws_unit_attention(h, l, u, q, kn, vn, out)
                if after_call is not None:
                    after_call(s, l)
            ws.ws_flow_step(x_dev, vel[s] if vel_of is None else vel_of(s), w.dt)
        ws.ws_cache_append(h, u, ws.WS_SEG_LATENT, commit_k, commit_v)
        next_unit[0] = u + 1

    for _ in range(args.warmup):
        unit_step(x)
    assert ws.ws_sync(h, check=False) == ws.WS_OK
    ws.ws_profile_enable(h, True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, local_rank)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        torch.cuda.nvtx.range_push("timed")
        e0.record(stream)
        for _ in range(args.steps):
            unit_step(x)
        e1.record(stream)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
    barrier(world, local_rank)
    step_ms = e0.elapsed_time(e1) / args.steps
    prof = ws.ws_profile_read(h)
    ws.ws_profile_enable(h, False)
    st = ws.ws_sync(h, check=False)
    if st != ws.WS_OK:
        raise RuntimeError(f"device status after the timed region: {ws.status_string(st)}")
    step_ms_max = max_over_ranks(step_ms, world, dev)
    flops_unit = w.flops_per_call() * L * S
    value = aggregate(flops_unit, world, step_ms_max / 1e3, 1)

    # ---- dominant kernel: attention, event-timed per launch inside the timed region
    pk = peaks()
    n_attn = prof["attention_launches"]
    attn_ms_avg = prof["attention_ms"] / max(1, n_attn)
    achieved = w.flops_per_call() / (attn_ms_avg / 1e3) / 1e12
    traffic = recorded_traffic()
    roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": pk["bf16_sustained"], "unit": "TFLOP/s",
                "frac": round(achieved / pk["bf16_sustained"], 4), "traffic": traffic,
                "peak_kind": f"{pk['source']} bf16 dense, sustained (kernel timed inside a long step)"}
    # conditioning, commit; per call the attention, a latent write when the kernel does
    # not fold it in, a merge when items were cut; Euler
    launches_per_step = 2 + S + (n_attn + prof["latent_write_launches"] + prof["combine_launches"]) // max(1, args.steps)

    # ---- HBM-bound kernels, timed on their own on the same stream
    extra = hbm_kernels(ws, g, w, torch, dev, pk, x, vel, commit_k, commit_v, cond_k, cond_v, next_unit)

    # ---- end to end: the same unit step with inputs copied from pinned host memory each step
    e2e = run_e2e(args, ws, w, torch, dev, unit_step, q_all, kn_all, vn_all, vel, x0, (cond_k, cond_v), world,
                  local_rank, flops_unit)

    clocks = clk.summary()
    g.close()
    return {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_ms_max, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "layers": L, "euler_steps": S, "heads": w.n_heads, "head_dim": w.head_dim,
                   "query_tokens": w.n_query, "video_tokens": w.n_video, "audio_tokens": w.n_audio,
                   "cond_tokens": w.n_cond, "history_units": w.history_units, "keys_per_query": w.n_keys,
                   "cache_gb": round(g_cache_bytes(w) / 1e9, 1), "tflop_per_unit": round(flops_unit / 1e12, 2),
                   "unit_budget_ms": 160, "l2": "no flush: inputs larger than L2 (the 50.9 GB cache is streamed)",
                   "parallelism": f"replicas x{world}", "attention_splits": prof["last_n_split"],
                   "attention_ctas": prof["last_ctas"]},
        "roofline": roofline,
        "kernels": extra,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }


def g_cache_bytes(w):
    return w.n_layers * 2 * w.n_heads * (w.history_units + 1) * w.tokens_per_unit * w.head_dim * 2


def hbm_kernels(ws, g, w, torch, dev, pk, x, vel, commit_k, commit_v, cond_k, cond_v, next_unit):
    """Append (all-layer latent commit) and Euler update timed on their own."""
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    u = next_unit[0] - 1                         # the last committed unit: still resident
    reps = 10
    ws.ws_cache_append(g.h, u, ws.WS_SEG_LATENT, commit_k, commit_v)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        ws.ws_cache_append(g.h, u, ws.WS_SEG_LATENT, commit_k, commit_v)
    e1.record(stream)
    torch.cuda.synchronize()
    commit_ms = e0.elapsed_time(e1) / reps
    commit_bytes = 2 * 2 * commit_k.numel() * 2  # K and V, read + write
    # Euler on a buffer larger than L2 (2^28 elements = 1.5 GB moved per call)
    n = 1 << 28
    xb = torch.empty(n, dtype=torch.bfloat16, device=dev)
    vb = torch.empty(n, dtype=torch.bfloat16, device=dev)
    g.fill(xb, 12345)
    g.fill(vb, 54321)
    ws.ws_flow_step(xb, vb, 0.25)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        ws.ws_flow_step(xb, vb, 0.25)
    e1.record(stream)
    torch.cuda.synchronize()
    euler_ms = e0.elapsed_time(e1) / reps
    euler_bytes = n * 6
    del xb, vb
    hbm = pk["hbm"]
    return {
        "latent_commit": {"bytes": commit_bytes, "ms": round(commit_ms, 4),
                          "GB/s": round(commit_bytes / commit_ms / 1e6, 1),
                          "frac_of_measured_hbm": round(commit_bytes / commit_ms / 1e6 / hbm, 4),
                          "frac_of_8TBs": round(commit_bytes / commit_ms / 1e6 / 8000, 4)},
        "euler_2^28": {"bytes": euler_bytes, "ms": round(euler_ms, 4), "GB/s": round(euler_bytes / euler_ms / 1e6, 1),
                       "frac_of_measured_hbm": round(euler_bytes / euler_ms / 1e6 / hbm, 4),
                       "frac_of_8TBs": round(euler_bytes / euler_ms / 1e6 / 8000, 4)},
    }


def run_e2e(args, ws, w, torch, dev, unit_step, q_all, kn_all, vn_all, vel, x0, cond, world, local_rank,
            flops_unit):
    """Same unit step, each step's inputs copied host->device from pinned memory on a
    copy stream (double-buffered per layer-step) and the final latent copied back."""
    L, S = w.n_layers, w.steps
    n_sets = 8                                   # distinct host input sets, cycled
    qs = q_all.shape[2:]
    host = torch.empty((n_sets, 3) + tuple(qs), dtype=torch.bfloat16, pin_memory=True)
    for i in range(n_sets):
        s, l = divmod(i, L)
        host[i, 0].copy_(q_all[s, l])
        host[i, 1].copy_(kn_all[s, l])
        host[i, 2].copy_(vn_all[s, l])
    host_vel = vel.cpu().pin_memory()
    host_x = x0.cpu().pin_memory()
    host_x_out = torch.empty_like(host_x).pin_memory()
    host_ck, host_cv = cond[0].cpu().pin_memory(), cond[1].cpu().pin_memory()
    dck, dcv = torch.empty_like(cond[0]), torch.empty_like(cond[1])
    dbuf = torch.empty((2, 3) + tuple(qs), dtype=torch.bfloat16, device=dev)
    dvel = torch.empty_like(vel)
    x = torch.empty_like(x0)
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream(device=dev)
    ready = [torch.cuda.Event() for _ in range(2)]
    free = [torch.cuda.Event() for _ in range(2)]
    order = [(s, l) for s in range(S) for l in range(L)]

    def one_unit():
        with torch.cuda.stream(copy):
            x.copy_(host_x, non_blocking=True)
            dvel.copy_(host_vel, non_blocking=True)
            dck.copy_(host_ck, non_blocking=True)
            dcv.copy_(host_cv, non_blocking=True)
            first = torch.cuda.Event()
            first.record(copy)

        def stage(i):
            s, l = order[i]
            b = i % 2
            with torch.cuda.stream(copy):
                if i >= 2:
                    copy.wait_event(free[b])
                dbuf[b].copy_(host[(s * L + l) % n_sets], non_blocking=True)
                ready[b].record(copy)

        stage(0)
        comp.wait_event(first)
        pos = {sl: i for i, sl in enumerate(order)}

        def inputs(s, l):
            i = pos[(s, l)]
            if i + 1 < len(order):
                stage(i + 1)
            comp.wait_event(ready[i % 2])
            return dbuf[i % 2, 0], dbuf[i % 2, 1], dbuf[i % 2, 2]

        def after_call(s, l):
            free[pos[(s, l)] % 2].record(comp)

        unit_step(x, inputs, after_call, lambda s: dvel[s], (dck, dcv))
        host_x_out.copy_(x, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        one_unit()
    torch.cuda.synchronize()
    barrier(world, local_rank)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for _ in range(args.steps):
        one_unit()
    e1.record(comp)
    torch.cuda.synchronize()
    barrier(world, local_rank)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    h2d = (L * S * 3 * q_all[0, 0].numel() + vel.numel() + x0.numel() + 2 * cond[0].numel()) * 2
    d2h = x0.numel() * 2
    return {"value": round(aggregate(flops_unit, world, ms / 1e3, 1), 2), "unit": UNIT, "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "note": "per step, q/k_new/v_new of all 160 layer-steps, the conditioning slice, velocities and x "
                    "are copied from pinned host memory; the committed latent K/V is produced on the device"}


# ------------------------------------------------------- the oracle arm --

_ORACLE = {}


def oracle_sample(target_s: float, max_rows=None):
    """Time the fp64 oracle on a bounded sample of the same workload: up to four heads
    of one layer-step (layer 17, Euler step 1), as many (head, query row) pairs as fit
    in about target_s seconds.  Input generation is not timed."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from kv_cache_serving_ws_b200.workloads import FULL
    from oracle_side import oracle_cache
    w = FULL
    n_heads = 4
    if "case" not in _ORACLE:
        _ORACLE["case"] = oracle_cache(w, 17, list(range(n_heads)), 1)
    cache, q, kn, vn = _ORACLE["case"]
    # calibrate: the per-call cost (latent write, key assembly) and the per-pair cost
    t0 = time.perf_counter()
    cache.unit_attention(0, w.unit, q, kn, vn, rows=[], heads=[0])
    t_fixed = time.perf_counter() - t0
    t0 = time.perf_counter()
    cache.unit_attention(0, w.unit, q, kn, vn, rows=list(range(8)), heads=[0])
    t_pair = max(1e-6, (time.perf_counter() - t0 - t_fixed) / 8)
    pairs = max(2, int((target_s - t_fixed) / t_pair))
    heads = min(n_heads, max(1, -(-pairs // w.n_query)))
    rows = max(2, min(w.n_query, pairs // heads))
    if max_rows:
        rows = min(rows, max_rows)
    t0 = time.perf_counter()
    st, _ = cache.unit_attention(0, w.unit, q, kn, vn, rows=list(range(rows)), heads=list(range(heads)))
    dt = time.perf_counter() - t0
    assert st == 0
    flops = 4.0 * rows * heads * w.n_keys * w.head_dim
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"), default=1)
    except Exception:
        cores = os.cpu_count() or 1
    per_unit_s = dt * (w.n_heads / heads) * (w.n_query / rows) * w.n_layers * w.steps
    return {"value": round(flops / dt / 1e12, 6), "unit": UNIT, "cores": int(cores), "kind": "oracle",
            "sample": f"{heads} head(s) x {rows} query rows of one layer-step of {w.name} ({w.n_keys} keys) "
                      f"in {dt:.1f} s; a whole unit extrapolates to {per_unit_s:.0f} s",
            "seconds": round(dt, 2)}


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_config(w, heads: int, rows=None):
    """The fp64 oracle over `heads` heads (all query rows unless `rows`) of one attention
    call of workload w, timed on the host cores; the whole call is extrapolated from the
    sample by heads and rows (factor 1 = timed in full).  Input generation is not timed."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle_side import oracle_cache
    cache, q, kn, vn = oracle_cache(w, 0, list(range(heads)))
    rows = w.n_query if rows is None else rows
    t0 = time.perf_counter()
    st, _ = cache.unit_attention(0, w.unit, q, kn, vn, rows=list(range(rows)), heads=list(range(heads)))
    dt = time.perf_counter() - t0
    assert st == 0
    factor = (w.n_heads / heads) * (w.n_query / rows)
    flops = 4.0 * rows * heads * w.n_keys * w.head_dim
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"), default=1)
    except Exception:
        cores = os.cpu_count() or 1
    return {"kind": "oracle", "value": round(flops / dt / 1e12, 6), "unit": UNIT,
            "ms_per_call": round(dt * factor * 1e3, 1), "extrapolated_x": round(factor, 2),
            "sample": f"{heads} of {w.n_heads} heads x {rows} of {w.n_query} query rows in {dt:.2f} s",
            "cores": int(cores), "cpu": cpu_model()}


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return None
    samples = []
    for _ in range(args.warmup):
        oracle_sample(1.0, max_rows=4)
    t_all = 0.0
    for _ in range(args.steps):
        s = oracle_sample(args.ref_step_seconds)
        samples.append(s)
        t_all += s["seconds"]
    val = statistics.median([s["value"] for s in samples])
    base = dict(samples[-1])
    base["value"] = val
    from kv_cache_serving_ws_b200.workloads import FULL
    return {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(t_all / args.steps * 1e3, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": FULL.name, "sample": base["sample"]},
            "cpu_baseline": base,
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_case(args):
    """A single workload's attention calls, for profiler captures: prefill the
    history, then `calls` attention calls of layer 0 of the current unit."""
    import torch

    from kv_cache_serving_ws_b200 import native as ws
    from kv_cache_serving_ws_b200.workloads import ALL, GpuSession
    w = {"tiny": "tiny-192x336-5units-8x64", "v01": "v01-192x336-hist16-40x128", "v02": "v02-640x368-hist32-40x128",
         "ring": "v02-640x368-ring128-u1000-40x128"}.get(args.case, args.case)
    w = ALL[w]
    g = GpuSession(w)
    g.prefill()
    q, kn, vn = g.step_inputs(0)
    out = torch.empty_like(q)
    for _ in range(2):                       # warm-up: first-call set-up, caches
        ws.ws_unit_attention(g.h, 0, w.unit, q, kn, vn, out)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(args.calls):
        ws.ws_unit_attention(g.h, 0, w.unit, q, kn, vn, out)
    e1.record()
    st = ws.ws_sync(g.h, check=False)
    ms = e0.elapsed_time(e1) / max(1, args.calls)
    print(json.dumps({"case": w.name, "calls": args.calls, "ms_per_call": round(ms, 4),
                      "TFLOP/s": round(w.flops_per_call() / ms / 1e9, 1), "status": ws.status_string(st)}))
    g.close()
    if st != ws.WS_OK:
        sys.exit(1)


def run_prefill(args):
    """Prompt prefill: n query units of the 640x368 stream attend at once, each over its
    own window (block-causal across units), one layer; reports TFLOP/s of the useful
    work and the key tiles the block-causal mask skips compared with a dense one."""
    import torch

    from kv_cache_serving_ws_b200 import native as ws
    from kv_cache_serving_ws_b200 import synth
    from kv_cache_serving_ws_b200.workloads import Workload, key
    n = args.prefill_units
    w = Workload("prefill-640x368-40x128", 1, 40, 128, 920, 4, 32, 64, seed=6, unit=0)
    _, h = ws.ws_cache_create(ws.make_config(1, w.n_heads, w.head_dim, w.n_video, w.n_audio, w.n_cond,
                                             w.history_units))
    dev = torch.device("cuda")
    ck = torch.empty((1, w.n_cond, w.n_heads, w.head_dim), dtype=torch.bfloat16, device=dev)
    cv = torch.empty_like(ck)
    for u in range(n):
        ws.synth_fill(ck, key(w, synth.KIND_COND_K, u))
        ws.synth_fill(cv, key(w, synth.KIND_COND_V, u))
        ws.ws_cache_append(h, u, ws.WS_SEG_COND, ck, cv)
    shape = (n, w.n_query, w.n_heads, w.head_dim)
    q = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    kn, vn, out = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws.synth_fill(q, key(w, synth.KIND_Q, 0))
    ws.synth_fill(kn, key(w, synth.KIND_K_NEW, 0))
    ws.synth_fill(vn, key(w, synth.KIND_V_NEW, 0))
    for _ in range(2):
        ws.ws_prefill_attention(h, 0, 0, n, q, kn, vn, out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.calls):
        ws.ws_prefill_attention(h, 0, 0, n, q, kn, vn, out)
    e1.record()
    st = ws.ws_sync(h, check=False)
    ms = e0.elapsed_time(e1) / args.calls
    T = w.tokens_per_unit
    keys = [min(j, w.history_units) * T + T for j in range(n)]           # window of query unit j (from scratch)
    flops = sum(4.0 * w.n_query * k * w.n_heads * w.head_dim for k in keys)
    tiles = sum((k + 127) // 128 for k in keys)
    dense_tiles = n * ((n * T + 127) // 128)
    print(json.dumps({"mode": "prefill", "workload": w.name, "query_units": n, "query_rows": n * w.n_query,
                      "ms_per_call": round(ms, 3), "TFLOP/s": round(flops / ms / 1e9, 1),
                      "key_tiles": tiles, "dense_mask_key_tiles": dense_tiles,
                      "skipped_tile_fraction": round(1 - tiles / dense_tiles, 4), "status": ws.status_string(st)}))
    ws.ws_cache_destroy(h)
    if st != ws.WS_OK:
        sys.exit(1)


def percentiles(xs):
    a = sorted(xs)

    def pct(p):
        i = min(len(a) - 1, max(0, int(round(p / 100.0 * (len(a) - 1)))))
        return round(a[i], 3)
    return {"p50": pct(50), "p99": pct(99), "max": round(a[-1], 3), "min": round(a[0], 3),
            "mean": round(statistics.fmean(a), 3)}


def run_schedule(args):
    """Per-unit schedule of the whole unit (conditioning append, 40 layers x 4 Euler
    steps of attention, commit), units back to back and paced at the stream's 160 ms
    cadence.  Direct calls (one launch per layer call plus a few per unit) against the unit program (one CUDA
    graph per unit, updated in place).  Reports per-unit device time percentiles, the
    host time the program spends recording a unit, and, paced, the latency from a
    unit's release (its conditioning slice copied from pinned host memory) to its
    completion, with the backlog's growth per unit when a unit outlasts 160 ms."""
    import torch

    from kv_cache_serving_ws_b200 import native as ws
    from kv_cache_serving_ws_b200 import synth
    from kv_cache_serving_ws_b200.workloads import FULL, FULL32, GpuSession, key
    period_s = 0.160
    n = args.units
    for w in (FULL32, FULL):
        L, S = w.n_layers, w.steps
        g = GpuSession(w)
        dev = g.dev
        bf = torch.bfloat16
        qs = (w.n_query, w.n_heads, w.head_dim)
        n_lat = w.n_query * w.n_heads * w.head_dim
        q_all = torch.empty((S, L) + qs, dtype=bf, device=dev)
        kn_all, vn_all = torch.empty_like(q_all), torch.empty_like(q_all)
        for s in range(S):
            for l in range(L):
                g.fill(q_all[s, l], key(w, synth.KIND_Q, w.unit, l, s))
                g.fill(kn_all[s, l], key(w, synth.KIND_K_NEW, w.unit, l, s))
                g.fill(vn_all[s, l], key(w, synth.KIND_V_NEW, w.unit, l, s))
        vel = torch.empty((S, n_lat), dtype=bf, device=dev)
        for s in range(S):
            g.fill(vel[s], key(w, synth.KIND_VEL, w.unit, 0, s))
        x = torch.empty(n_lat, dtype=bf, device=dev)
        g.fill(x, key(w, synth.KIND_X, w.unit))
        out = torch.empty(qs, dtype=bf, device=dev)
        ck, cv = torch.empty_like(g.cond_k), torch.empty_like(g.cond_v)
        g.fill(ck, key(w, synth.KIND_COND_K, w.unit))
        g.fill(cv, key(w, synth.KIND_COND_V, w.unit))
        commit_k, commit_v = g.commit_buffers()
        for u in range(w.unit):
            g.append_cond(u)
            g.commit(u)
        g.fill(commit_k, key(w, synth.KIND_COMMIT_K, w.unit))
        g.fill(commit_v, key(w, synth.KIND_COMMIT_V, w.unit))
        host_ck, host_cv = ck.cpu().pin_memory(), cv.cpu().pin_memory()
        torch.cuda.synchronize()
        nxt = [w.unit]

        def direct():
            u = nxt[0]
            ws.ws_cache_append(g.h, u, ws.WS_SEG_COND, ck, cv)
            for s in range(S):
                for l in range(L):
                    ws.ws_unit_attention(g.h, l, u, q_all[s, l], kn_all[s, l], vn_all[s, l], out)
                ws.ws_flow_step(x, vel[s], w.dt)
            ws.ws_cache_append(g.h, u, ws.WS_SEG_LATENT, commit_k, commit_v)
            nxt[0] = u + 1

        _, prog = ws.ws_unit_graph_create(g.h, S, w.dt, ck, cv, q_all, kn_all, vn_all, out, x, vel, commit_k,
                                          commit_v, out_per_call=False)

        def graph():
            ws.ws_unit_graph_launch(prog, nxt[0])
            nxt[0] += 1

        def back_to_back(fn):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
            t0 = time.perf_counter()
            ev[0].record()
            for i in range(n):
                fn()
                ev[i + 1].record()
            t_host = time.perf_counter() - t0
            torch.cuda.synchronize()
            per = [ev[i].elapsed_time(ev[i + 1]) for i in range(n)]
            return per, t_host * 1e3 / n

        with ClockSampler(0) as clk:
            per_direct, host_direct = back_to_back(direct)
            s0 = ws.ws_unit_graph_get_stats(prog)
            per_graph, host_graph = back_to_back(graph)
            s1 = ws.ws_unit_graph_get_stats(prog)

            # paced: unit k is released at t0 + k * 160 ms with its conditioning slice
            torch.cuda.synchronize()
            pending, lat = [], []
            t0 = time.perf_counter() + 0.02
            k = 0
            while k < n or pending:
                now = time.perf_counter()
                while pending and pending[0][1].query():
                    lat.append((now - pending[0][0]) * 1e3)
                    pending.pop(0)
                if k < n and now >= t0 + k * period_s:
                    ck.copy_(host_ck, non_blocking=True)
                    cv.copy_(host_cv, non_blocking=True)
                    graph()
                    e = torch.cuda.Event()
                    e.record()
                    pending.append((t0 + k * period_s, e))
                    k += 1
                    continue
                time.sleep(0.0002)
        st = ws.ws_sync(g.h, check=False)
        ws.ws_unit_graph_destroy(prog)
        slope = 0.0
        if len(lat) > 1:
            xs = list(range(len(lat)))
            mx, my = statistics.fmean(xs), statistics.fmean(lat)
            slope = sum((a - mx) * (b - my) for a, b in zip(xs, lat)) / sum((a - mx) ** 2 for a in xs)
        upd = s1["updates"] - s0["updates"]
        inst = s1["instantiations"] - s0["instantiations"]
        flops_unit = w.flops_per_call() * L * S
        print(json.dumps({
            "mode": "schedule", "workload": w.name, "units": n, "unit_budget_ms": period_s * 1e3,
            "tflop_per_unit": round(flops_unit / 1e12, 2),
            "direct": {"unit_ms": percentiles(per_direct), "host_ms_per_unit": round(host_direct, 3),
                       "launches_per_unit": 2 + S + L * S * (1 if ws.ws_profile_read(g.h)["last_kernel"] == 1 else 2)},
            "graph": {"unit_ms": percentiles(per_graph), "host_ms_per_unit": round(host_graph, 3),
                      "record_ms_per_unit": round((s1["record_ms"] - s0["record_ms"]) / max(1, n + 3), 3),
                      "kernel_nodes": s1["nodes"], "updates_in_place": upd, "instantiations": inst,
                      "TFLOP/s_p50": round(flops_unit / percentiles(per_graph)["p50"] / 1e9, 1)},
            "paced_160ms": {"latency_ms": percentiles(lat), "backlog_growth_ms_per_unit": round(slope, 2),
                            "units_over_budget": sum(1 for v in lat if v > period_s * 1e3)},
            "clocks": clk.summary(), "status": ws.status_string(st)}), flush=True)
        del q_all, kn_all, vn_all
        g.close()
        torch.cuda.empty_cache()
        if st != ws.WS_OK:
            sys.exit(1)


def run_sessions(args):
    """Concurrent sessions: N conversations in one pool, their current units in one
    attention launch, against N separate launches (one layer, steady-state windows).
    Two stream shapes: the 640x368 stream with a 32-unit history and the 192x336
    stream with a 16-unit history."""
    import torch

    from kv_cache_serving_ws_b200 import native as ws
    from kv_cache_serving_ws_b200 import synth
    from kv_cache_serving_ws_b200.workloads import V01, V02
    for w, n in ((V02, args.sessions), (V01, 4 * args.sessions)):
        n = min(n, 64)
        _, h = ws.ws_pool_create(ws.make_config(1, w.n_heads, w.head_dim, w.n_video, w.n_audio, w.n_cond,
                                                w.history_units), n)
        dev = torch.device("cuda")
        bf = torch.bfloat16
        ck = torch.empty((1, w.n_cond, w.n_heads, w.head_dim), dtype=bf, device=dev)
        cv = torch.empty_like(ck)
        lk = torch.empty((1, w.n_query, w.n_heads, w.head_dim), dtype=bf, device=dev)
        lv = torch.empty_like(lk)
        units = []
        for s in range(n):
            first = 7 * s                                   # sessions at different stream positions
            for u in range(first, first + w.history_units + 1):
                ws.synth_fill(ck, synth.stream_key(w.seed + 1000 * s, synth.KIND_COND_K, u))
                ws.synth_fill(cv, synth.stream_key(w.seed + 1000 * s, synth.KIND_COND_V, u))
                ws.ws_session_append(h, s, u, ws.WS_SEG_COND, ck, cv)
                if u < first + w.history_units:
                    ws.synth_fill(lk, synth.stream_key(w.seed + 1000 * s, synth.KIND_COMMIT_K, u))
                    ws.synth_fill(lv, synth.stream_key(w.seed + 1000 * s, synth.KIND_COMMIT_V, u))
                    ws.ws_session_append(h, s, u, ws.WS_SEG_LATENT, lk, lv)
            units.append(first + w.history_units)
        shape = (n, w.n_query, w.n_heads, w.head_dim)
        q = torch.empty(shape, dtype=bf, device=dev)
        kn, vn, out = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        ws.synth_fill(q, synth.stream_key(w.seed, synth.KIND_Q, 0))
        ws.synth_fill(kn, synth.stream_key(w.seed, synth.KIND_K_NEW, 0))
        ws.synth_fill(vn, synth.stream_key(w.seed, synth.KIND_V_NEW, 0))
        sess = list(range(n))

        def batched():
            ws.ws_session_attention(h, 0, sess, units, q, kn, vn, out)

        def separate():
            for s in sess:
                ws.ws_session_attention(h, 0, [s], [units[s]], q[s], kn[s], vn[s], out[s])

        def timed(fn):
            for _ in range(2):
                fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(args.calls):
                fn()
            e1.record()
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / args.calls

        ms_b = timed(batched)
        ms_s = timed(separate)
        st = ws.ws_sync(h, check=False)
        flops = n * w.flops_per_call()
        print(json.dumps({"mode": "sessions", "workload": w.name, "sessions": n, "keys_per_query": w.n_keys,
                          "batched": {"ms_per_call": round(ms_b, 4), "TFLOP/s": round(flops / ms_b / 1e9, 1),
                                      "attention_launches": 1},
                          "separate": {"ms_per_call": round(ms_s, 4), "TFLOP/s": round(flops / ms_s / 1e9, 1),
                                       "attention_launches": n},
                          "speedup": round(ms_s / ms_b, 3), "status": ws.status_string(st)}), flush=True)
        ws.ws_cache_destroy(h)
        del q, kn, vn, out
        torch.cuda.empty_cache()
        if st != ws.WS_OK:
            sys.exit(1)


def run_configs(args):
    """Attention of one layer at each configuration of the scope table, one call at a
    time with L2 flushed before each (a 256 MB write), CUDA events around the call
    only: 5 warm-up calls, then `calls` timed ones; median and min.  Reports TFLOP/s
    against the measured burst bf16 peak (a kernel timed alone) and, for the small
    cases, the byte roofline (K/V read once + Q, k_new, v_new and the output)."""
    import torch

    from kv_cache_serving_ws_b200 import native as ws
    from kv_cache_serving_ws_b200.workloads import RING, TINY, V01, V02, GpuSession
    pk = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for w in (TINY, V01, V02, RING):
        g = GpuSession(w)
        g.prefill()
        q, kn, vn = g.step_inputs(0)
        out = torch.empty_like(q)
        for _ in range(5):
            ws.ws_unit_attention(g.h, 0, w.unit, q, kn, vn, out)
        times = []
        for _ in range(args.calls):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            ws.ws_unit_attention(g.h, 0, w.unit, q, kn, vn, out)
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        st = ws.ws_sync(g.h, check=False)
        med, mn = statistics.median(times), min(times)
        flops = w.flops_per_call()
        kv_bytes = 2 * w.n_keys * w.n_heads * w.head_dim * 2
        io_bytes = 4 * w.n_query * w.n_heads * w.head_dim * 2
        t_compute = flops / (pk["bf16"] * 1e12) * 1e3
        t_memory = (kv_bytes + io_bytes) / (pk["hbm"] * 1e9) * 1e3
        line = {"mode": "configs", "workload": w.name, "calls": args.calls, "l2": "flushed before each call",
                "ms_median": round(med, 4), "ms_min": round(mn, 4),
                "TFLOP/s": round(flops / med / 1e9, 1),
                "frac_of_burst_bf16": round(flops / med / 1e9 / pk["bf16"], 4),
                "bytes": kv_bytes + io_bytes, "GB/s": round((kv_bytes + io_bytes) / med / 1e6, 1),
                "frac_of_measured_hbm": round((kv_bytes + io_bytes) / med / 1e6 / pk["hbm"], 4),
                "roofline_ms": round(max(t_compute, t_memory), 4),
                "bound": "tensor" if t_compute >= t_memory else "hbm",
                "status": ws.status_string(st)}
        g.close()
        if not args.no_cpu_baseline:
            # the oracle beside it: in full for the tiny and 192x336 cases, four heads
            # (all rows) at 640x368 and one head of the 128-unit ring, extrapolated
            heads = {TINY.name: TINY.n_heads, V01.name: V01.n_heads, V02.name: 4, RING.name: 1}[w.name]
            line["cpu_baseline"] = oracle_config(w, heads)
            line["cpu_baseline"]["gpu_speedup"] = round(line["cpu_baseline"]["ms_per_call"] / med, 1)
        print(json.dumps(line), flush=True)
        if args.library:
            for name, res in library_attention(w, args.calls, flush):
                line = {"mode": "configs", "impl": "library:" + name, "workload": w.name, "calls": args.calls,
                        "l2": "flushed before each call"}
                if isinstance(res, str):
                    line["unavailable"] = res
                else:
                    line.update({"ms_median": round(res, 4), "TFLOP/s": round(flops / res / 1e9, 1),
                                 "frac_of_burst_bf16": round(flops / res / 1e9 / pk["bf16"], 4)})
                print(json.dumps(line), flush=True)


def library_attention(w, calls, flush):
    """Context for the configurations above: vendor attention kernels timed on dense
    bf16 N(0,1) tensors of the same sizes (a one-unit query sees every key of its
    window, so the FLOPs are the same), with the same protocol (L2 flushed, CUDA events
    around the call, 5 warm-up calls, median).  Never on the product path.  Yields
    (name, median ms) or (name, reason it could not run)."""
    import torch
    import torch.nn.functional as F

    nq, nk, H, D = w.n_query, w.n_keys, w.n_heads, w.head_dim

    def timed(fn):
        for _ in range(5):
            fn()
        ts = []
        for _ in range(calls):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    gen = torch.Generator(device="cuda").manual_seed(w.seed)
    q = torch.randn(nq, H, D, device="cuda", dtype=torch.bfloat16, generator=gen)
    k = torch.randn(nk, H, D, device="cuda", dtype=torch.bfloat16, generator=gen)
    v = torch.randn(nk, H, D, device="cuda", dtype=torch.bfloat16, generator=gen)
    try:
        from torch.nn.attention import SDPBackend, sdpa_kernel
        qh, kh, vh = (t.transpose(0, 1).unsqueeze(0).contiguous() for t in (q, k, v))
        with sdpa_kernel([SDPBackend.CUDNN_ATTENTION]):
            yield "torch-sdpa-cudnn", timed(lambda: F.scaled_dot_product_attention(qh, kh, vh))
        del qh, kh, vh
    except Exception as ex:                                   # noqa: BLE001 - reported, not hidden
        yield "torch-sdpa-cudnn", f"{type(ex).__name__}: {str(ex)[:160]}"
    for backend in ("cutlass", "cute-dsl"):
        try:
            import flashinfer
            ws_buf = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
            fw = flashinfer.BatchPrefillWithRaggedKVCacheWrapper(ws_buf, "NHD", backend=backend)
            ind = lambda n: torch.tensor([0, n], dtype=torch.int32, device="cuda")
            fw.plan(ind(nq), ind(nk), H, H, D, causal=False, q_data_type=torch.bfloat16,
                    kv_data_type=torch.bfloat16)
            yield "flashinfer-" + backend, timed(lambda: fw.run(q, k, v))
            del fw, ws_buf
        except Exception as ex:                               # noqa: BLE001 - reported, not hidden
            yield "flashinfer-" + backend, f"{type(ex).__name__}: {str(ex)[:160]}"


def run_euler_sweep(args):
    """Euler update bandwidth over n = 2^20 .. 2^28 elements (6 bytes moved per
    element), inputs larger than L2 from 2^25 on, L2 flushed before each call below."""
    import torch

    from kv_cache_serving_ws_b200 import native as ws
    pk = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for lg in range(20, 29):
        n = 1 << lg
        x = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        v = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        ws.synth_fill(x, 1000 + lg)
        ws.synth_fill(v, 2000 + lg)
        for _ in range(3):
            ws.ws_flow_step(x, v, 0.25)
        times = []
        for _ in range(args.calls):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            ws.ws_flow_step(x, v, 0.25)
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        med = statistics.median(times)
        gbs = 6 * n / med / 1e6
        print(json.dumps({"mode": "euler_sweep", "n": n, "bytes": 6 * n, "ms_median": round(med, 5),
                          "GB/s": round(gbs, 1), "frac_of_measured_hbm": round(gbs / pk["hbm"], 4),
                          "frac_of_8TBs": round(gbs / 8000, 4)}), flush=True)
        del x, v


def run_hbm_kernels(args):
    """The HBM-bound kernels at sizes larger than L2 on a small cache (a few GB on the
    device, so ncu can capture them): the 40-layer latent commit of one 640x368 unit
    (append_kernel, 1.51 GB moved) into a 40-layer cache with a one-unit history, and
    the Euler update of 2^28 elements (euler_kernel, 1.61 GB moved).  3 warm-up calls,
    then `calls` timed ones, each after a 256 MB write that flushes L2; CUDA events
    around the call only; median."""
    import torch

    from kv_cache_serving_ws_b200 import native as ws
    from kv_cache_serving_ws_b200 import synth
    pk = peaks()
    L, H, D, Nv, Na, Nc = 40, 40, 128, 920, 4, 32
    _, h = ws.ws_cache_create(ws.make_config(L, H, D, Nv, Na, Nc, 1))
    dev = torch.device("cuda")
    ck = torch.empty((L, Nc, H, D), dtype=torch.bfloat16, device=dev)
    cv = torch.empty_like(ck)
    ws.synth_fill(ck, synth.stream_key(8, synth.KIND_COND_K, 0))
    ws.synth_fill(cv, synth.stream_key(8, synth.KIND_COND_V, 0))
    ws.ws_cache_append(h, 0, ws.WS_SEG_COND, ck, cv)
    lk = torch.empty((L, Nv + Na, H, D), dtype=torch.bfloat16, device=dev)
    lv = torch.empty_like(lk)
    ws.synth_fill(lk, synth.stream_key(8, synth.KIND_COMMIT_K, 0))
    ws.synth_fill(lv, synth.stream_key(8, synth.KIND_COMMIT_V, 0))
    n = 1 << 28
    x = torch.empty(n, dtype=torch.bfloat16, device=dev)
    v = torch.empty(n, dtype=torch.bfloat16, device=dev)
    ws.synth_fill(x, 12345)
    ws.synth_fill(v, 54321)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def timed(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(args.calls):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    cases = (("append_kernel", "latent commit, 40 layers x 924 rows x 40 heads x 128, K and V",
              2 * 2 * lk.numel() * 2, lambda: ws.ws_cache_append(h, 0, ws.WS_SEG_LATENT, lk, lv)),
             ("euler_kernel", "x <- RN_bf16(x + 0.25 v), 2^28 elements", 6 * n,
              lambda: ws.ws_flow_step(x, v, 0.25)))
    for kernel, what, nbytes, fn in cases:
        ms = timed(fn)
        gbs = nbytes / ms / 1e6
        print(json.dumps({"mode": "hbm_kernels", "kernel": kernel, "what": what, "bytes": nbytes,
                          "calls": args.calls, "l2": "flushed before each call", "ms_median": round(ms, 4),
                          "GB/s": round(gbs, 1), "frac_of_measured_hbm": round(gbs / pk["hbm"], 4),
                          "frac_of_8TBs": round(gbs / 8000, 4)}), flush=True)
    st = ws.ws_sync(h, check=False)
    ws.ws_cache_destroy(h)
    if st != ws.WS_OK:
        sys.exit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-baseline-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-seconds", type=float, default=5.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default=None, help="profiling mode: tiny|v01|v02|ring (attention calls only)")
    ap.add_argument("--calls", type=int, default=3)
    ap.add_argument("--prefill", action="store_true", help="time a multi-unit prompt prefill instead")
    ap.add_argument("--prefill-units", type=int, default=64)
    ap.add_argument("--schedule", action="store_true",
                    help="per-unit schedule: direct calls vs the unit program, back to back and paced at 160 ms")
    ap.add_argument("--units", type=int, default=24)
    ap.add_argument("--configs", action="store_true", help="attention of one layer at every configuration, L2 flushed")
    ap.add_argument("--library", action="store_true",
                    help="with --configs: also time vendor attention kernels on dense tensors of the same sizes")
    ap.add_argument("--euler-sweep", action="store_true", help="Euler update bandwidth for n = 2^20 .. 2^28")
    ap.add_argument("--hbm-kernels", action="store_true",
                    help="latent commit and Euler update on a small cache, L2 flushed (ncu capture target)")
    ap.add_argument("--sessions", type=int, default=0,
                    help="concurrent sessions: N conversations batched in one launch vs N launches")
    args = ap.parse_args()
    if args.case:
        run_case(args)
        return
    if args.prefill:
        run_prefill(args)
        return
    if args.schedule:
        run_schedule(args)
        return
    if args.sessions:
        run_sessions(args)
        return
    if args.configs:
        run_configs(args)
        return
    if args.euler_sweep:
        run_euler_sweep(args)
        return
    if args.hbm_kernels:
        run_hbm_kernels(args)
        return
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    rank, local_rank, world = dist_env()
    if args.impl == "reference":
        line = run_reference(args)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, local_rank, world)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_sample(args.cpu_baseline_seconds)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
