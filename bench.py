#!/usr/bin/env python
"""Benchmark of the Graph Machine sparse-layer hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  1. gm_ser_sea_forward  - SER (two-hop referral, merge, top-s1) fused with SEA forward,
  2. gm_sea_backward     - the SEA backward (dq, dK/dV, d ln w) on the refreshed edges with
                           upstream gradient dO: edge count, scan, row pass, per-target gather.
Metric: tokens/s per sparse layer (B*n tokens per step / step time), summed over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Timing: W untimed warm-up steps, then exactly K steps between a barrier +
torch.cuda.synchronize() on both sides, timed with CUDA events on the launching stream, max
over ranks. The inputs (q, k, v, dO, edges: 0.55 GB per step at the default workload) are
larger than the 126 MB L2, so no flush runs between steps. Per-call CUDA events inside the
timed region give each call's average duration, which with the compulsory bytes counted
from the actual index tensors gives the HBM roofline fraction. SM clocks and throttle
reasons are sampled through NVML during the timed region.

`--impl reference` times the CPU oracle (the plain C restatement used by the tests) on the
host cores on a bounded sample of the same workload, in the same units.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_dynamic_routing_b200 import inputs as I  # noqa: E402

DEFAULT_WORKLOAD = "layer_b8_n4096_s4_local"
METRIC = "SER+SEA tokens/s per sparse layer (1xB200) and achieved HBM GB/s vs ~8 TB/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(I.WORKLOADS))
    p.add_argument("--batch", type=int, default=None,
                   help="override the workload's batch size (small cases for profiling)")
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra", action="store_true",
                   help="skip the separately timed calls around the step (legs, SER backward)")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="target CPU time of the oracle sample")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the other workloads (s = 2 layer, 21-layer stack, n = 32768 step)")
    p.add_argument("--profile-call", default=None, choices=["dense_refresh"],
                   help="run only this call, warmup + steps times, for a profiler; print nothing")
    p.add_argument("--write-traffic", default=None, metavar="CSV",
                   help="write profiles/dram_traffic.txt from an ncu --csv log of dram__bytes_read.sum "
                        "and dram__bytes_write.sum over a bench run (no GPU needed), then exit")
    p.add_argument("--traffic-batch", type=int, default=None,
                   help="batch size the --write-traffic capture ran at (traffic is scaled to the workload's)")
    p.add_argument("--traffic-command", default="",
                   help="the command line of the capture, recorded in the table")
    return p.parse_args(argv)


# ---- distributed plumbing ------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def shard_seed(wl: I.Workload, rank: int) -> I.Workload:
    """Weak scaling: every rank runs the full per-GPU workload on its own independent draw."""
    return wl if rank == 0 else wl.with_(seed=wl.seed + 7919 * rank)


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of x over all ranks (the bench reports the slowest rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, local: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local])


# ---- clocks ----------------------------------------------------------------------------------

class ClockSampler:
    """Polls SM clock, power and clock-event reasons through NVML (read-only)."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.ok = False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            phys = device_index
            if vis:
                ids = [v.strip() for v in vis.split(",") if v.strip()]
                if device_index < len(ids) and ids[device_index].isdigit():
                    phys = int(ids[device_index])
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(phys)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                t = time.perf_counter()
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((t, mhz, rs, pw))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.thread.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.thread.join()

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed_region"
        if len(inside) < 3:  # a short timed region: widen to the samples around it
            pad = 0.25
            inside = [s for s in self.samples if t0 - pad <= s[0] <= t1 + pad]
            window = "timed_region+-250ms"
        if not inside:
            return {"error": "no samples"}
        reasons = 0
        for s in inside:
            reasons |= s[2]
        names = sorted(k for k, v in self.REASONS.items() if reasons & v and k != "gpu_idle")
        return {
            "sm_mhz": statistics.median(s[1] for s in inside),
            "sm_max_mhz": self.max_mhz,
            "reasons": names,
            "power_w_max": max(s[3] for s in inside),
            "samples": len(inside),
            "window": window,
            "source": "nvml",
        }


# ---- byte accounting --------------------------------------------------------------------------

def distinct_rows(idx: np.ndarray, w: np.ndarray, n: int) -> int:
    """Distinct (b, t, h) rows referenced by the active slots of an edge tensor [B,n,H,s]."""
    B, _, H, s = idx.shape
    act = w > 0
    b = np.broadcast_to(np.arange(B)[:, None, None, None], idx.shape)
    h = np.broadcast_to(np.arange(H)[None, None, :, None], idx.shape)
    keys = (b[act].astype(np.int64) * n + idx[act]) * H + h[act]
    return int(np.unique(keys).size)


def compulsory_bytes(wl: I.Workload, a1_idx, a1_w, ap_idx, ap_w) -> dict:
    """Minimum DRAM bytes of each call: every input byte read once, every output written once,
    gathered rows counted once per distinct row actually referenced."""
    es = 2 if wl.dtype == "bf16" else 4
    B, n, hq, hkv, d = wl.B, wl.n, wl.hq, wl.hkv, wl.d
    tok = B * n
    feat_q = tok * hq * d * es
    kv_row = d * es
    a2_rows = distinct_rows(a1_idx, a1_w, n)
    kv_rows = distinct_rows(ap_idx, ap_w, n)
    fwd = {
        "q": feat_q, "o": feat_q, "lse": tok * hq * 4,
        "a1": tok * hkv * wl.s2 * 8, "a2_rows": a2_rows * wl.s3 * 8,
        "a_prime": tok * hkv * wl.s1 * 8, "kv_rows": kv_rows * kv_row * 2,
    }
    bwd = {
        "q_dout": 2 * feat_q, "edges": tok * hkv * wl.s1 * 8, "kv_rows": kv_rows * kv_row * 2,
        "dq": tok * hq * d * 4, "dlogw": tok * hkv * wl.s1 * 4,
        "dk_dv": 2 * tok * hkv * d * 4,  # every gradient row is written once (zeros included)
    }
    logical_fwd = (2 * hq * d * es + hq * 4
                   + hkv * (wl.s2 * 8 + wl.s2 * wl.s3 * 8 + wl.s1 * 8 + wl.s1 * 2 * kv_row)) * tok
    return {
        "fused_forward": sum(fwd.values()), "backward": sum(bwd.values()),
        "fused_forward_logical": logical_fwd,
        "kv_rows_touched": kv_rows, "kv_rows_total": tok * hkv, "a2_rows_touched": a2_rows,
        "detail": {"fused_forward": fwd, "backward": bwd},
    }


def source_hash() -> str:
    h = hashlib.sha256()
    cdir = os.path.join(ROOT, "sparse_dynamic_routing_b200", "csrc")
    for name in sorted(os.listdir(cdir)):
        if name.endswith((".cu", ".cuh")):
            h.update(open(os.path.join(cdir, name), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    cur = source_hash()
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        f = dict(kv.split("=", 1) for kv in line.split())
        if f.get("kernel") == kernel.replace(" ", "_") and f.get("workload") == workload:
            if f.get("source") != cur:
                return None
            return float(f["dram_bytes_per_launch"])
    return None


# The kernels of each timed call, as ncu names them (one launch of each per call).
TRAFFIC_CALLS = {
    "sea_fwd_tile_kernel (fused SER->SEA)": ("sea_fwd_tile_kernel",),
    "gm_sea_backward (count + scan + row pass + gather)": (
        "zero_i32_kernel", "edge_count_kernel", "scan_lookback_kernel", "sea_bwd_tile_kernel",
        "sea_bwd_gather_kernel"),
}


def write_traffic_table(csv_path: str, workload: str, capture_batch: int, command: str) -> str:
    """profiles/dram_traffic.txt from ncu's per-launch DRAM byte counters: per kernel the median
    over its launches, summed over the call's kernels, scaled from the captured batch to the
    workload's (every kernel processes the B*n*hkv edge rows independently)."""
    import csv
    per = {}  # (launch id, kernel) -> bytes
    with open(csv_path) as fh:
        rows = [ln for ln in fh if ln.startswith('"')]
    for r in csv.DictReader(rows):
        if r["Metric Name"] not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        name = r["Kernel Name"].replace("void ", "").split("<")[0].split("(")[0].strip()
        scale_unit = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}[r["Metric Unit"]]
        key = (r["ID"], name)
        per[key] = per.get(key, 0.0) + float(r["Metric Value"].replace(",", "")) * scale_unit
    by_kernel = {}
    for (_, name), b in per.items():
        by_kernel.setdefault(name, []).append(b)
    wl = I.WORKLOADS[workload]
    scale = wl.B / capture_batch
    lines = [
        "# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the bench's timed",
        f"# calls on {workload} (B={wl.B}), read by bench.py for the roofline's \"traffic\" field.",
        f"# Written by `python bench.py --write-traffic <csv> --traffic-batch {capture_batch}` from one ncu",
        f"# capture at B={capture_batch}, scaled by {scale:g}: every kernel processes the B*n*hkv edge rows",
        "# independently. Per kernel the median over its launches; a call sums its kernels. DRAM write",
        "# bytes count lines written back during the kernel: results still dirty in L2 at its end are",
        "# not counted, so writes can read below the bytes a kernel stores.",
        f"# Capture: {command}",
        "# `source` is bench.py's hash of the kernel sources; when they change bench.py reports null.",
    ]
    src = source_hash()
    for call, kernels in TRAFFIC_CALLS.items():
        parts = {}
        for k in kernels:
            if k not in by_kernel:
                raise SystemExit(f"{csv_path}: no DRAM counters for {k}")
            parts[k] = statistics.median(by_kernel[k]) * scale
        detail = ",".join(f"{k}:{int(v)}" for k, v in parts.items())
        lines.append(f"kernel={call.replace(' ', '_')} workload={workload} "
                     f"dram_bytes_per_launch={int(sum(parts.values()))} source={src} kernels={detail}")
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    with open(path, "w") as fh:
        fh.write("\n".join(lines) + "\n")
    return path


def peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            return float(json.load(fh)["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_HBM_GBS, "fallback"


# ---- CPU oracle (baseline / reference arm) -------------------------------------------------------

def oracle_sample_step(wl: I.Workload, x: dict) -> None:
    import oracle
    oi, ow, _ = oracle.ser(x["a1_idx"], x["a1_w"], x["a2_idx"], x["a2_w"], wl.s1)
    oracle.sea_forward(x["q"], x["k"], x["v"], oi, ow, wl.scale)
    oracle.sea_backward(x["q"], x["k"], x["v"], x["dout"], oi, ow, wl.scale)


def cpu_baseline(wl: I.Workload, seconds: float) -> dict:
    """Oracle (SER + SEA forward + SEA backward) on one sequence of the workload: best of 3 passes
    on all host threads, and best of 3 on one thread (bounded by `seconds` in total)."""
    import oracle
    sample = wl.with_(B=1)
    x = I.make(sample, grad=True)
    x = {k: (v.float().numpy() if v.dtype == torch.bfloat16 else v.numpy()) for k, v in x.items()}
    cores = oracle.num_threads()

    def best_of(reps, budget):
        times = []
        for _ in range(reps):
            t0 = time.perf_counter()
            oracle_sample_step(sample, x)
            times.append(time.perf_counter() - t0)
            if sum(times) > budget:
                break
        return min(times), len(times)

    best_all, n_all = best_of(3, seconds / 3)
    oracle.set_num_threads(1)
    try:
        best_one, n_one = best_of(3, 2 * seconds / 3)
    finally:
        oracle.set_num_threads(cores)
    return {
        "value": sample.n / best_all, "unit": "tokens/s", "cores": cores, "kind": "oracle",
        "sample": f"1 of {wl.B} sequences ({sample.n} tokens, same recipe): SER + SEA fwd + SEA bwd "
                  f"in the C oracle, best of {n_all} passes on {cores} threads",
        "one_core": {"value": sample.n / best_one, "unit": "tokens/s", "cores": 1,
                     "sample": f"same sequence, best of {n_one} passes on 1 thread"},
    }


# ---- our arm -------------------------------------------------------------------------------------

def run_ours(args):
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    import sparse_dynamic_routing_b200 as gm
    gm.load_library()

    wl = I.WORKLOADS[args.workload]
    if args.batch is not None:
        wl = wl.with_(B=args.batch)
    wl = shard_seed(wl, rank)
    assert wl.kind == "ser_sea", "the bench step is SER->SEA forward + SEA backward"
    x = I.make(wl, grad=True)
    g = {k: v.to(dev) for k, v in x.items()}
    B, n, hq, hkv, d = wl.B, wl.n, wl.hq, wl.hkv, wl.d
    f32 = torch.float32
    if args.profile_call == "dense_refresh":
        lse_dense = causal_lse(g["q"], g["k"], wl.scale)
        for _ in range(args.warmup + args.steps):
            gm.gm_dense_refresh_edges(g["q"], g["k"], lse_dense, wl.s1, wl.scale)
        gm.gm_check_device_errors()
        return None
    ap_i = torch.empty((B, n, hkv, wl.s1), dtype=torch.int32, device=dev)
    ap_w = torch.empty((B, n, hkv, wl.s1), dtype=f32, device=dev)
    o = torch.empty_like(g["q"])
    lse = torch.empty((B, n, hq), dtype=f32, device=dev)
    dq = torch.empty((B, n, hq, d), dtype=f32, device=dev)
    dk = torch.empty((B, n, hkv, d), dtype=f32, device=dev)
    dv = torch.empty_like(dk)
    dlw = torch.empty((B, n, hkv, wl.s1), dtype=f32, device=dev)
    ws_bytes = gm.gm_sea_backward_workspace_size(g["q"].dtype, wl.s1, B, n, hq, hkv, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        gm.gm_ser_sea_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"], g["a2_idx"],
                              g["a2_w"], wl.s1, wl.scale, out_idx=ap_i, out_w=ap_w, o=o, lse=lse,
                              stream=stream)
        if ev is not None:
            ev[1].record(stream)
        gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], ap_i, ap_w, wl.scale, dq=dq, dk=dk,
                           dv=dv, dlogw=dlw, workspace=ws, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    # fused forward; backward = counter zero-fill, count pass, three scan passes, row pass,
    # gather (with a workspace) or zero-fill + scatter row pass (without)
    launches_per_step = 1 + (7 if ws is not None else 2)

    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    gm.gm_check_device_errors(stream)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier(world, local)
    torch.cuda.synchronize(dev)
    w0 = time.perf_counter()
    t_start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    w1 = time.perf_counter()
    barrier(world, local)
    sampler.stop()
    clocks = sampler.summary(w0, w1)
    gm.gm_check_device_errors(stream)

    ms_local = t_start.elapsed_time(t_end)
    ms = max_over_ranks(ms_local, world, dev)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    tokens = B * n * world
    value = tokens * args.steps / (ms / 1e3)

    # byte accounting from the actual edge tensors (outside the timed region)
    cb = compulsory_bytes(wl, x["a1_idx"].numpy(), x["a1_w"].numpy(), ap_i.cpu().numpy(),
                          ap_w.cpu().numpy())
    peak, peak_kind = peak_hbm()
    calls = {
        "fused_forward": {"kernel": "sea_fwd_tile_kernel (fused SER->SEA)", "us": fwd_ms * 1e3,
                          "bytes": cb["fused_forward"]},
        "backward": {"kernel": "gm_sea_backward (count + scan + row pass + gather)"
                     if ws is not None else "gm_sea_backward (zero-fill + scatter row pass)",
                     "us": bwd_ms * 1e3, "bytes": cb["backward"]},
    }
    for c in calls.values():
        c["GBps"] = c["bytes"] / (c["us"] * 1e-6) / 1e9
        c["frac"] = c["GBps"] / peak
    calls["fused_forward"]["logical_bytes"] = cb["fused_forward_logical"]
    calls["fused_forward"]["logical_GBps"] = (cb["fused_forward_logical"]
                                              / (fwd_ms * 1e-3) / 1e9)
    dom_name = max(calls, key=lambda k: calls[k]["us"])
    dom = calls[dom_name]
    roofline = {
        "bound": "hbm", "kernel": dom["kernel"], "call": dom_name,
        "achieved": round(dom["GBps"], 1), "peak": peak, "unit": "GB/s",
        "frac": round(dom["frac"], 4), "peak_kind": peak_kind,
        "traffic": ncu_traffic(dom["kernel"], wl.name),
        "bytes_per_launch": dom["bytes"], "bytes_kind": "compulsory",
    }

    extra = None
    if not args.no_extra:
        extra = measure_extra(gm, wl, g, x, ap_i, ap_w, dlw, dev, stream, peak)

    configs = None
    if not args.no_configs:
        configs = measure_configs(gm, dev, stream, peak)

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(gm, wl, x, dev, stream, args.e2e_steps, world)

    result = None
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            cpu = cpu_baseline(wl, args.cpu_seconds)
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16"
            if wl.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {
                "workload": wl.name, "B_per_gpu": B, "n": n, "hq": hq, "hkv": hkv, "d": d,
                "s1": wl.s1, "s2": wl.s2, "s3": wl.s3, "alpha": wl.alpha,
                "local_frac": wl.local_frac, "step": "ser_sea_forward + sea_backward",
                "global_batch": B * world, "seq_len": n, "parallelism": f"dp{world}",
                "l2": "no flush; inputs larger than L2 "
                      f"({(cb['detail']['backward']['q_dout'] + 2 * g['k'].numel() * g['k'].element_size()) / 1e6:.0f} MB read per step)",
            },
            "roofline": roofline,
            "calls": {k: {kk: (round(vv, 3) if isinstance(vv, float) else vv)
                          for kk, vv in c.items()} for k, c in calls.items()},
            "extra_calls": extra, "configs": configs,
            "kv_rows_touched_frac": cb["kv_rows_touched"] / cb["kv_rows_total"],
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks, "source_hash": source_hash(),
        }
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return result


def measure_extra(gm, wl, g, x, ap_i, ap_w, dlw, dev, stream, peak, reps=20):
    """The calls around the step, each timed alone with CUDA events, L2 flushed between reps.

    ser_forward and sea_forward are the fused forward's two halves as separate calls, and
    ser_forward_then_sea_forward the pair in sequence (A' written, then read back);
    leg_sparsify builds the step's two legs from the workload's stored edges; ser_backward
    takes the step's d ln w back to the legs; leg_backward takes those leg gradients back to
    the stored weights and the mixing coefficients; ser_sea_refresh_forward is the fused
    forward with the stored edges joining the referral as refresh edges;
    ser_sea_chain_forward is the fused forward through a three-leg referral chain;
    ser_refresh_backward and ser_chain_backward take the step's d ln w back through the
    referral with refresh edges and through the three-leg chain. Bytes are
    compulsory: every input read once, every output written once (ser_backward's second-leg
    rows counted in full; the refresh and chain forwards' gathered rows counted from their own
    edges, the chain's third leg in full).
    """
    le = {k: v.to(dev) for k, v in I.leg_inputs(wl).items()}
    B, n, k = wl.B, wl.n, wl.hkv
    tok = B * n
    f32 = torch.float32
    a1i = torch.empty((B, n, k, wl.s2), dtype=torch.int32, device=dev)
    a1w = torch.empty((B, n, k, wl.s2), dtype=f32, device=dev)
    a2i = torch.empty((B, n, k, wl.s3), dtype=torch.int32, device=dev)
    a2w = torch.empty((B, n, k, wl.s3), dtype=f32, device=dev)
    dw1 = torch.empty((B, n, k, wl.s2), dtype=f32, device=dev)
    dw2 = torch.empty((B, n, k, wl.s3), dtype=f32, device=dev)
    dew = torch.empty((B, n, k, wl.s1), dtype=f32, device=dev)
    dm1 = torch.empty((B, n, k, k), dtype=f32, device=dev)
    dm2 = torch.empty_like(dm1)
    # L2 is evicted by reading a 256 MB buffer (a write would leave dirty lines whose
    # write-back the next timed call would pay for)
    flush = torch.zeros(64 << 20, dtype=torch.int32, device=dev)
    rf_i = torch.empty_like(ap_i)
    rf_w = torch.empty_like(ap_w)
    rf_o = torch.empty_like(g["q"])
    rf_lse = torch.empty((B, n, wl.hq), dtype=f32, device=dev)
    gm.gm_ser_sea_refresh_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"], g["a2_idx"],
                                  g["a2_w"], le["e_idx"], le["e_w"], wl.s1, wl.scale, out_idx=rf_i,
                                  out_w=rf_w, o=rf_o, lse=rf_lse, stream=stream)
    torch.cuda.synchronize(dev)
    rf_bytes = (compulsory_bytes(wl, x["a1_idx"].numpy(), x["a1_w"].numpy(), rf_i.cpu().numpy(),
                                 rf_w.cpu().numpy())["fused_forward"] + e_b_refresh(wl))
    # a three-leg chain (the pages' R3): the step's two legs and one more drawn the same way
    leg3 = [v.to(dev) for v in I.edges(wl, 2, wl.s3, layer=1)]
    ch_legs = [(g["a2_idx"], g["a2_w"]), (leg3[0], leg3[1])]
    ch_i = torch.empty_like(ap_i)
    ch_w = torch.empty_like(ap_w)
    ch_o = torch.empty_like(g["q"])
    ch_lse = torch.empty((B, n, wl.hq), dtype=f32, device=dev)
    gm.gm_ser_sea_chain_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"], ch_legs, wl.s2,
                                wl.s1, wl.scale, out_idx=ch_i, out_w=ch_w, o=ch_o, lse=ch_lse,
                                stream=stream)
    torch.cuda.synchronize(dev)
    ch_bytes = (compulsory_bytes(wl, x["a1_idx"].numpy(), x["a1_w"].numpy(), ch_i.cpu().numpy(),
                                 ch_w.cpu().numpy())["fused_forward"] + tok * k * wl.s3 * 8)
    rf_dw1 = torch.empty((B, n, k, wl.s2), dtype=f32, device=dev)
    rf_dw2 = torch.empty((B, n, k, wl.s3), dtype=f32, device=dev)
    rf_dfw = torch.empty((B, n, k, wl.s1), dtype=f32, device=dev)
    ch_dw1 = torch.empty((B, n, k, wl.s2), dtype=f32, device=dev)
    ch_dl = [torch.empty((B, n, k, wl.s3), dtype=f32, device=dev) for _ in ch_legs]
    e_b, mix_b = tok * k * wl.s1 * 8, 2 * tok * k * k * 4
    leg_b, grad_b = tok * k * (wl.s2 + wl.s3) * 8, tok * k * (wl.s2 + wl.s3) * 4
    # the fused backward of the referral and the attention (its bytes: the attention backward's
    # plus the legs read, their gradients written, dw2 read-modify-written)
    bwd_b = compulsory_bytes(wl, x["a1_idx"].numpy(), x["a1_w"].numpy(), ap_i.cpu().numpy(),
                             ap_w.cpu().numpy())["backward"]
    f_dq = torch.empty((B, n, wl.hq, wl.d), dtype=f32, device=dev)
    f_dk = torch.empty((B, n, k, wl.d), dtype=f32, device=dev)
    f_dv = torch.empty_like(f_dk)
    f_dlw = torch.empty((B, n, k, wl.s1), dtype=f32, device=dev)
    f_dw1 = torch.empty((B, n, k, wl.s2), dtype=f32, device=dev)
    f_dw2 = torch.empty((B, n, k, wl.s3), dtype=f32, device=dev)
    f_ws = torch.empty(gm.gm_sea_backward_workspace_size(g["q"].dtype, wl.s1, B, n, wl.hq, k, wl.d),
                       dtype=torch.uint8, device=dev)
    # the two halves of the fused forward as separate calls (the unfused entry points
    # gm_ser_forward and gm_sea_forward), and the two in sequence: A' makes one round trip
    # through HBM
    fd = compulsory_bytes(wl, x["a1_idx"].numpy(), x["a1_w"].numpy(), ap_i.cpu().numpy(),
                          ap_w.cpu().numpy())["detail"]["fused_forward"]
    ser_b = fd["a1"] + fd["a2_rows"] + fd["a_prime"]
    sea_b = fd["q"] + fd["o"] + fd["lse"] + fd["a_prime"] + fd["kv_rows"]
    so_i = torch.empty_like(ap_i)
    so_w = torch.empty_like(ap_w)
    so_o = torch.empty_like(g["q"])
    so_lse = torch.empty((B, n, wl.hq), dtype=f32, device=dev)
    calls = {
        "ser_forward": ("ser_thread_kernel", ser_b,
                        lambda: gm.gm_ser_forward(g["a1_idx"], g["a1_w"], g["a2_idx"], g["a2_w"], wl.s1,
                                                  out_idx=so_i, out_w=so_w, stream=stream)),
        "sea_forward": ("sea_fwd_tile_kernel (SEA alone, edges read)", sea_b,
                        lambda: gm.gm_sea_forward(g["q"], g["k"], g["v"], ap_i, ap_w, wl.scale, o=so_o,
                                                  lse=so_lse, stream=stream)),
        "ser_forward_then_sea_forward": ("the unfused pair of the step's fused forward", ser_b + sea_b,
                                         lambda: (gm.gm_ser_forward(g["a1_idx"], g["a1_w"], g["a2_idx"],
                                                                    g["a2_w"], wl.s1, out_idx=so_i,
                                                                    out_w=so_w, stream=stream),
                                                  gm.gm_sea_forward(g["q"], g["k"], g["v"], so_i, so_w,
                                                                    wl.scale, o=so_o, lse=so_lse,
                                                                    stream=stream))),
        "leg_sparsify": ("leg_fwd_tile_kernel", e_b + mix_b + leg_b,
                         lambda: gm.gm_leg_sparsify(le["e_idx"], le["e_w"], le["mix1"], le["mix2"],
                                                    wl.s2, wl.s3, a1i, a1w, a2i, a2w, stream=stream)),
        "ser_backward": ("zero_i32_kernel + ser_bwd_thread_kernel",
                         leg_b + tok * k * wl.s1 * 4 + grad_b + tok * k * wl.s3 * 4,
                         lambda: gm.gm_ser_backward(g["a1_idx"], g["a1_w"], g["a2_idx"], g["a2_w"],
                                                    dlw, grad_is_log=True, dw1=dw1, dw2=dw2,
                                                    stream=stream)),
        "ser_sea_refresh_forward": ("sea_fwd_tile_kernel (fused SER->SEA, refresh candidates)", rf_bytes,
                                    lambda: gm.gm_ser_sea_refresh_forward(
                                        g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"], g["a2_idx"],
                                        g["a2_w"], le["e_idx"], le["e_w"], wl.s1, wl.scale,
                                        out_idx=rf_i, out_w=rf_w, o=rf_o, lse=rf_lse,
                                        stream=stream)),
        "ser_sea_chain_forward": ("sea_fwd_tile_kernel (fused 3-leg referral->SEA)", ch_bytes,
                                  lambda: gm.gm_ser_sea_chain_forward(
                                      g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"], ch_legs,
                                      wl.s2, wl.s1, wl.scale, out_idx=ch_i, out_w=ch_w, o=ch_o,
                                      lse=ch_lse, stream=stream)),
        "ser_refresh_backward": ("zero_i32_kernel + ser_bwd_thread_kernel (refresh slots)",
                                 leg_b + e_b + tok * k * wl.s1 * 4 + grad_b + tok * k * wl.s1 * 4
                                 + tok * k * wl.s3 * 4,
                                 lambda: gm.gm_ser_refresh_backward(
                                     g["a1_idx"], g["a1_w"], g["a2_idx"], g["a2_w"], le["e_idx"],
                                     le["e_w"], dlw, grad_is_log=True, dw1=rf_dw1, dw2=rf_dw2,
                                     dfw=rf_dfw, stream=stream)),
        "ser_chain_backward": ("zero_i32_kernel x2 + ser_chain_bwd_thread_kernel (3 legs)",
                               leg_b + tok * k * wl.s3 * 8 + tok * k * wl.s1 * 4
                               + tok * k * (wl.s2 + 2 * wl.s3) * 4 + 2 * tok * k * wl.s3 * 4,
                               lambda: gm.gm_ser_chain_backward(
                                   g["a1_idx"], g["a1_w"], ch_legs, wl.s2, dlw, grad_is_log=True,
                                   dw1=ch_dw1, dlegs=ch_dl, stream=stream)),
        "ser_sea_backward": ("count + scan + sea_bwd_tile_kernel with the referral backward + gather",
                             bwd_b + leg_b + grad_b + tok * k * wl.s3 * 4,
                             lambda: gm.gm_ser_sea_backward(
                                 g["q"], g["k"], g["v"], g["dout"], g["a1_idx"], g["a1_w"], g["a2_idx"],
                                 g["a2_w"], ap_i, ap_w, wl.scale, dq=f_dq, dk=f_dk, dv=f_dv, dlogw=f_dlw,
                                 dw1=f_dw1, dw2=f_dw2, workspace=f_ws, stream=stream)),
        "sea_backward_then_ser_backward": ("the unfused pair of the row above",
                                           bwd_b + leg_b + grad_b + tok * k * wl.s3 * 4,
                                           lambda: (gm.gm_sea_backward(
                                               g["q"], g["k"], g["v"], g["dout"], ap_i, ap_w, wl.scale,
                                               dq=f_dq, dk=f_dk, dv=f_dv, dlogw=f_dlw, workspace=f_ws,
                                               stream=stream),
                                               gm.gm_ser_backward(g["a1_idx"], g["a1_w"], g["a2_idx"],
                                                                  g["a2_w"], f_dlw, grad_is_log=True,
                                                                  dw1=f_dw1, dw2=f_dw2, stream=stream))),
        "leg_backward": ("leg_bwd_tile_kernel", e_b + mix_b + grad_b + tok * k * wl.s1 * 4 + mix_b,
                         lambda: gm.gm_leg_backward(le["e_idx"], le["e_w"], le["mix1"], le["mix2"],
                                                    dw1, dw2, dew=dew, dmix1=dm1, dmix2=dm2,
                                                    stream=stream)),
    }
    # refresh edges from a dense layer: the step's q/k stand in for the dense layer's, with
    # that layer's normaliser (tensor-core kernel: reported in TFLOP/s, not in the loop below)
    lse_dense = causal_lse(g["q"], g["k"], wl.scale)
    dr_i = torch.empty((B, n, k, wl.s1), dtype=torch.int32, device=dev)
    dr_w = torch.empty((B, n, k, wl.s1), dtype=f32, device=dev)
    dense = lambda: gm.gm_dense_refresh_edges(g["q"], g["k"], lse_dense, wl.s1, wl.scale,  # noqa: E731
                                              out_idx=dr_i, out_w=dr_w, stream=stream)
    out = {}
    for name, (kernel, nbytes, fn) in calls.items():
        for _ in range(3):
            fn()
        # all reps are queued before one synchronize: the flush keeps the device busy while
        # the host queues the next call, so no event brackets host-side launch latency
        evs = []
        for _ in range(reps):
            flush.sum()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            evs.append((e0, e1))
        torch.cuda.synchronize(dev)
        us = statistics.median(e0.elapsed_time(e1) * 1e3 for e0, e1 in evs)
        gbps = nbytes / (us * 1e-6) / 1e9
        out[name] = {"kernel": kernel, "us": round(us, 2), "bytes": nbytes,
                     "GBps": round(gbps, 1), "frac": round(gbps / peak, 4)}
    for _ in range(3):
        dense()
    evs = []
    for _ in range(reps):
        flush.sum()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        dense()
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize(dev)
    us = statistics.median(e0.elapsed_time(e1) * 1e3 for e0, e1 in evs)
    flops = dense_refresh_flops(wl)
    tf_peak, tf_kind = peak_bf16()
    out["dense_refresh_edges"] = {
        "kernel": "dense_refresh_kernel (tcgen05 QK^T + streaming top-sf)", "us": round(us, 2),
        "flops": flops, "TFLOPs": round(flops / (us * 1e-6) / 1e12, 1),
        "frac": round(flops / (us * 1e-6) / 1e12 / tf_peak, 4), "peak_TFLOPs": tf_peak,
        "peak_kind": tf_kind, "bound": "tensor",
        "note": "causal q.k products (2 d flops per (b, i, hq, t <= i)); sf = s1",
    }
    gm.gm_check_device_errors(stream)
    out["note"] = ("timed alone, median of %d reps, L2 flushed (256 MB read) before each; "
                   "not part of the step's value" % reps)
    return out


def timed_calls(fns, reps, stream, dev, warmup=3):
    """Run the calls `fns` (a list) warmup times, then reps times with an event around each call
    (all queued before one synchronize). Returns the mean microseconds of each call and of the
    whole sequence."""
    for _ in range(warmup):
        for f in fns:
            f()
    evs = []
    for _ in range(reps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
        e[0].record(stream)
        for f, ev in zip(fns, e[1:]):
            f()
            ev.record(stream)
        evs.append(e)
    torch.cuda.synchronize(dev)
    per = [statistics.mean(e[c].elapsed_time(e[c + 1]) * 1e3 for e in evs) for c in range(len(fns))]
    total = statistics.mean(e[0].elapsed_time(e[-1]) * 1e3 for e in evs)
    return per, total


def kv_row_bytes(idx, w, n, d, es):
    """Distinct gathered K and V rows of an edge tensor, in bytes."""
    return distinct_rows(idx, w, n) * d * es * 2


def measure_configs(gm, dev, stream, peak, reps=10):
    """The other workloads, each timed on its own (not part of the headline value).

    layer_b8_n4096_s2: the same step (fused SER->SEA forward + SEA backward) with 2 slots;
    stack21_b16_n4096_s4: 21 fused SER->SEA forwards, fresh q/k/v per layer, the edges carried
    from layer to layer (E' = SER(E, E), ping-pong buffers); long_b1_n32768_s4_train: SEA
    forward + backward on one 32768-token sequence. Bytes are compulsory, from the actual
    edges (for the stack, summed over its layers).
    """
    f32, i32 = torch.float32, torch.int32
    out = {}

    # ---- 2 slots per KV head: the step of the headline
    wl = I.WORKLOADS["layer_b8_n4096_s2"]
    x = I.make(wl, grad=True)
    g = {k: v.to(dev) for k, v in x.items()}
    B, n, hq, hkv, d = wl.B, wl.n, wl.hq, wl.hkv, wl.d
    ap_i = torch.empty((B, n, hkv, wl.s1), dtype=i32, device=dev)
    ap_w = torch.empty((B, n, hkv, wl.s1), dtype=f32, device=dev)
    o = torch.empty_like(g["q"])
    lse = torch.empty((B, n, hq), dtype=f32, device=dev)
    dq = torch.empty((B, n, hq, d), dtype=f32, device=dev)
    dk = torch.empty((B, n, hkv, d), dtype=f32, device=dev)
    dv = torch.empty_like(dk)
    dlw = torch.empty((B, n, hkv, wl.s1), dtype=f32, device=dev)
    ws = torch.empty(gm.gm_sea_backward_workspace_size(g["q"].dtype, wl.s1, B, n, hq, hkv, d),
                     dtype=torch.uint8, device=dev)
    fwd = lambda: gm.gm_ser_sea_forward(g["q"], g["k"], g["v"], g["a1_idx"], g["a1_w"],  # noqa: E731
                                        g["a2_idx"], g["a2_w"], wl.s1, wl.scale, out_idx=ap_i,
                                        out_w=ap_w, o=o, lse=lse, stream=stream)
    bwd = lambda: gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], ap_i, ap_w, wl.scale,  # noqa: E731
                                     dq=dq, dk=dk, dv=dv, dlogw=dlw, workspace=ws, stream=stream)
    (f_us, b_us), step_us = timed_calls([fwd, bwd], reps, stream, dev)
    cb = compulsory_bytes(wl, x["a1_idx"].numpy(), x["a1_w"].numpy(), ap_i.cpu().numpy(),
                          ap_w.cpu().numpy())
    out[wl.name] = {
        "step": "ser_sea_forward + sea_backward", "step_us": round(step_us, 2),
        "tokens_per_s": round(B * n / (step_us * 1e-6), 1),
        "fused_forward": {"us": round(f_us, 2), "bytes": cb["fused_forward"],
                          "frac": round(cb["fused_forward"] / (f_us * 1e-6) / 1e9 / peak, 4)},
        "backward": {"us": round(b_us, 2), "bytes": cb["backward"],
                     "frac": round(cb["backward"] / (b_us * 1e-6) / 1e9 / peak, 4)},
    }
    del g, ap_i, ap_w, o, lse, dq, dk, dv, dlw, ws

    # ---- 21-layer stack: edges carried through SER, fresh features per layer
    wl = I.WORKLOADS["stack21_b16_n4096_s4"]
    B, n, hq, hkv, d, L = wl.B, wl.n, wl.hq, wl.hkv, wl.d, wl.layers
    e0_idx, e0_w = I.edges(wl, 1, wl.s1)
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed)
    feats = [tuple(torch.randn(shape, generator=gen, device=dev).to(torch.bfloat16)
                   for shape in ((B, n, hq, d), (B, n, hkv, d), (B, n, hkv, d))) for _ in range(L)]
    e_idx = [e0_idx.to(dev), torch.empty((B, n, hkv, wl.s1), dtype=i32, device=dev)]
    e_w = [e0_w.to(dev), torch.empty((B, n, hkv, wl.s1), dtype=f32, device=dev)]
    so = torch.empty((B, n, hq, d), dtype=torch.bfloat16, device=dev)
    slse = torch.empty((B, n, hq), dtype=f32, device=dev)

    def stack(keep=None):
        cur = 0
        for layer in range(L):
            q, kk, v = feats[layer]
            nxt = 1 - cur
            gm.gm_ser_sea_forward(q, kk, v, e_idx[cur], e_w[cur], e_idx[cur], e_w[cur], wl.s1,
                                  wl.scale, out_idx=e_idx[nxt], out_w=e_w[nxt], o=so, lse=slse,
                                  stream=stream)
            if keep is not None:
                keep.append((e_idx[cur].cpu().numpy(), e_w[cur].cpu().numpy(),
                             e_idx[nxt].cpu().numpy(), e_w[nxt].cpu().numpy()))
            cur = nxt
        return cur

    def reset():
        e_idx[0].copy_(e0_idx)
        e_w[0].copy_(e0_w)

    # bytes: every layer's compulsory forward bytes from its own edges
    reset()
    layers = []
    stack(keep=layers)
    torch.cuda.synchronize(dev)
    es = 2
    total_bytes = 0
    for a_i, a_w, p_i, p_w in layers:
        tok = B * n
        total_bytes += (2 * tok * hq * d * es + tok * hq * 4 + tok * hkv * wl.s1 * 8
                        + distinct_rows(a_i, a_w, n) * wl.s1 * 8 + tok * hkv * wl.s1 * 8
                        + kv_row_bytes(p_i, p_w, n, d, es))
    times = []
    for r in range(reps // 2 + 2):
        reset()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        stack()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if r >= 2:  # two warm-up stacks
            times.append(e0.elapsed_time(e1) * 1e3)
    st_us = statistics.mean(times)
    out[wl.name] = {
        "step": f"{L} fused ser_sea_forward layers, edges carried", "stack_us": round(st_us, 1),
        "layer_us": round(st_us / L, 2), "tokens_per_s_per_layer": round(B * n / (st_us / L * 1e-6), 1),
        "bytes": total_bytes, "frac": round(total_bytes / (st_us * 1e-6) / 1e9 / peak, 4),
        "features": "N(0,1) bf16 drawn on the device per layer (torch generator, seeded)",
    }
    del feats, e_idx, e_w, so, slse

    # ---- one 32768-token sequence: SEA forward + backward
    wl = I.WORKLOADS["long_b1_n32768_s4_train"]
    x = I.make(wl, grad=True)
    g = {k: v.to(dev) for k, v in x.items()}
    B, n, hq, hkv, d = wl.B, wl.n, wl.hq, wl.hkv, wl.d
    o = torch.empty_like(g["q"])
    lse = torch.empty((B, n, hq), dtype=f32, device=dev)
    dq = torch.empty((B, n, hq, d), dtype=f32, device=dev)
    dk = torch.empty((B, n, hkv, d), dtype=f32, device=dev)
    dv = torch.empty_like(dk)
    dlw = torch.empty((B, n, hkv, wl.s1), dtype=f32, device=dev)
    ws = torch.empty(gm.gm_sea_backward_workspace_size(g["q"].dtype, wl.s1, B, n, hq, hkv, d),
                     dtype=torch.uint8, device=dev)
    fwd = lambda: gm.gm_sea_forward(g["q"], g["k"], g["v"], g["idx"], g["w"], wl.scale, o=o,  # noqa: E731
                                    lse=lse, stream=stream)
    bwd = lambda: gm.gm_sea_backward(g["q"], g["k"], g["v"], g["dout"], g["idx"], g["w"],  # noqa: E731
                                     wl.scale, dq=dq, dk=dk, dv=dv, dlogw=dlw, workspace=ws,
                                     stream=stream)
    (f_us, b_us), step_us = timed_calls([fwd, bwd], reps, stream, dev)
    tok, es = B * n, 2
    kvb = kv_row_bytes(x["idx"].numpy(), x["w"].numpy(), n, d, es)
    edges_b = tok * hkv * wl.s1 * 8
    fb = 2 * tok * hq * d * es + tok * hq * 4 + edges_b + kvb
    bb = 2 * tok * hq * d * es + edges_b + kvb + tok * hq * d * 4 + tok * hkv * wl.s1 * 4 + 2 * tok * hkv * d * 4
    out[wl.name] = {
        "step": "sea_forward + sea_backward", "step_us": round(step_us, 2),
        "tokens_per_s": round(tok / (step_us * 1e-6), 1),
        "forward": {"us": round(f_us, 2), "bytes": fb, "frac": round(fb / (f_us * 1e-6) / 1e9 / peak, 4)},
        "backward": {"us": round(b_us, 2), "bytes": bb, "frac": round(bb / (b_us * 1e-6) / 1e9 / peak, 4)},
    }
    gm.gm_check_device_errors(stream)
    out["note"] = ("each timed alone: mean of the events around each call, inputs larger than L2, "
                   "no flush; not part of the headline value")
    return out


def dense_refresh_flops(wl: I.Workload) -> int:
    """Algorithmic flops of the dense-refresh call: one d-long dot product per causal pair."""
    return wl.B * wl.hq * (wl.n * (wl.n + 1) // 2) * 2 * wl.d


def causal_lse(q, k, scale):
    """Normaliser of causal softmax attention per (b, i, hq), fp32 [B, n, hq]: set-up data for
    timing the dense-refresh call (torch TF32 matmuls, outside any timed region)."""
    B, n, hq, d = q.shape
    G = hq // k.shape[2]
    out = torch.empty((B, n, hq), dtype=torch.float32, device=q.device)
    mask = torch.ones((n, n), dtype=torch.bool, device=q.device).triu(1)
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = True
    try:
        for b in range(B):
            qb = q[b].float().permute(1, 0, 2)
            kb = k[b].float().permute(1, 0, 2).repeat_interleave(G, 0)
            sc = torch.bmm(qb, kb.transpose(1, 2)) * scale
            sc.masked_fill_(mask, float("-inf"))
            out[b] = torch.logsumexp(sc, -1).transpose(0, 1)
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    return out


def peak_bf16():
    """Dense bf16 tensor peak (TFLOP/s): the measured burst figure, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            return float(json.load(fh)["bf16_tflops"]), "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_BF16_TFLOPS, "fallback"


def e_b_refresh(wl: I.Workload) -> int:
    """Bytes of a refresh edge set [B, n, hkv, s1] (int32 index + fp32 weight per slot)."""
    return wl.B * wl.n * wl.hkv * wl.s1 * 8


def measure_e2e(gm, wl, x, dev, stream, steps, world):
    """Same step through the public API with host buffers: pinned H2D of every input, the two
    calls, D2H of every output, all inside the timed region. Steps are pipelined over three
    streams and two sets of device buffers, as a training loop would feed them: step k+1's
    inputs go host to device while step k computes and step k-1's outputs come back (PCIe
    copies in the two directions overlap; every step still moves all of its bytes)."""
    pin_in = {k: v.contiguous().pin_memory() for k, v in x.items()}
    B, n, hq, hkv, d = wl.B, wl.n, wl.hq, wl.hkv, wl.d
    f32 = torch.float32

    def buffers():
        dev_in = {k: torch.empty_like(v, device=dev) for k, v in x.items()}
        outs = {
            "ap_i": torch.empty((B, n, hkv, wl.s1), dtype=torch.int32, device=dev),
            "ap_w": torch.empty((B, n, hkv, wl.s1), dtype=f32, device=dev),
            "o": torch.empty_like(dev_in["q"]),
            "lse": torch.empty((B, n, hq), dtype=f32, device=dev),
            "dq": torch.empty((B, n, hq, d), dtype=f32, device=dev),
            "dk": torch.empty((B, n, hkv, d), dtype=f32, device=dev),
            "dv": torch.empty((B, n, hkv, d), dtype=f32, device=dev),
            "dlw": torch.empty((B, n, hkv, wl.s1), dtype=f32, device=dev),
        }
        return dev_in, outs

    sets = [buffers(), buffers()]
    outs_host = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in sets[0][1].items()}
    ws_bytes = gm.gm_sea_backward_workspace_size(sets[0][0]["q"].dtype, wl.s1, B, n, hq, hkv, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    h2d = sum(v.numel() * v.element_size() for v in pin_in.values())
    d2h = sum(v.numel() * v.element_size() for v in outs_host.values())
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    comp_done = [ev(), ev()]
    out_done = [ev(), ev()]
    for e in comp_done + out_done:
        e.record(stream)

    def one(k):
        dev_in, od = sets[k % 2]
        s_in.wait_event(comp_done[k % 2])      # step k-2 has finished reading these inputs
        with torch.cuda.stream(s_in):
            for name, v in pin_in.items():
                dev_in[name].copy_(v, non_blocking=True)
        in_done = torch.cuda.Event()
        in_done.record(s_in)
        stream.wait_event(in_done)
        stream.wait_event(out_done[k % 2])     # step k-2's outputs have left these buffers
        gm.gm_ser_sea_forward(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["a1_idx"],
                              dev_in["a1_w"], dev_in["a2_idx"], dev_in["a2_w"], wl.s1, wl.scale,
                              out_idx=od["ap_i"], out_w=od["ap_w"], o=od["o"], lse=od["lse"],
                              stream=stream)
        gm.gm_sea_backward(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["dout"], od["ap_i"],
                           od["ap_w"], wl.scale, dq=od["dq"], dk=od["dk"], dv=od["dv"],
                           dlogw=od["dlw"], workspace=ws, stream=stream)
        comp_done[k % 2].record(stream)
        s_out.wait_event(comp_done[k % 2])
        with torch.cuda.stream(s_out):
            for name, v in od.items():
                outs_host[name].copy_(v, non_blocking=True)
        out_done[k % 2].record(s_out)

    for k in range(2):
        one(k)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for e in comp_done + out_done:
        e.record(s_in)                         # every wait of the first steps starts after e0
    for k in range(steps):
        one(k)
    for e in out_done:
        stream.wait_event(e)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    return {"value": round(B * n * world * steps / (ms / 1e3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": ms / steps, "pipelined": "3 streams, 2 buffer sets"}


# ---- reference arm: the CPU oracle --------------------------------------------------------------

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    wl = I.WORKLOADS[args.workload]
    sample = wl.with_(B=1)
    x = I.make(sample, grad=True)
    x = {k: (v.float().numpy() if v.dtype == torch.bfloat16 else v.numpy()) for k, v in x.items()}
    for _ in range(max(args.warmup, 0)):
        oracle_sample_step(sample, x)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(sample, x)
    el = time.perf_counter() - t0
    value = sample.n * args.steps / el
    cores = oracle.num_threads()
    return {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": wl.name, "B_per_gpu": wl.B, "n": wl.n, "hq": wl.hq,
                   "hkv": wl.hkv, "d": wl.d, "s1": wl.s1, "s2": wl.s2, "s3": wl.s3,
                   "step": "ser_sea_forward + sea_backward", "global_batch": wl.B,
                   "seq_len": wl.n, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"each step: 1 of {wl.B} sequences ({sample.n} tokens, same "
                                   "recipe), SER + SEA fwd + SEA bwd in the C oracle"},
        "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    if args.write_traffic:
        if not args.traffic_batch:
            raise SystemExit("--write-traffic needs --traffic-batch")
        print(write_traffic_table(args.write_traffic, args.workload, args.traffic_batch, args.traffic_command))
        return
    if args.impl == "reference":
        res = run_reference(args)
    else:
        res = run_ours(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
