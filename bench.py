#!/usr/bin/env python
"""Benchmark of the per-frame hot path: page-aligned append + frame attention over the
paged cache + commit / sliding-window eviction, on the 518x378 streaming workload
(1004 tokens/frame, 16 heads x 64, W=64 + S=8 frames, page 16, bf16).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one steady-state frame (the cache holds S + W frames; attention spans
S + W + 1 = 73 frames = 73,292 tokens). The cache is filled first, then W warm-up frames
run, then exactly K frames are timed with CUDA events on the cache's stream between a
barrier + synchronize on both sides; N > 1 (torchrun) runs one independent stream per
rank (weak scaling, no collective on the data path) and reports the max time over ranks.
Rank 0 prints one JSON line.

`--impl reference` times the fp64 CPU oracle on the host cores instead (each step a
bounded sample of the same workload, extrapolated to a whole frame).
"""
from __future__ import annotations

import argparse
import contextlib
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time
from datetime import timedelta

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "frames/s of per-frame KV-cache attention+update; % of TC / HBM peak"
UNIT = "frames/s"
WORKLOAD = "vggt_518x378"
PROFILE_ATTN = os.path.join(ROOT, "profiles", "attn_tc_kernel_vggt_518x378.md")
ATTN_SRC = os.path.join(ROOT, "transformer_kv_cache_b200", "csrc", "kvc_attn_tc.cu")
# B200 spec-sheet dense bf16 tensor rate (TFLOP/s), reported beside the measured peak
SPEC_DENSE_BF16_TFLOPS = 2250.0


def log(msg: str):
    """Progress on stderr (the result line goes to stdout)."""
    sys.stderr.write(f"[bench {time.strftime('%H:%M:%S')}] {msg}\n")
    sys.stderr.flush()


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=64)
    ap.add_argument("--append-all-steps", type=int, default=8,
                    help="timed calls of the 24-layer one-launch append leg (0: skip it)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kv-splits", type=int, default=0)
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="replicas (default): one independent stream per rank; heads: one stream, "
                         "heads sharded over the ranks, O all-gathered")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="vggt_518x378 (default, the headline), vggt_24layer_k4, vggt_budget_16k, vggt_518x518_fp8, "
                         "vggt_infinite_12l, vggt_518x378_joint, vggt_518x378_special")
    ap.add_argument("--fill", type=int, default=0,
                    help="frames streamed before warm-up for a non-default workload (0: enough to fill the window); "
                         "smaller values give short cases for profiling")
    return ap.parse_args()


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


def _peak_number(d, key):
    """The positive number stored under `key` in the peaks file: at the top level, as
    {"value": x} there, or one level down in a section; None when absent."""
    def num(v):
        if isinstance(v, dict):
            v = v.get("value")
        if isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0:
            return float(v)
        return None
    if not isinstance(d, dict):
        return None
    if num(d.get(key)) is not None:
        return num(d.get(key))
    for sec in d.values():
        if isinstance(sec, dict) and num(sec.get(key)) is not None:
            return num(sec.get(key))
    return None


def load_peaks(path=None):
    """Roofline denominators: the measured copy bandwidth and bf16 GEMM rates when the
    peaks file holds them, else the fallback figures. Returns (peaks, "measured" |
    "fallback"); a file that cannot be read or lacks the HBM or bf16 figure counts as
    absent, and a missing sustained figure alone takes its fallback."""
    p = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p)) if os.path.exists(p) else None
    except (OSError, ValueError):
        d = None
    got = {k: _peak_number(d, k) for k in FALLBACK_PEAKS}
    if got["hbm_gbs"] is None or got["bf16_tflops"] is None:
        return dict(FALLBACK_PEAKS), "fallback"
    return {k: (v if v is not None else FALLBACK_PEAKS[k]) for k, v in got.items()}, "measured"


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ oracle sample (CPU)

def oracle_sample(wl, frames: int, rows: int, seed: int = 0, time_budget_s: float = 1e9):
    """Time the fp64 oracle on `frames` steady-state frames of one head of the workload,
    attention for `rows` query rows; extrapolate each to a whole frame (all heads, all
    rows): 16 x (append + commit/evict + gather + T x per-row attention)."""
    import numpy as np
    from kvc_streams import FrameStream
    from oracle import OracleConfig, StreamOracle
    H = wl.num_heads
    w1 = wl.replace(num_heads=1)
    st = FrameStream(w1, seed=seed)
    orc = StreamOracle(OracleConfig.from_workload(w1))
    fill = w1.scale_frames + w1.window_frames
    for t in range(fill):
        q, k, v = st.frame(0, t)
        orc.append(0, t, k.double().numpy(), v.double().numpy(), True)
        orc.commit(0)
    per_frame = []
    t_start = time.perf_counter()
    rr = list(range(0, w1.tokens_per_frame, max(1, w1.tokens_per_frame // rows)))[:rows]
    for i in range(frames):
        t = fill + i
        q, k, v = st.frame(0, t)
        qn, kn, vn = q.double().numpy(), k.double().numpy(), v.double().numpy()
        a0 = time.perf_counter()
        orc.append(0, t, kn, vn, True)
        a1 = time.perf_counter()
        orc.gather(0)
        a2 = time.perf_counter()
        orc.attend(0, qn, rows=rr, commit=False)
        a3 = time.perf_counter()
        orc.commit(0)
        a4 = time.perf_counter()
        t_gather = a2 - a1
        per_row = max(a3 - a2 - t_gather, 0.0) / len(rr)
        frame_s = H * ((a1 - a0) + (a4 - a3) + t_gather + w1.tokens_per_frame * per_row)
        per_frame.append(frame_s)
        if time.perf_counter() - t_start > time_budget_s:
            break
    return per_frame, len(rr), time.perf_counter() - t_start


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from kvc_streams import WORKLOADS
    wl = WORKLOADS[WORKLOAD]
    steps, warm = args.steps, args.warmup
    # bound the whole run to a few minutes: about 0.15 s of fixed work per sampled frame
    # (append, gather, commit of one head) plus ~6 ms per sampled query row
    budget_per_step = 150.0 / max(1, steps + warm)
    rows = int(max(1, min(16, (budget_per_step - 0.15) / 0.006)))
    # torchrun sets OMP_NUM_THREADS=1 in every rank; here rank 0 is the only one at work,
    # so the oracle gets the host's cores as it does in a plain single-process run
    ctx = contextlib.nullcontext()
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        try:
            from threadpoolctl import threadpool_limits
            ctx = threadpool_limits(limits=len(os.sched_getaffinity(0)))
        except Exception:
            pass
    with ctx:
        per_frame, r, wall = oracle_sample(wl, steps + warm, rows)
        cores = blas_threads()
    timed = per_frame[warm:] if len(per_frame) > warm else per_frame
    mean_s = statistics.mean(timed)
    value = 1.0 / mean_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": len(timed), "warmup": warm, "ms_per_step": mean_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens_per_frame": wl.tokens_per_frame, "heads": wl.num_heads,
                   "head_dim": wl.head_dim, "window_frames": wl.window_frames, "scale_frames": wl.scale_frames,
                   "page_size": wl.page_size, "kv_tokens_attended": (wl.scale_frames + wl.window_frames + 1) *
                   wl.tokens_per_frame},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"fp64 oracle, 1 of {wl.num_heads} heads, {r} of {wl.tokens_per_frame} query rows "
                                   f"per steady-state frame, extrapolated x{wl.num_heads} heads and per-row to all rows; "
                                   f"{len(per_frame)} frames, {wall:.1f} s of CPU work"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ clocks during the timed region

def sync_polling(stream) -> None:
    """Wait for the stream by polling an event with short sleeps, so the clock sampler's
    thread keeps running while the GPU works (a blocking synchronize can hold the
    interpreter for the whole wait)."""
    import torch
    done = torch.cuda.Event()
    done.record(stream)
    while not done.query():
        time.sleep(0.0002)
    stream.synchronize()


class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self.stop_ev = threading.Event()
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            # NVML enumerates every GPU of the host; find ours by UUID
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self.stop_ev.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = get_r(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.th = threading.Thread(target=self._run, daemon=True)
            self.th.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop_ev.set()
            self.th.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0,
                    "source": "unavailable"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


def profile_traffic():
    """Per-launch DRAM bytes of the attention kernel from the committed ncu summary, only
    while the kernel source is the one that was profiled."""
    if not os.path.exists(PROFILE_ATTN):
        return None
    txt = open(PROFILE_ATTN).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    h = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    if not m or not h:
        return None
    cur = hashlib.sha256(open(ATTN_SRC, "rb").read()).hexdigest()
    return float(m.group(1)) if h.group(1) == cur else None


# ------------------------------------------------------------------ ranks
# N > 1: one process per GPU, each running its own independent stream (replicas, weak
# scaling). The only collectives are the barriers around the timed region and the
# max-over-ranks of the device times; none is on the data path.

def rank_seed(rank: int) -> int:
    """Seed of a rank's synthetic stream: every rank streams different frames."""
    return 1000 + rank


def max_over_ranks(value_ms: float, world: int, device) -> float:
    """The largest of the ranks' device times (all ranks must call it)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, units_per_rank: int, max_ms: float) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / (max_ms / 1e3)


def head_range(rank: int, world: int, H: int):
    """Heads [h0, h1) of a rank when one stream's step is sharded by head (attention and
    cache are independent per head, so each rank holds its heads' pages)."""
    if H % world:
        raise ValueError(f"{world} ranks do not divide {H} heads")
    n = H // world
    return rank * n, (rank + 1) * n


def gather_heads(o_local, world: int):
    """Every rank's O slice [T, H/N, D] gathered into the full [T, H, D] on every rank,
    heads in rank order: the one exchange of a head-sharded step (NCCL on GPUs, any
    torch.distributed backend)."""
    import torch
    import torch.distributed as dist
    if world == 1:
        return o_local
    parts = [torch.empty_like(o_local) for _ in range(world)]
    dist.all_gather(parts, o_local.contiguous())
    return torch.cat(parts, dim=1)


# ------------------------------------------------------------------ our CUDA path

def run_ours(args):
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    import transformer_kv_cache_b200 as kvc
    from kvc_streams import WORKLOADS, FrameStream

    wl = WORKLOADS[WORKLOAD]
    T, H, D, P = wl.tokens_per_frame, wl.num_heads, wl.head_dim, wl.page_size
    S, W = wl.scale_frames, wl.window_frames
    fill, warm, steps = S + W, args.warmup, args.steps
    n_frames = fill + warm + steps + 3              # + the end-to-end leg's 3 warm-up steps
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)
    peaks, peak_kind = load_peaks()

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    log(f"rank {rank}/{world}: generating {n_frames} frames")
    with torch.cuda.stream(stream):
        st = FrameStream(wl, seed=rank_seed(rank), device=dev)
        frames = [st.frame(0, t) for t in range(n_frames)]
        torch.cuda.synchronize()
        log("frames ready; filling the cache")
        out = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
        h = kvc.kvc_create(kvc.config_from_workload(wl, kv_splits=args.kv_splits), stream)
        for t in range(fill + warm):
            q, k, v = frames[t]
            kvc.kvc_append_frame(h, 0, t, k, v, True)
            kvc.kvc_attend(h, 0, q, out)
        _, info0 = kvc.kvc_page_table(h, 0)
        log(f"cache filled ({info0['pages_used']} pages); timing {steps} steps")
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        with ClockSampler(local) as clk:
            e0.record(stream)
            for i in range(steps):
                t = fill + warm + i
                q, k, v = frames[t]
                ev[i][0].record(stream)
                kvc.kvc_append_frame(h, 0, t, k, v, True)
                ev[i][1].record(stream)
                kvc.kvc_attend(h, 0, q, out)
                ev[i][2].record(stream)
            e1.record(stream)
            sync_polling(stream)
        barrier()
        elapsed_ms = e0.elapsed_time(e1)
        log(f"timed region {elapsed_ms:.2f} ms")
        _, info1 = kvc.kvc_page_table(h, 0)
        append_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(steps))
        attend_ms = statistics.mean(ev[i][1].elapsed_time(ev[i][2]) for i in range(steps))
        launches = info1["kernel_launches"] - info0["kernel_launches"]
        assert info1["device_error"] == 0

    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)

    # every layer of the 24-layer keyframe workload appended in one call (one launch:
    # allocation and copy fused); sources are distinct per layer and rotate over 4 sets of
    # 24 frames (400 MB, more than L2); only the append call is inside the events, the
    # attention that commits each frame runs between them
    app_all = None
    if args.append_all_steps > 0:
        log("all-layer append leg")
        wl24 = WORKLOADS["vggt_24layer_k4"]
        L24 = wl24.num_layers
        with torch.cuda.stream(stream):
            st24 = FrameStream(wl24, seed=rank_seed(rank) + 77, device=dev)
            sets = [[st24.frame(l, u) for l in range(L24)] for u in range(4)]
            h24 = kvc.kvc_create(kvc.config_from_workload(wl24), stream)
            ev24 = []
            for t in range(3 + args.append_all_steps):
                fr = sets[t % 4]
                a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a0.record(stream)
                kvc.kvc_append_frame_all(h24, t, [x[1] for x in fr], [x[2] for x in fr], True)
                a1.record(stream)
                for l in range(L24):
                    kvc.kvc_attend(h24, l, fr[l][0], out)
                if t >= 3:
                    ev24.append((a0, a1))
            stream.synchronize()
            _, info24 = kvc.kvc_page_table(h24, 0)
            assert info24["device_error"] == 0
            kvc.kvc_destroy(h24)
            del sets
        a_ms = statistics.mean(a.elapsed_time(b) for a, b in ev24)
        a_bytes = L24 * 2 * 2 * T * H * D * 2
        app_all = {"bound": "hbm", "bytes_per_launch": a_bytes, "avg_launch_ms": a_ms,
                   "achieved_gbs": a_bytes / (a_ms * 1e-3) / 1e9, "peak_gbs": float(peaks["hbm_gbs"]),
                   "frac": a_bytes / (a_ms * 1e-3) / 1e9 / float(peaks["hbm_gbs"]),
                   "launches_per_call": 1, "layers": L24, "steps": len(ev24),
                   "note": "kvc_append_frame_all on the 24-layer keyframe workload: page allocation and copy of "
                           "every layer in one launch; inputs rotate over 4 x 24 frames (larger than L2)"}

    # end to end through the public API from pinned host buffers
    e2e = None
    if args.e2e_steps > 0:
        log("end-to-end leg")
        kvc.kvc_reset(h)
        n_e2e = min(args.e2e_steps, steps)
        e2e_warm = 3
        with torch.cuda.stream(stream):
            for t in range(fill):
                q, k, v = frames[t]
                kvc.kvc_append_frame(h, 0, t, k, v, True)
                kvc.kvc_attend(h, 0, q, out)
            host = [tuple(x.cpu().pin_memory() for x in frames[fill + i]) for i in range(e2e_warm + n_e2e)]
            oh = torch.empty((T, H, D), dtype=torch.bfloat16).pin_memory()
            # untimed warm-up: every pinned buffer crosses the bus once (its first transfer is
            # slower), and e2e_warm host-buffer steps run before the timed ones
            scratch = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
            for x in host:
                for y in x:
                    scratch.copy_(y, non_blocking=True)
            oh.copy_(scratch, non_blocking=True)
            for i in range(e2e_warm):
                qh, kh, vh = host[i]
                kvc.kvc_step_host_async(h, 0, fill + i, True, qh, kh, vh, oh)
            kvc.kvc_synchronize(h)
            stream.synchronize()
            host = host[e2e_warm:]
            fill += e2e_warm
            barrier()
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            # every step uploads its inputs and downloads its output; the library overlaps
            # one step's copies with its neighbours' compute; the end event follows the
            # host wait for the last download
            for i in range(n_e2e):
                qh, kh, vh = host[i]
                kvc.kvc_step_host_async(h, 0, fill + i, True, qh, kh, vh, oh)
            kvc.kvc_synchronize(h)
            f1.record(stream)
            stream.synchronize()
            barrier()
        e_ms = max_over_ranks(f0.elapsed_time(f1), world, dev)
        fb = T * H * D * 2
        e2e = {"value": job_rate(world, n_e2e, e_ms), "unit": UNIT, "h2d_bytes_per_step": 3 * fb,
               "d2h_bytes_per_step": fb, "steps": n_e2e, "warmup": e2e_warm,
               "api": "kvc_step_host_async + kvc_synchronize"}
    kvc.kvc_destroy(h)

    if rank == 0:
        n_kv = (S + W + 1) * T
        flops = 4.0 * T * n_kv * H * D
        achieved = flops / (attend_ms * 1e-3) / 1e12
        peak = float(peaks["bf16_tflops"])
        app_bytes = 2 * 2 * T * H * D * 2           # read K,V + write K,V (valid tokens)
        app_gbs = app_bytes / (append_ms * 1e-3) / 1e9
        value = job_rate(world, steps, elapsed_ms)
        clocks = clk.summary()
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps, "warmup": warm,
            "ms_per_step": elapsed_ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens_per_frame": T, "heads": H, "head_dim": D, "page_size": P,
                       "window_frames": W, "scale_frames": S, "kv_tokens_attended": n_kv,
                       "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": "inputs larger than L2: the layer cache is 294 MB of pages, read every step",
                       "frames_per_rank": n_frames},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": profile_traffic(),
                         "frac_of_spec_sheet": achieved / SPEC_DENSE_BF16_TFLOPS,
                         "kernel": "attention (attn_tc_kernel, pieces merged in the kernel, + commit/evict, per kvc_attend)",
                         "flops_per_launch": flops, "avg_launch_ms": attend_ms,
                         "peak_source": f"{peak_kind} bf16 dense burst"},
            "kernels": {"append": {"bound": "hbm", "bytes_per_launch": app_bytes, "avg_launch_ms": append_ms,
                                   "achieved_gbs": app_gbs, "peak_gbs": float(peaks["hbm_gbs"]),
                                   "frac": app_gbs / float(peaks["hbm_gbs"]),
                                   "note": "one layer's frame (8.2 MB), page allocation fused into the one "
                                           "launch; bound by launch latency at this size"}},
            "gpu_launches": int(launches),
            "clocks": clocks,
        }
        if app_all:
            line["kernels"]["append_all_layers"] = app_all
        if e2e:
            line["e2e"] = e2e
        if world == 1 and not args.no_cpu_baseline:
            log("cpu baseline (oracle sample)")
            per_frame, r, wall = oracle_sample(wl, 24, 16, time_budget_s=25.0)
            v = 1.0 / statistics.mean(per_frame)
            line["cpu_baseline"] = {
                "value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                "sample": f"fp64 oracle, 1 of {H} heads, {r} of {T} query rows on {len(per_frame)} steady-state "
                          f"frames ({wall:.1f} s), extrapolated x{H} heads and per-row to all rows"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_workload(args):
    """One JSON line for a non-default workload: a step is one frame through every layer
    (batched append of all layers, attention per layer, and scoring/compression per layer in
    budget mode, or pruning per layer with the rolling memory). All K steps' inputs are
    resident in HBM: a few seeded frames per layer cycle, except with the rolling memory,
    whose pruning depends on the key values and so gets a distinct frame every step."""
    import torch
    import transformer_kv_cache_b200 as kvc
    from kvc_streams import WORKLOADS, FrameStream, keyframe_schedule

    wl = WORKLOADS[args.workload]
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)
    peaks, peak_kind = load_peaks()
    L, T, H, D, P = wl.num_layers, wl.tokens_per_frame, wl.num_heads, wl.head_dim, wl.page_size
    S, W, k = wl.scale_frames, wl.window_frames, wl.keyframe_interval
    budget = wl.budget_tokens > 0
    rolling = wl.diversity_budget > 0
    if args.fill > 0:
        fill = args.fill
    elif rolling:
        fill = 3                                      # anchor, then two prunings: the kept sets are full
    elif budget:
        fill = -(-wl.budget_tokens // T) + 3          # past the first compression of every layer
    elif wl.special_frames > 0:                       # the window is full and 128 frames have
        fill = S + W * k + min(wl.special_frames, 128)   # left it, keeping their special tokens
    else:
        fill = S + W * k                              # the window is full of keyframes
    warm, steps = args.warmup, args.steps
    # the rolling memory's pruning depends on the key values: every frame distinct, as in a
    # video (a repeated frame would duplicate every key of the kept set); elsewhere data
    # values do not change the work and a few frames cycle
    distinct = fill + warm + steps if rolling else 4
    log(f"{wl.name}: {L} layers, fill {fill} frames, {distinct} distinct input frames per layer")
    with torch.cuda.stream(stream):
        st = FrameStream(wl, seed=2000, device=dev)
        pool = [[st.frame(l, t) for t in range(distinct)] for l in range(L)]
        res = [[st.residual(l, t) for t in range(distinct)] for l in range(L)] if budget else None
        outs = [torch.empty((T, H, D), dtype=torch.bfloat16, device=dev) for _ in range(L)]
        h = kvc.kvc_create(kvc.config_from_workload(wl, kv_splits=args.kv_splits), stream)

        def step(t, ev=None):
            key = True if rolling else keyframe_schedule(t, S, k)
            i = t % distinct
            if ev: ev[0].record(stream)
            kvc.kvc_append_frame_all(h, t, [pool[l][i][1] for l in range(L)], [pool[l][i][2] for l in range(L)], key)
            if ev: ev[1].record(stream)
            fired = 0
            if rolling:                               # prune every layer, then attend every layer
                if t > 0:
                    kvc.kvc_prune_all(h)
                    fired = L
                if ev: ev[2].record(stream)
                kvc.kvc_attend_all(h, [pool[l][i][0] for l in range(L)], outs)
                if ev: ev[3].record(stream)
                return key, fired
            kvc.kvc_attend_all(h, [pool[l][i][0] for l in range(L)], outs)
            if ev: ev[2].record(stream)
            if budget:
                fired += sum(kvc.kvc_compress_all(h, [res[l][i] for l in range(L)]))
            if ev: ev[3].record(stream)
            return key, fired

        for t in range(fill + warm):
            step(t)
        _, info0 = kvc.kvc_page_table(h, 0)
        torch.cuda.synchronize()
        log(f"filled: layer 0 holds {info0['pages_used']} pages, {info0['tokens']} tokens; timing {steps} steps")
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        keys, fires, n_kv = 0, 0, []
        with ClockSampler(local) as clk:
            for i in range(steps):
                t = fill + warm + i
                _, before = (None, None)
                key, fired = step(t, evs[i])
                keys += key
                fires += fired
            sync_polling(stream)
        _, info1 = kvc.kvc_page_table(h, 0)
        assert info1["device_error"] == 0
        kvc.kvc_destroy(h)
    tot = [evs[i][0].elapsed_time(evs[i][3]) for i in range(steps)]
    app = [evs[i][0].elapsed_time(evs[i][1]) for i in range(steps)]
    att = [evs[i][1].elapsed_time(evs[i][2]) for i in range(steps)]
    cmp_ = [evs[i][2].elapsed_time(evs[i][3]) for i in range(steps)]
    if rolling:                                       # the prune comes before the attention
        att, cmp_ = cmp_, att
    ms = statistics.mean(tot)
    line = {"metric": METRIC, "value": 1e3 / ms, "unit": UNIT, "n_gpus": 1, "steps": steps, "warmup": warm,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8_e4m3 storage, bf16 I/O" if wl.kv_dtype == "fp8_e4m3" else "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "layers": L, "tokens_per_frame": T, "heads": H, "head_dim": D,
                       "page_size": P, "window_frames": W, "scale_frames": S, "keyframe_interval": k,
                       "budget_tokens": wl.budget_tokens, "diversity_budget": wl.diversity_budget,
                       "special_frames": wl.special_frames, "kv_tokens_attended": info0["tokens"] + T,
                       "inputs": (f"{distinct} distinct seeded frames per layer" if rolling else
                                  f"{distinct} seeded frames per layer, cycled"),
                       "keyframes_timed": keys, "compressions_timed": fires},
            "clocks": clk.summary()}
    # per layer: read K and V in bf16, write them as stored (bf16, or E4M3 codes + scales)
    kv_elem = 1 if wl.kv_dtype == "fp8_e4m3" else 2
    app_bytes = 2 * T * H * D * (2 + kv_elem) * L
    att_ms = statistics.mean(att)
    line["kernels"] = {
        "append_all_layers": {"bound": "hbm", "avg_ms": statistics.mean(app), "bytes_per_launch": app_bytes,
                              "achieved_gbs": app_bytes / (statistics.mean(app) * 1e-3) / 1e9,
                              "peak_gbs": float(peaks["hbm_gbs"])},
        "attention_all_layers": {"avg_ms": att_ms}}
    if rolling:
        kv_tokens = T + min(wl.diversity_budget, 2 * T)   # per head: the anchor and the kept tokens
    if not budget:
        if not rolling:
            kv_tokens = info0["tokens"] + T           # the cache before the timed steps, plus the new frame
        flops = 4.0 * T * kv_tokens * H * D * L
        ach = flops / (att_ms * 1e-3) / 1e12
        line["roofline"] = {"bound": "tensor", "achieved": ach, "peak": float(peaks["bf16_tflops"]), "unit": "TFLOP/s",
                            "frac": ach / float(peaks["bf16_tflops"]), "traffic": None,
                            "frac_of_spec_sheet": ach / SPEC_DENSE_BF16_TFLOPS,
                            "kernel": "attention over all layers per frame", "flops_per_launch": flops / L}
    if budget:
        line["kernels"]["score_and_compress_all_layers"] = {"avg_ms": statistics.mean(cmp_),
                                                            "max_ms": max(cmp_)}
    if rolling:
        # per layer and head: read the candidates' keys, move the kept tokens' K and V
        n_cand = min(wl.diversity_budget, 2 * T) + T
        prune_bytes = H * L * (n_cand * D * 2 + 4 * min(wl.diversity_budget, n_cand) * D * 2)
        pm = statistics.mean(cmp_)
        line["kernels"]["prune_all_layers"] = {"bound": "hbm", "avg_ms": pm, "max_ms": max(cmp_),
                                               "bytes_per_step": prune_bytes,
                                               "achieved_gbs": prune_bytes / (pm * 1e-3) / 1e9,
                                               "candidates_per_head": n_cand}
    line["kernels"]["append_all_layers"]["frac"] = (line["kernels"]["append_all_layers"]["achieved_gbs"] /
                                                    float(peaks["hbm_gbs"]))
    print(json.dumps(line), flush=True)
    return 0


def run_joint(args):
    """The joint scale-frame phase: a step is kvc_reset (a new stream) followed by
    kvc_scale_phase of the stream's first joint_frames frames on every layer; the metric
    counts those frames. Inputs are resident in HBM."""
    import torch
    import transformer_kv_cache_b200 as kvc
    from kvc_streams import WORKLOADS, FrameStream

    wl = WORKLOADS[args.workload]
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)
    peaks, peak_kind = load_peaks()
    L, T, H, D, n = wl.num_layers, wl.tokens_per_frame, wl.num_heads, wl.head_dim, wl.joint_frames
    warm, steps = args.warmup, args.steps
    with torch.cuda.stream(stream):
        st = FrameStream(wl, seed=2000, device=dev)
        qkv = []
        for l in range(L):
            fr = [st.frame(l, t) for t in range(n)]
            qkv.append(tuple(torch.cat([x[i] for x in fr]) for i in range(3)))
        out = torch.empty((n * T, H, D), dtype=torch.bfloat16, device=dev)
        h = kvc.kvc_create(kvc.config_from_workload(wl, kv_splits=args.kv_splits), stream)

        def step(ev=None):
            if ev: ev[0].record(stream)
            kvc.kvc_reset(h)
            if ev: ev[1].record(stream)
            for l in range(L):
                kvc.kvc_scale_phase(h, l, n, qkv[l][0], qkv[l][1], qkv[l][2], out)
            if ev: ev[2].record(stream)

        for _ in range(warm):
            step()
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        with ClockSampler(local) as clk:
            for i in range(steps):
                step(evs[i])
            sync_polling(stream)
        _, info = kvc.kvc_page_table(h, 0)
        assert info["device_error"] == 0
        kvc.kvc_destroy(h)
    tot = statistics.mean(evs[i][0].elapsed_time(evs[i][2]) for i in range(steps))
    ph = statistics.mean(evs[i][1].elapsed_time(evs[i][2]) for i in range(steps))
    flops = 4.0 * (n * T) ** 2 * H * D * L
    ach = flops / (ph * 1e-3) / 1e12
    line = {"metric": METRIC, "value": n * 1e3 / tot, "unit": UNIT, "n_gpus": 1, "steps": steps, "warmup": warm,
            "ms_per_step": tot, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": wl.name, "layers": L, "tokens_per_frame": T, "heads": H, "head_dim": D,
                       "joint_frames": n, "queries": n * T, "keys": n * T,
                       "step": "kvc_reset, then the joint phase of every layer"},
            "clocks": clk.summary(),
            "kernels": {"reset_ms": tot - ph, "joint_phase_ms": ph},
            "roofline": {"bound": "tensor", "achieved": ach, "peak": float(peaks["bf16_tflops"]), "unit": "TFLOP/s",
                         "frac": ach / float(peaks["bf16_tflops"]), "traffic": None,
                         "frac_of_spec_sheet": ach / SPEC_DENSE_BF16_TFLOPS,
                         "kernel": "attention of the joint phase (append of the frames included)",
                         "flops_per_launch": flops / L, "peak_source": peak_kind}}
    print(json.dumps(line), flush=True)
    return 0


def run_sharded(args):
    """One 518x378 stream with its step sharded by head over the ranks: every rank holds the
    full-width Q, K and V; its cache holds heads [h0, h1) of them (the library's head
    range), appends and attends that slice and writes it into its O; the slices are then
    all-gathered. Total work per step is fixed (strong scaling); the value is the stream's
    frames/s."""
    import torch
    import torch.distributed as dist
    import transformer_kv_cache_b200 as kvc
    from kvc_streams import WORKLOADS, FrameStream, keyframe_schedule

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    wl = WORKLOADS[WORKLOAD]
    T, H, D, S, W = wl.tokens_per_frame, wl.num_heads, wl.head_dim, wl.scale_frames, wl.window_frames
    h0, h1 = head_range(rank, world, H)
    stream = torch.cuda.Stream(device=dev)
    distinct = 4
    with torch.cuda.stream(stream):
        st = FrameStream(wl, seed=rank_seed(0), device=dev)            # one stream, the same on every rank
        frames = [st.frame(0, t) for t in range(distinct)]
        out = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
        cfg = kvc.config_from_workload(wl.replace(num_heads=h1 - h0), kv_splits=args.kv_splits,
                                       model_heads=H if world > 1 else 0, head_begin=h0)
        h = kvc.kvc_create(cfg, stream)

        def step(t):
            q, k, v = frames[t % distinct]
            key = keyframe_schedule(t, S, wl.keyframe_interval)
            kvc.kvc_append_frame(h, 0, t, k, v, key)
            kvc.kvc_attend(h, 0, q, out)
            return gather_heads(out[:, h0:h1].contiguous() if world > 1 else out, world)

        fill = S + W
        for t in range(fill + args.warmup):
            step(t)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            full = step(fill + args.warmup + i)
        e1.record(stream)
        stream.synchronize()
        _, info = kvc.kvc_page_table(h, 0)
        assert info["device_error"] == 0 and full.shape == (T, H, D)
        kvc.kvc_destroy(h)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    if rank == 0:
        line = {"metric": METRIC, "value": 1e3 / ms, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": wl.name, "tokens_per_frame": T, "heads": H, "heads_per_rank": h1 - h0,
                           "head_dim": D, "window_frames": W, "scale_frames": S, "parallelism": f"heads{world}",
                           "exchange": "all-gather of O per step (NCCL)"}}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if os.environ.get("KVC_BENCH_WATCHDOG"):
        import faulthandler
        faulthandler.dump_traceback_later(float(os.environ["KVC_BENCH_WATCHDOG"]), exit=False)
    if args.impl == "reference":
        return run_reference(args)
    if args.shard == "heads":
        return run_sharded(args)
    if args.workload != WORKLOAD:
        from kvc_streams import WORKLOADS
        if WORKLOADS[args.workload].joint_frames > 0:
            return run_joint(args)
        return run_workload(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
