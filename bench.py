#!/usr/bin/env python3
"""Benchmark of the MoE SwiGLU FFN layer on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mixtral] [--n-c -1]
    python bench.py --impl reference ...      # the CPU oracle on the host cores

A step is one pass of the whole layer (plan -> dispatch -> GEMM1+SwiGLU -> GEMM2
+gate-weighted scatter -> combine) over one batch of M tokens, through the
public call moe_ffn_fused.  Inputs are seeded and synthetic (grouped_gemm_plan_b200
.workload); weights are resident in HBM.  L2 is flushed (a 256 MiB write)
before every timed step, outside the timed events.  With N GPUs every rank runs
its own batch (its own seed): tokens are independent, so the layer shards with
no collective on the data path (weak scaling); the only collectives are the
barrier and the max-over-ranks of the timings.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import shutil
import signal
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

MEASURED_PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "MoE-layer tokens/s"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="mixtral")
    ap.add_argument("--n-c", type=int, default=-1, dest="n_c")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--n-c-sweep", default=None, dest="n_c_sweep",
                    help="comma-separated n_c values: print one timing line per value "
                         "(profiling for the n_c table) instead of the benchmark line")
    return ap.parse_args(argv)


def peaks():
    try:
        with open(MEASURED_PEAKS) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and throttle reasons sampled while the timed region runs.

    Reads NVML from a background thread every 5 ms (read-only queries; nothing is
    set), so a timed region of tens of milliseconds still gets a dozen samples.
    Falls back to `nvidia-smi -lms 200` when NVML is not importable.
    """
    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.index = index
        self.period = period_s
        self.samples: list[tuple[float, float, int, float]] = []  # (t, mhz, reason bits, watts)
        self.window = (0.0, float("inf"))
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        self._proc = None
        self._lines: list[str] = []

    def mark(self, t0: float, t1: float):
        """Keep only samples taken between host times t0 and t1 (time.monotonic())."""
        self.window = (t0, t1)

    def start(self):
        sys.setswitchinterval(0.0005)   # let the polling thread run between launches
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._poll_nvml, args=(h,), daemon=True)
            self._thread.start()
            return
        except Exception:
            self._nvml = None
        try:
            cmd = ["nvidia-smi", f"--id={self.index}", "--query-gpu=clocks.sm,clocks.max.sm",
                   "--format=csv,noheader,nounits", "-lms", "200"]
            if shutil.which("stdbuf"):
                cmd = ["stdbuf", "-oL"] + cmd
            self._proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                          text=True, bufsize=1)
            self._thread = threading.Thread(target=self._read_smi, daemon=True)
            self._thread.start()
        except OSError:
            self._proc = None

    def _poll_nvml(self, h):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                t = time.monotonic()
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                watts = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.samples.append((t, float(mhz), int(bits), watts))
            except Exception:
                pass
            self._stop.wait(self.period)

    def _read_smi(self):
        for line in self._proc.stdout:
            self._lines.append(line.strip())

    def stop(self) -> dict:
        self._stop.set()
        if self._proc is not None:
            time.sleep(0.3)
            self._proc.send_signal(signal.SIGINT)
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._thread is not None:
            self._thread.join(timeout=5)
        sys.setswitchinterval(0.005)
        reasons = set()
        if self._nvml is not None:
            t0, t1 = self.window
            inside = [x for x in self.samples if t0 <= x[0] <= t1]
            for name, const in self.REASONS.items():
                bit = getattr(self._nvml, const, 0)
                if any(b & bit for _, _, b, _ in inside):
                    reasons.add(name)
            mhz = [m for _, m, _, _ in inside]
            watts = [w for _, _, _, w in inside]
            return {"sm_mhz": statistics.median(mhz) if mhz else None,
                    "sm_mhz_min": min(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                    "power_w_max": max(watts) if watts else None,
                    "reasons": sorted(reasons), "samples": len(mhz), "source": "nvml 5 ms"}
        sm, smax = [], []
        for line in self._lines:
            parts = [p.strip() for p in line.split(",")]
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except (ValueError, IndexError):
                continue
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": [],
                "samples": len(sm), "source": "nvidia-smi 200 ms (reasons not sampled)"}


# ---------------------------------------------------------------------------- oracle arm

def oracle_inputs(wl):
    from grouped_gemm_plan_b200 import workload as W
    x = W.make_x(wl)
    W1, W2 = W.make_weights(wl)
    ids, tw = W.make_routing(wl)
    return x, W1, W2, ids, tw


def oracle_tokens_per_s(wl, seconds: float, inputs=None):
    """Time the CPU oracle (per-token brute force, all host cores) on a bounded sample."""
    import oracle
    x, W1, W2, ids, tw = inputs if inputs is not None else oracle_inputs(wl)
    cores = oracle.num_threads()
    t0 = time.perf_counter()
    oracle.bruteforce_tokens(x, W1, W2, ids, tw, np.arange(min(cores, wl.M)))
    per_token = max(time.perf_counter() - t0, 1e-4) / min(cores, wl.M)   # all cores busy
    n = int(max(1, min(wl.M, seconds / per_token)))
    tokens = np.arange(n) * max(1, wl.M // n)
    tokens = tokens[tokens < wl.M]
    t0 = time.perf_counter()
    oracle.bruteforce_tokens(x, W1, W2, ids, tw, tokens)
    dt = time.perf_counter() - t0
    return len(tokens) / dt, len(tokens), dt, cores


def run_reference(args):
    from grouped_gemm_plan_b200 import workload as W
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = W.WORKLOADS[args.workload]
    import oracle
    oracle.build()
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps))
    inputs = oracle_inputs(wl)
    vals = []
    n_tok = 0
    cores = 1
    for i in range(args.warmup + args.steps):
        v, n, dt, cores = oracle_tokens_per_s(wl, per_step if i >= args.warmup else 0.5, inputs)
        if i >= args.warmup:
            vals.append(v)
            n_tok = n
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * wl.M / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "M": wl.M, "H": wl.H, "F": wl.F, "E": wl.E,
                   "topk": wl.topk, "routing": wl.routing, "std": wl.std, "seed": wl.seed},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n_tok} tokens per step of the {wl.name} batch, per-token "
                                   f"brute force in fp64"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------- our arm

GEMM_SOURCES = ["grouped_gemm.cu", "grouped_gemm_2sm.cu", "pair.cuh", "epilogue.cuh", "common.cuh"]


def kernel_sources_sha() -> str:
    """Hash of the sources the measured GEMM kernel is built from: a recorded DRAM
    traffic figure is used only while these are unchanged."""
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(ROOT, "grouped_gemm_plan_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str):
    try:
        with open(TRAFFIC_FILE) as f:
            rows = json.load(f)
    except (OSError, ValueError):
        return None
    sha = kernel_sources_sha()
    for r in rows:
        if r.get("kernel") == kernel and r.get("workload") == workload and r.get("source_sha") == sha:
            return r.get("dram_bytes_per_launch")
    return None


def plan_launches(R: int, num_sms: int) -> int:
    """Kernels the plan launches for R routed rows (mirrors its chunking)."""
    max_chunks = min(num_sms, 256)
    per_cta = -(-R // max_chunks)
    seg = max(32, -(-(-(-per_cta // 16)) // 32) * 32)
    return 1 if -(-R // (16 * seg)) <= 1 else 2


def run_ours(args):
    import torch
    from grouped_gemm_plan_b200 import binding as B
    from grouped_gemm_plan_b200 import dist as D
    from grouped_gemm_plan_b200 import workload as W

    rank, local, world = D.env_rank()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    D.init("nccl", timeout_s=120, device=dev)
    B.load()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    wl = D.shard(W.WORKLOADS[args.workload], rank)
    M, H, F, E, topk, R = wl.M, wl.H, wl.F, wl.E, wl.topk, wl.R
    x_h = W.make_x(wl).pin_memory()
    ids_np, tw_np = W.make_routing(wl)
    ids_h = torch.from_numpy(ids_np).pin_memory()
    tw_h = torch.from_numpy(tw_np).pin_memory()
    W1 = torch.empty((E, H, 2 * F), dtype=torch.bfloat16, device=dev)
    W2 = torch.empty((E, F, H), dtype=torch.bfloat16, device=dev)
    W.make_weights(wl, W1, W2)
    x = x_h.to(dev)
    ids = ids_h.to(dev)
    tw = tw_h.to(dev)
    out = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(R, dtype=torch.int32, device=dev)
    ws = B.alloc_workspace(B.OP_FFN_FUSED, M, H, F, E, topk, dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        B.moe_ffn_fused(x, W1, W2, ids, tw, out, counts, offsets, perm, ws, n_c=args.n_c)

    def barrier():
        D.barrier(dev)

    if args.n_c_sweep:
        for nc in [int(v) for v in args.n_c_sweep.split(",")]:
            for _ in range(args.warmup):
                flush.fill_(1)
                B.moe_ffn_fused(x, W1, W2, ids, tw, out, counts, offsets, perm, ws, n_c=nc)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for i in range(args.steps):
                flush.fill_(1)
                evs[i][0].record(stream)
                B.moe_ffn_fused(x, W1, W2, ids, tw, out, counts, offsets, perm, ws, n_c=nc)
                evs[i][1].record(stream)
            torch.cuda.synchronize()
            st = B.moe_get_device_status(ws)
            ms = [a.elapsed_time(b) for a, b in evs]
            if rank == 0:
                print(json.dumps({"workload": wl.name, "n_c": nc, "status": st,
                                  "ms_per_step": statistics.mean(ms), "ms_min": min(ms),
                                  "tokens_per_s": M / (statistics.mean(ms) / 1e3)}), flush=True)
        D.finish()
        return 0

    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    st = B.moe_get_device_status(ws)
    if st != B.MOE_OK:
        raise RuntimeError(f"device status {B.STATUS_NAMES.get(st)} after warm-up")

    # ---- timed region: K layer steps (the public call moe_ffn_fused), L2 flushed
    # before each, device time by CUDA events on the launching stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    # On large layers (no programmatic dependent launch between the stages, see
    # moe_ffn_fused) the library also records an event between its stages, so the
    # dominant kernel's duration comes from these very steps.
    in_step = R * H * F >= 2 ** 32
    tev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)] \
        if in_step else None
    barrier()
    t_begin = time.monotonic()
    for i in range(args.steps):
        flush.fill_(1)
        if in_step:
            B.moe_set_stage_events(tev[i])
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    if in_step:
        B.moe_set_stage_events(None)
    barrier()
    clocks.mark(t_begin, time.monotonic())
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    stage_names = ["plan", "dispatch", "gemm1_swiglu", "gemm2_scatter", "combine"]
    in_step_ms = {n: statistics.mean(tev[i][j].elapsed_time(tev[i][j + 1])
                                     for i in range(args.steps))
                  for j, n in enumerate(stage_names)} if in_step else None
    total_ms = sum(step_ms)
    st = B.moe_get_device_status(ws)
    if st != B.MOE_OK:
        raise RuntimeError(f"device status {B.STATUS_NAMES.get(st)} in the timed region")

    # ---- per-kernel times: K more steps, each stage a separate public call (the
    # same kernels as the n_c = 0 path) with events between them; its own clock
    # record decides which measured peak the dominant kernel is held to
    inv = torch.empty(R, dtype=torch.int32, device=dev)
    w_sorted = torch.empty(R, dtype=torch.float32, device=dev)
    xp = torch.empty((R, H), dtype=torch.bfloat16, device=dev)
    hbuf = torch.empty((R, F), dtype=torch.bfloat16, device=dev)
    yk = torch.empty((R, H), dtype=torch.float32, device=dev)
    out_chain = torch.empty_like(out)
    small_ws = B.alloc_workspace(B.OP_PLAN, M, H, F, E, topk, dev)
    names = ["plan", "dispatch", "gemm1_swiglu", "gemm2_scatter", "combine"]
    calls = [
        lambda: B.moe_plan(ids, tw, E, counts, offsets, perm, inv, w_sorted, small_ws),
        lambda: B.moe_dispatch(x, perm, topk, xp, small_ws),
        lambda: B.moe_grouped_gemm(xp, W1, offsets, B.EPI_SWIGLU, hbuf, small_ws),
        lambda: B.moe_grouped_gemm(hbuf, W2, offsets, B.EPI_WEIGHT_SCATTER, yk, small_ws,
                                   w_sorted=w_sorted, perm=perm),
        lambda: B.moe_combine(yk, None, None, M, topk, out_chain, small_ws),
    ]
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
           for _ in range(args.steps)]
    sclocks = ClockSampler(local)
    sclocks.start()
    barrier()
    s_begin = time.monotonic()
    for i in range(args.steps):
        flush.fill_(1)
        sev[i][0].record(stream)
        for j, c in enumerate(calls):
            c()
            sev[i][j + 1].record(stream)
    barrier()
    sclocks.mark(s_begin, time.monotonic())
    sclk = sclocks.stop()
    stage_avg = {n: statistics.mean(sev[i][j].elapsed_time(sev[i][j + 1])
                                    for i in range(args.steps))
                 for j, n in enumerate(names)}
    assert B.moe_get_device_status(small_ws) == B.MOE_OK
    assert torch.equal(out_chain.view(torch.int16), out.view(torch.int16)), \
        "stage-by-stage result differs from the layer call"

    # ---- the router in front of the layer (moe_route): fp32 logits [M, E] -> ids, w
    g = torch.Generator(device=dev).manual_seed(wl.seed)
    logits = torch.randn((M, E), generator=g, device=dev, dtype=torch.float32)
    r_ids = torch.empty((M, topk), dtype=torch.int32, device=dev)
    r_w = torch.empty((M, topk), dtype=torch.float32, device=dev)
    r_ws = B.alloc_workspace(B.OP_ROUTE, M, 0, 0, E, topk, dev)
    rev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    B.moe_route(logits, topk, r_ids, r_w, r_ws)
    rev[0].record(stream)
    for _ in range(10):
        B.moe_route(logits, topk, r_ids, r_w, r_ws)
    rev[1].record(stream)
    torch.cuda.synchronize()
    router_us = rev[0].elapsed_time(rev[1]) * 100.0
    assert B.moe_get_device_status(r_ws) == B.MOE_OK

    # ---- the layer with the FP8 (E4M3) down projection (moe_ffn_fused_fp8): W2
    # quantised once (offline step, not timed), then K steps timed like the bf16
    # ones, and the FP8 GEMM2 alone on the quantised h of the last step
    W2q = torch.empty((E, H, F), dtype=torch.uint8, device=dev)
    w2s = torch.empty((E, H), dtype=torch.float32, device=dev)
    B.moe_quantize_weights_e4m3(W2, W2q, w2s)
    ws8 = B.alloc_workspace(B.OP_FFN_FP8, M, H, F, E, topk, dev)
    out8 = torch.empty_like(out)
    for _ in range(args.warmup):
        flush.fill_(1)
        B.moe_ffn_fused_fp8(x, W1, W2q, w2s, ids, tw, out8, counts, offsets, perm, ws8)
    ev8 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(1)
        ev8[i][0].record(stream)
        B.moe_ffn_fused_fp8(x, W1, W2q, w2s, ids, tw, out8, counts, offsets, perm, ws8)
        ev8[i][1].record(stream)
    torch.cuda.synchronize()
    assert B.moe_get_device_status(ws8) == B.MOE_OK
    fp8_ms = statistics.mean(a.elapsed_time(b) for a, b in ev8)
    hq = torch.empty((R, F), dtype=torch.uint8, device=dev)
    hs = torch.empty(R, dtype=torch.float32, device=dev)
    B.moe_quantize_rows_e4m3(hbuf, hq, hs, small_ws)
    yk8 = torch.empty((R, H), dtype=torch.float32, device=dev)
    g8 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(1)
        g8[i][0].record(stream)
        B.moe_grouped_gemm_e4m3(hq, hs, W2q, w2s, offsets, yk8, small_ws, w_sorted=w_sorted,
                                perm=perm)
        g8[i][1].record(stream)
    torch.cuda.synchronize()
    assert B.moe_get_device_status(small_ws) == B.MOE_OK
    g8_ms = statistics.mean(a.elapsed_time(b) for a, b in g8)
    of, ob = out8.float(), out.float()
    fp8_info = {
        "ms_per_step": fp8_ms, "tokens_per_s": D.whole_job_rate(M, 1, fp8_ms / 1e3),
        "gemm2_e4m3_ms": g8_ms, "gemm2_e4m3_tflops": 2.0 * R * H * F / (g8_ms / 1e3) / 1e12,
        "rel_diff_vs_bf16_layer": float(torch.linalg.norm(of - ob) / torch.linalg.norm(ob)),
        "how": "moe_ffn_fused_fp8 (h and W2 in E4M3, per-row / per-column fp32 scales), L2 "
               "flushed before each step; the GEMM2 rate on the quantised h of the last step",
    }
    del W2q, ws8, hq, yk8

    # ---- end to end: every step's inputs are copied in from pinned host memory and
    # its result copied back, through the public call.  As in a serving loop, step
    # i+1's upload (one copy stream) and step i-1's download (another) overlap step
    # i's compute; device inputs and outputs are double-buffered.  The timed region
    # runs from before the first upload to after the last download.
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    bufs = [{"x": torch.empty_like(x), "ids": torch.empty_like(ids), "tw": torch.empty_like(tw),
             "out": torch.empty_like(out)} for _ in range(2)]
    outs_h = [torch.empty((M, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    n = args.steps
    up_done = [torch.cuda.Event() for _ in range(n)]
    comp_done = [torch.cuda.Event() for _ in range(n)]
    down_done = [torch.cuda.Event() for _ in range(n)]
    e2e_start = torch.cuda.Event(enable_timing=True)
    e2e_end = torch.cuda.Event(enable_timing=True)

    def upload(i):
        b = bufs[i % 2]
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(comp_done[i - 2])      # step i-2 has consumed this buffer
            b["x"].copy_(x_h, non_blocking=True)
            b["ids"].copy_(ids_h, non_blocking=True)
            b["tw"].copy_(tw_h, non_blocking=True)
            up_done[i].record(up)

    barrier()
    e2e_start.record(stream)
    up.wait_stream(stream)
    down.wait_stream(stream)
    upload(0)
    for i in range(n):
        if i + 1 < n:
            upload(i + 1)
        b = bufs[i % 2]
        stream.wait_event(up_done[i])
        if i >= 2:
            stream.wait_event(down_done[i - 2])      # this output buffer was read back
        B.moe_ffn_fused(b["x"], W1, W2, b["ids"], b["tw"], b["out"], counts, offsets, perm, ws,
                        n_c=args.n_c, stream=stream)
        comp_done[i].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(comp_done[i])
            outs_h[i % 2].copy_(b["out"], non_blocking=True)
            down_done[i].record(down)
    stream.wait_event(down_done[n - 1])
    e2e_end.record(stream)
    barrier()
    e2e_ms = e2e_start.elapsed_time(e2e_end)
    st = B.moe_get_device_status(ws)
    if st != B.MOE_OK:
        raise RuntimeError(f"device status {B.STATUS_NAMES.get(st)} in the end-to-end run")
    assert torch.equal(outs_h[(n - 1) % 2].view(torch.int16), out.cpu().view(torch.int16)), \
        "end-to-end result differs from the device-timed result"
    h2d = x_h.numel() * 2 + ids_h.numel() * 4 + tw_h.numel() * 4
    d2h = outs_h[0].numel() * 2

    # ---- max over ranks
    total_ms, e2e_ms = D.max_over_ranks([total_ms, e2e_ms], dev)
    ms_per_step = total_ms / args.steps
    value = D.whole_job_rate(M * args.steps, world, total_ms / 1e3)
    e2e_value = D.whole_job_rate(M * args.steps, world, e2e_ms / 1e3)

    pk, pk_kind = peaks()
    flops_g1 = 4.0 * R * H * F
    # GEMM1's launches inside the timed steps when the library recorded them there,
    # else the separate stage-by-stage loop.
    src_ms, src_clk = (in_step_ms, clk) if in_step else (stage_avg, sclk)
    g1_s = src_ms["gemm1_swiglu"] / 1e3
    achieved = flops_g1 / g1_s / 1e12
    # Held to the burst figure of the measured cuBLAS bf16 GEMM while the SM clock
    # stays near its maximum; to the sustained (power-capped) figure once the clock
    # has dropped.
    capped = (src_clk.get("sm_mhz") is not None and src_clk.get("sm_max_mhz")
              and src_clk["sm_mhz"] < 0.9 * src_clk["sm_max_mhz"])
    peak = pk.get("bf16_tflops_sustained", pk["bf16_tflops"]) if capped else pk["bf16_tflops"]
    traffic = measured_traffic("gemm1_swiglu", wl.name)
    # which GEMM kernel the library runs for this shape (its rule: CTA pairs once
    # experts average 1024 rows or more, unless MOE_GEMM_PAIR forces one)
    forced = os.environ.get("MOE_GEMM_PAIR", "")
    pair = forced == "1" or (forced != "0" and R >= 1024 * E)
    roofline = {"kernel": "grouped GEMM1 + SwiGLU epilogue",
                "kernel_variant": ("grouped_gemm_2sm_kernel (CTA pair, 256x256 tiles)" if pair
                                   else "grouped_gemm_kernel (single CTA, 128x256 tiles)"),
                "bound": "tensor",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_source": f"{pk_kind} " + ("bf16_tflops_sustained (SM clock dropped under the "
                                                 "power cap)" if capped else "bf16_tflops (burst)"),
                "timed_in": ("the timed layer steps (events between the library's stage "
                             "launches)" if in_step else "the stage-by-stage loop"),
                "kernel_loop_clocks": src_clk,
                "peak_sustained": pk.get("bf16_tflops_sustained"), "traffic": traffic,
                "algorithmic": f"4*R*H*F = {flops_g1:.4g} FLOP per launch"}
    g2 = 2.0 * R * H * F / (src_ms["gemm2_scatter"] / 1e3) / 1e12
    # E4M3 peak = the measured bf16 peak x 2 (the nominal fp8 : bf16 dense ratio)
    fp8_info["gemm2_e4m3_frac_of_fp8_peak"] = fp8_info["gemm2_e4m3_tflops"] / (2.0 * peak)
    fp8_info["fp8_peak_tflops"] = 2.0 * peak
    disp_bytes = M * H * 2 + R * H * 2 + R * 4
    comb_bytes = R * H * 4 + M * H * 2
    extra = {
        "stages_ms": stage_avg,
        "stages_in_timed_steps_ms": in_step_ms,
        "gemm1_tflops": achieved, "gemm2_tflops": g2,
        "grouped_gemm_frac_of_bf16_peak": {"gemm1": achieved / peak, "gemm2": g2 / peak},
        "dispatch_gbs": disp_bytes / (src_ms["dispatch"] / 1e3) / 1e9,
        # read + written bytes over the measured copy bandwidth (which counts both)
        "dispatch_frac_of_hbm": disp_bytes / (src_ms["dispatch"] / 1e3) / 1e9 / pk["hbm_gbs"],
        "combine_frac_of_hbm": comb_bytes / (src_ms["combine"] / 1e3) / 1e9 / pk["hbm_gbs"],
        "combine_gbs": comb_bytes / (src_ms["combine"] / 1e3) / 1e9,
        "hbm_peak_gbs": pk["hbm_gbs"],
        "layer_tflops": wl.flops() / (ms_per_step / 1e3) / 1e12,
        "router_us": router_us,
        "fp8_layer": fp8_info,
    }

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        v, n, dt, cores = oracle_tokens_per_s(W.WORKLOADS[args.workload], args.cpu_seconds)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} tokens of the {wl.name} batch, per-token brute force in fp64, "
                         f"{dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": wl.name, "M": M, "H": H, "F": F, "E": E, "topk": topk,
                       "routing": wl.routing, "std": wl.std, "seed": W.WORKLOADS[args.workload].seed,
                       "n_c": args.n_c, "l2": "flushed (256 MiB write) before every timed step",
                       "parallelism": f"dp{world} (independent batches, no collective)"},
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "how": "public call moe_ffn_fused; every step uploads x, topk_ids, topk_w "
                           "from pinned host memory and downloads out; uploads and downloads "
                           "run on two copy streams, double-buffered, overlapping the "
                           "neighbouring steps' compute; one event pair around all steps"},
            "gpu_launches": args.steps * (plan_launches(R, sms) + 4),
            "roofline": roofline,
            "cpu_baseline": cpu,
            "clocks": clk,
            **extra,
        }
        print(json.dumps(line), flush=True)
    D.finish()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
