#!/usr/bin/env python3
"""Benchmark of the residual binarized linear layer on B200.

Workload: the Llama-7B q_proj shape, N = K = 4096 with k = 2 residual sign
planes (W ~ N(0, 0.02) with 0.1% x20 outliers, greedy-SVID scales), decode
M = 1.  One step = 32 decode tokens, one after another; each token applies 96
distinct, independent packed layers of that shape to its activation vector
with one rb_gemv_batch call (one launch; programmatic dependent launch between
the tokens' launches; captured in a CUDA graph).  The 96 layers hold ~403 MB of
sign planes, more than the 126 MB L2, so every step streams the planes from
HBM.  Metric: packed-weight bytes read per second (GB/s).  The same 3072
applications issued as single-layer rb_gemv calls in one dependent chain are
reported beside it (decode_chain).

Legs (one JSON line on rank 0):
  value       device-timed (CUDA events) throughput, inputs resident in HBM;
  e2e         the same step with X copied host->device from pinned memory and
              the last layer's Y copied back, inside the timed region;
  roofline    the GEMV kernel's algorithmic bytes per launch / its average
              duration against the measured HBM copy bandwidth;
  cpu_baseline  the CPU oracle (float64 dequantise-then-multiply) on a bounded
              sample of the same workload (rank 0, N = 1 only);
  rows        the other hot-path steps measured in the same run (rb_pack,
              rb_gemv at M = 4 and 16, rb_gemm).
--impl reference times the CPU oracle itself on this workload.
Multi-GPU: every rank runs its own independent layer stack (weak scaling, no
data-path collective); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import math
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

N_OUT, K_IN, K_PLANES = 4096, 4096, 2
WORKLOAD = "q_proj_4096x4096_k2"
METRIC = "packed-weight HBM GB/s (% of B200 peak) for k=2 binary GEMV; GEMM TFLOP/s"
LAYERS, TOKENS = 96, 32
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ---------------------------------------------------------------- distributed plumbing
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False

    def init(self, backend):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, x: float, device=None) -> float:
        if not self.pg:
            return x
        import torch
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


def rowsplit_gather(dist, y_local, n_out, shard_bounds):
    """Row-parallel split: every rank holds Y[:, row0_r:row1_r] ([M][rows_r], a
    torch tensor); returns the full [M][n_out] on every rank.  Shards are padded
    to the largest one for one all_gather, then cut and concatenated along N."""
    import torch
    if not dist.pg:
        return y_local
    import torch.distributed as td
    bounds = [shard_bounds(n_out, dist.world, r) for r in range(dist.world)]
    width = max(b1 - b0 for b0, b1 in bounds)
    M = y_local.shape[0]
    pad = torch.zeros(M, width, dtype=y_local.dtype, device=y_local.device)
    pad[:, :y_local.shape[1]] = y_local
    parts = [torch.empty_like(pad) for _ in range(dist.world)]
    td.all_gather(parts, pad)
    return torch.cat([p[:, :b1 - b0] for p, (b0, b1) in zip(parts, bounds)], dim=1)


def assemble_line(*, value, unit, n_gpus, steps, warmup, ms_per_step, extra) -> dict:
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": n_gpus, "steps": steps,
            "warmup": warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u32 sign planes x bf16 -> f32",
            "data": "synthetic"}
    line.update(extra)
    return line


def throughput(bytes_per_step_per_rank: float, world: int, steps: int, seconds_max: float) -> float:
    """Whole-job GB/s: bytes all ranks processed / max-over-ranks time."""
    return bytes_per_step_per_rank * world * steps / seconds_max / 1e9


# ---------------------------------------------------------------- peaks, clocks, profiles
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


REJECT_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


def clocks_rejected(clocks) -> bool:
    """A timed region that saw thermal or hardware slowdown, or whose median SM
    clock sat well below the maximum with no power cap to explain it (a clock
    lock left behind), is taken again."""
    if not clocks:
        return False
    reasons = set(clocks.get("reasons") or [])
    if reasons & REJECT_REASONS:
        return True
    sm, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    return bool(sm and mx and sm < 0.8 * mx and "sw_power_cap" not in reasons)


def timed_with_retake(dist, sample_and_time, device=None):
    """Run the timed region (sample_and_time() -> (seconds, clocks)) and take it
    once more when the clock record of ANY rank is rejected.  The decision is
    collective (MAX over ranks of a 0/1 flag), so every rank runs the same
    sequence of barriers and reductions whichever rank saw the slowdown."""
    t_local, clocks = sample_and_time()
    if dist.max(1.0 if clocks_rejected(clocks) else 0.0, device) > 0.0:
        first = clocks
        t_local, clocks = sample_and_time()
        clocks = dict(clocks or {})
        clocks["retaken"] = True
        clocks["first_attempt"] = first
    return t_local, clocks


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region.

    Each sample is stamped on arrival; only samples that arrive between begin()
    and end() (the host-side bracket of the timed region) count.
    """

    def __init__(self, gpu_id: str | None, interval_ms=20):
        self.gpu_id, self.interval_ms = gpu_id, interval_ms
        self.proc, self.lines = None, []
        self.t0 = self.t1 = None

    def start(self, wait_s=5.0):
        cmd = ["nvidia-smi", "--query-gpu=clocks.sm,clocks.max.sm,utilization.gpu,power.draw,clocks_event_reasons.active",
               "--format=csv,noheader,nounits", "-lms", str(self.interval_ms)]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except Exception:
            self.proc = None
            return
        deadline = time.monotonic() + wait_s          # the first sample marks a running sampler
        while not self.lines and time.monotonic() < deadline and self.proc.poll() is None:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def begin(self):
        self.t0 = time.monotonic()

    def end(self):
        self.t1 = time.monotonic()
        time.sleep(2.5 * self.interval_ms / 1e3)     # let the last in-window sample arrive

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.reader.join(timeout=2)
        t0 = self.t0 if self.t0 is not None else float("-inf")
        t1 = self.t1 if self.t1 is not None else float("inf")
        sm, mx, reasons = [], [], set()
        for ts, ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 5:
                continue
            try:
                s, m = float(parts[0]), float(parts[1])
                bits = int(parts[4], 16) if parts[4].lower().startswith("0x") else int(parts[4])
            except ValueError:
                continue
            mx.append(m)
            if t0 <= ts <= t1:
                sm.append(s)
                for b, name in REASON_BITS.items():
                    if bits & b and name != "gpu_idle":
                        reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                    "samples_in_timed_region": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples_in_timed_region": len(sm)}


def kernel_sources_sha() -> str:
    h = hashlib.sha256()
    for f in ("rb_gemv.cu", "rbw_internal.cuh"):
        with open(os.path.join(ROOT, "residual_binarized_weight_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_tag: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(p):
        return None
    sha = kernel_sources_sha()
    for ln in open(p):
        f = dict(kv.split("=", 1) for kv in ln.split() if "=" in kv)
        if f.get("kernel") == kernel_tag and f.get("src_sha") == sha:
            return float(f["dram_bytes_per_launch"])
    return None


# ---------------------------------------------------------------- CPU oracle legs
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample(seconds_budget=12.0, max_layers=TOKENS * LAYERS, threads=None):
    """Time the oracle's float64 apply on the workload layer: applications until
    about seconds_budget of CPU work has run, at most one step's worth (on
    `threads` OpenMP threads if given, else all)."""
    import oracle
    if threads is not None:
        all_threads = oracle.threads()
        oracle.set_threads(threads)
        try:
            return oracle_sample(seconds_budget, max_layers)
        finally:
            oracle.set_threads(all_threads)
    from residual_binarized_weight_b200 import synth
    wl = synth.workload(WORKLOAD)
    W = synth.weights(wl.layers[0])
    g, h = oracle.svid_greedy(W, K_PLANES, iters=20)
    planes, g16, h16, st, _ = oracle.pack(W, g, h, K_PLANES)
    X = synth.activations_for(wl, TOKENS, K_IN)
    plane_bytes = 4 * planes.size
    t0 = time.perf_counter()
    n = 0
    while n < max_layers:
        oracle.apply(planes, g16, h16, N_OUT, K_IN, K_PLANES, X[n % TOKENS:n % TOKENS + 1])
        n += 1
        if time.perf_counter() - t0 > seconds_budget:
            break
    dt = time.perf_counter() - t0
    return {"value": plane_bytes * n / dt / 1e9, "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
            "cpu_model": cpu_model(), "nproc": os.cpu_count(),
            "sample": "%d single-token (M=1) applications of one %dx%d k=%d layer, float64 dequantise-then-multiply, %.1f s"
                      % (n, N_OUT, K_IN, K_PLANES, dt)}, dt / n


def run_reference(args, dist: Dist):
    """The CPU oracle as the reference arm.  One reference step is a bounded
    sample of the GPU arm's step: `apps` single-token applications of the
    workload layer (the GPU step runs 3072), sized from a calibration run so
    that warm-up plus timed steps take about a minute.  ms_per_step is the
    measured time of those steps, so steps x ms_per_step is the timed region."""
    if dist.rank != 0:
        return 0
    import oracle
    from residual_binarized_weight_b200 import synth
    wl = synth.workload(WORKLOAD)
    W = synth.weights(wl.layers[0])
    g, h = oracle.svid_greedy(W, K_PLANES, iters=20)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, K_PLANES)
    X = synth.activations_for(wl, TOKENS, K_IN)
    plane_bytes = 4 * planes.size

    def apply(n0, n):
        for j in range(n0, n0 + n):
            oracle.apply(planes, g16, h16, N_OUT, K_IN, K_PLANES, X[j % TOKENS:j % TOKENS + 1])
    t0 = time.perf_counter()
    apply(0, 2)                                   # calibration (also warms the library and caches)
    t_app = (time.perf_counter() - t0) / 2
    per_step_s = max(0.2, min(5.0, 60.0 / max(1, args.steps + args.warmup)))
    apps = max(1, min(TOKENS * LAYERS, int(per_step_s / t_app)))
    for w in range(args.warmup):
        apply(w * apps, apps)
    t0 = time.perf_counter()
    for s_ in range(args.steps):
        apply(s_ * apps, apps)
    dt = time.perf_counter() - t0
    value = plane_bytes * apps * args.steps / dt / 1e9
    cb = {"value": value, "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
          "cpu_model": cpu_model(), "nproc": os.cpu_count(),
          "sample": "each step: %d single-token (M=1) applications of one %dx%d k=%d layer (the GPU step runs %d), "
                    "float64 dequantise-then-multiply; %d steps in %.1f s" % (apps, N_OUT, K_IN, K_PLANES,
                                                                          TOKENS * LAYERS, args.steps, dt)}
    line = assemble_line(value=value, unit="GB/s", n_gpus=args.gpus, steps=args.steps, warmup=args.warmup,
                         ms_per_step=dt / max(1, args.steps) * 1e3,
                         extra={"impl": "reference", "config": config_dict(),
                                "reference_step": {"applications": apps, "of_gpu_step": TOKENS * LAYERS},
                                "cpu_baseline": cb,
                                "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}})
    print(json.dumps(line), flush=True)
    return 0


def config_dict():
    return {"workload": WORKLOAD, "n_out": N_OUT, "k_in": K_IN, "k_planes": K_PLANES, "M": 1,
            "layers_per_step": LAYERS, "tokens_per_step": TOKENS,
            "l2": "inputs larger than L2: %d distinct packed layers = %.0f MB of planes per pass" %
                  (LAYERS, LAYERS * 4.194304),
            "parallelism": "independent replicas (weak scaling, no collective)"}


# ---------------------------------------------------------------- GPU leg
def gpu_uuid(torch):
    try:
        u = torch.cuda.get_device_properties(torch.cuda.current_device()).uuid
        return "GPU-" + str(u)
    except Exception:
        return None


def run_rbw(args, dist: Dist):
    import torch
    from residual_binarized_weight_b200 import rbw, synth

    torch.cuda.set_device(dist.local_rank)
    dist.init("nccl")
    dev = torch.device("cuda", dist.local_rank)
    hbm_peak, bf16_peak, bf16_sust, peak_src = measured_peaks()
    wl = synth.workload(WORKLOAD)

    # ---- deploy: derive scales + pack one seeded layer, replicate to LAYERS distinct buffers
    W = torch.from_numpy(synth.weights(wl.layers[0])).to(dev)
    g, h = rbw.svid_greedy(W, K_PLANES, iters=20)
    base = rbw.pack(W, g, h, K_PLANES)
    layers = []
    for _ in range(LAYERS):
        L = rbw.PackedLayer(N_OUT, K_IN, K_PLANES, dev)
        L.planes.copy_(base.planes)
        L.g16.copy_(base.g16)
        L.h16.copy_(base.h16)
        layers.append(L)
    structs = [L.struct() for L in layers]
    X_host = synth.activations_for(wl, TOKENS, K_IN)
    X = torch.from_numpy(X_host.view(np.int16)).to(dev)
    Y_last = torch.empty(TOKENS, N_OUT, dtype=torch.float32, device=dev)
    lib = rbw.lib()
    import ctypes

    # batch of the 96 layers of a token: host arrays of device pointers, built once
    nb = LAYERS
    PER_LAUNCH = 96                          # layers per rb_gemv_batch call (one call per token)
    lp = (ctypes.POINTER(rbw.RbLayer) * nb)(*[ctypes.pointer(structs[j]) for j in range(nb)])
    ytmp = torch.empty(LAYERS - 1, N_OUT, dtype=torch.float32, device=dev)
    xps = [(ctypes.c_void_p * nb)(*([X.data_ptr() + t * K_IN * 2] * nb)) for t in range(TOKENS)]
    yps = [(ctypes.c_void_p * nb)(*([ytmp.data_ptr() + j * N_OUT * 4 for j in range(LAYERS - 1)] +
                                    [Y_last.data_ptr() + t * N_OUT * 4])) for t in range(TOKENS)]
    streams = [torch.cuda.Stream(dev)]

    def step_batched():
        """32 tokens, one after another; per token one rb_gemv_batch over the 96 layers."""
        sp = ctypes.c_void_p(streams[0].cuda_stream)
        for t in range(TOKENS):
            for b in range(0, nb, PER_LAUNCH):
                n = min(PER_LAUNCH, nb - b)
                st = lib.rb_gemv_batch(ctypes.c_void_p(ctypes.addressof(lp) + b * ctypes.sizeof(ctypes.c_void_p)),
                                       ctypes.c_void_p(ctypes.addressof(xps[t]) + b * ctypes.sizeof(ctypes.c_void_p)),
                                       ctypes.c_void_p(ctypes.addressof(yps[t]) + b * ctypes.sizeof(ctypes.c_void_p)),
                                       n, 1, rbw.RB_F32, None, rbw.RB_LAUNCH_PDL, sp)
                if st != 0:
                    raise rbw.RbError("rb_gemv_batch", st)

    def step_chain():
        """The same 3072 applications as single-layer rb_gemv calls, one dependent chain (PDL)."""
        sp = ctypes.c_void_p(streams[0].cuda_stream)
        for t in range(TOKENS):
            xp = ctypes.c_void_p(X.data_ptr() + t * K_IN * 2)
            for li in range(LAYERS):
                yp = ctypes.c_void_p((Y_last.data_ptr() + t * N_OUT * 4) if li == LAYERS - 1
                                     else ytmp.data_ptr() + li * N_OUT * 4)
                st = lib.rb_gemv(ctypes.byref(structs[li]), xp, 1, yp, rbw.RB_F32, None, 0, None,
                                 rbw.RB_LAUNCH_PDL, sp)
                if st != 0:
                    raise rbw.RbError("rb_gemv", st)

    def capture(fn, pre=None, post=None):
        with torch.cuda.stream(streams[0]):
            fn()                           # eager run (sets kernel attributes)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=streams[0]):
            if pre:
                pre()
            fn()
            if post:
                post()
        torch.cuda.synchronize()
        return gr

    def time_graph(gr, steps, sync_each=False, sampler=None):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(streams[0]):
            for _ in range(max(3, args.warmup)):
                gr.replay()
            torch.cuda.synchronize()
            dist.barrier()
            if sampler:
                sampler.begin()
            e0.record(streams[0])
            for _ in range(steps):
                gr.replay()
                if sync_each:
                    streams[0].synchronize()       # the host reads each step's result
            e1.record(streams[0])
        torch.cuda.synchronize()
        if sampler:
            sampler.end()
        dist.barrier()
        return e0.elapsed_time(e1) / 1e3

    launches_per_step = TOKENS * LAYERS          # layer applications per step
    kernel_launches_per_step = TOKENS * ((LAYERS + PER_LAUNCH - 1) // PER_LAUNCH)
    plane_bytes = layers[0].packed_bytes()
    bytes_per_step = plane_bytes * launches_per_step
    algo_bytes_per_launch = plane_bytes + 2 * K_PLANES * (N_OUT + K_IN) + 2 * K_IN + 4 * N_OUT

    graph = capture(step_batched)

    def sample_and_time():
        sampler = ClockSampler(gpu_uuid(torch))
        sampler.start()
        t = time_graph(graph, args.steps, sampler=sampler)
        return t, sampler.stop()
    t_local, clocks = timed_with_retake(dist, sample_and_time, dev)
    t_max = dist.max(t_local, dev)
    value = throughput(bytes_per_step, dist.world, args.steps, t_max)
    avg_launch_s = t_local / (args.steps * launches_per_step)      # per layer application
    achieved = algo_bytes_per_launch / avg_launch_s / 1e9
    del graph

    chain_graph = capture(step_chain)
    chain_steps = max(1, min(args.steps, 50))
    t_chain = dist.max(time_graph(chain_graph, chain_steps), dev)
    chain = {"GBps": throughput(bytes_per_step, dist.world, chain_steps, t_chain),
             "us_per_layer": t_chain / (chain_steps * launches_per_step) * 1e6,
             "what": "single-layer rb_gemv calls on one stream, each launched with PDL after the previous one (dependent decode chain)"}
    del chain_graph

    # ---- e2e: host X in pinned memory -> device, the step, Y of the last layer -> host
    X_pin = torch.from_numpy(X_host.view(np.int16).copy()).pin_memory()
    Y_pin = torch.empty(TOKENS, N_OUT, dtype=torch.float32).pin_memory()
    graph_e2e = capture(step_batched, pre=lambda: X.copy_(X_pin, non_blocking=True),
                        post=lambda: Y_pin.copy_(Y_last, non_blocking=True))
    e2e_steps = max(1, min(args.steps, 200))
    t_e2e = dist.max(time_graph(graph_e2e, e2e_steps, sync_each=True), dev)
    e2e = {"value": throughput(bytes_per_step, dist.world, e2e_steps, t_e2e), "unit": "GB/s",
           "h2d_bytes_per_step": X_pin.numel() * 2, "d2h_bytes_per_step": Y_pin.numel() * 4,
           "steps": e2e_steps}
    del graph_e2e

    rows = other_rows(args, torch, rbw, synth, dev, W, g, h, bf16_peak) if (dist.rank == 0 and not args.quick) else {}
    dist.barrier()
    line = None
    if dist.rank == 0:
        cb = None
        if dist.world == 1 and not args.no_cpu_baseline:
            cb, _ = oracle_sample(seconds_budget=args.cpu_seconds)
            one, _ = oracle_sample(seconds_budget=3.0, threads=1)
            cb["single_thread"] = {"value": one["value"], "unit": one["unit"], "cores": one["cores"],
                                   "sample": one["sample"]}
        line = assemble_line(
            value=value, unit="GB/s", n_gpus=dist.world, steps=args.steps, warmup=args.warmup,
            ms_per_step=t_max / args.steps * 1e3,
            extra={"impl": "rbw", "config": config_dict(),
                   "pct_of_peak": {"measured_hbm": value / dist.world / hbm_peak, "spec_8tbs": value / dist.world / 8000.0},
                   "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                                "frac": achieved / hbm_peak, "traffic": profiled_traffic("gemv_lut_kernel<2>"),
                                "traffic_unit": "DRAM bytes per launch of %d layers (ncu)" % PER_LAUNCH,
                                "kernel": "gemv_lut_kernel<2> via rb_gemv_batch", "peak_source": peak_src,
                                "algorithmic_bytes_per_layer": algo_bytes_per_launch,
                                "layers_per_launch": PER_LAUNCH,
                                "avg_us_per_layer": avg_launch_s * 1e6,
                                "avg_launch_us": avg_launch_s * 1e6 * PER_LAUNCH},
                   "cpu_baseline": cb, "e2e": e2e, "gpu_launches": args.steps * kernel_launches_per_step,
                   "decode_chain": chain,
                   "clocks": clocks, "rows": rows})
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


def time_events(torch, fn, reps, stream):
    with torch.cuda.stream(stream):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3 / reps


def time_graph_calls(torch, fn, reps, stream):
    """Per-call device time of `fn` with the host out of the way: `reps` calls are
    captured into one CUDA graph (after an eager call), which is replayed after
    warm-up between CUDA events on `stream`."""
    with torch.cuda.stream(stream):
        fn()
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr, stream=stream):
        for _ in range(reps):
            fn()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for _ in range(3):
            gr.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(5):
            gr.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / (5 * reps)
    del gr
    return t


def other_rows(args, torch, rbw, synth, dev, W, g, h, bf16_peak):
    """Device timings of the other hot-path steps on the same layer (kernels only)."""
    out = {}
    stream = torch.cuda.Stream(dev)
    # rb_pack: reads W (4NK bytes), writes planes + fp16 scales
    Lp = rbw.PackedLayer(N_OUT, K_IN, K_PLANES, dev)
    t = time_graph_calls(torch, lambda: rbw.pack(W, g, h, K_PLANES, out=Lp, stream=stream), 20, stream)
    pack_bytes = 4 * N_OUT * K_IN + Lp.packed_bytes() + 2 * K_PLANES * (N_OUT + K_IN)
    out["pack"] = {"us": t * 1e6, "GBps": pack_bytes / t / 1e9, "bytes": pack_bytes}
    # rb_gemv at M = 4 and 16 over 96 distinct layers (L2-defeating), plain launches
    layers = []
    for _ in range(LAYERS):
        L = rbw.PackedLayer(N_OUT, K_IN, K_PLANES, dev)
        L.planes.copy_(Lp.planes)
        L.g16.copy_(Lp.g16)
        L.h16.copy_(Lp.h16)
        layers.append(L)
    for M in (1, 4, 16):
        X = torch.from_numpy(synth.activations(M, K_IN, seed=M).view(np.int16)).to(dev)
        Y = torch.empty(M, N_OUT, dtype=torch.float32, device=dev)
        ws = rbw.workspace(rbw.gemv_workspace_bytes(N_OUT, K_IN, K_PLANES, M), dev)
        it = iter(range(10 ** 9))

        def f():
            rbw.gemv(layers[next(it) % LAYERS], X, Y=Y, ws=ws, stream=stream)
        t = time_events(torch, f, 2 * LAYERS, stream)
        out["gemv_M%d_plain_launches" % M] = {"us": t * 1e6, "packed_GBps": Lp.packed_bytes() / t / 1e9,
                               "tokens_per_s": M / t}
    # isolated single-layer launch at M = 1: a write of 2 x L2 bytes before each launch
    # evicts the planes, and the launch alone sits between the events (the figures above
    # are sustained: back-to-back launches over layers that do not fit in L2)
    try:
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
        X1 = torch.from_numpy(synth.activations(1, K_IN, seed=1).view(np.int16)).to(dev)
        Y1 = torch.empty(1, N_OUT, dtype=torch.float32, device=dev)
        ts = []
        with torch.cuda.stream(stream):
            for r in range(23):
                flush.fill_(r & 0xFF)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                rbw.gemv(layers[r % LAYERS], X1, Y=Y1, stream=stream)
                e1.record(stream)
                e1.synchronize()
                ts.append(e0.elapsed_time(e1) * 1e3)
        ts = sorted(ts[3:])
        med = ts[len(ts) // 2]
        out["gemv_M1_isolated"] = {"us_median": med, "packed_GBps": Lp.packed_bytes() / med / 1e3,
                                   "flush_bytes": 2 * l2, "launches": len(ts)}
        del flush
    except Exception as e:                       # an informational row: record why it is missing
        out["gemv_M1_isolated"] = {"unavailable": repr(e)[:200]}
    # rb_gemv_batch at M = 4 and 16 (one tensor-core launch over the 96 layers), and
    # rb_gemv at M = 64 (the path its size selects), 96 distinct layers
    for M in (4, 16):
        X = torch.from_numpy(synth.activations(M, K_IN, seed=M).view(np.int16)).to(dev)
        Ys = [torch.empty(M, N_OUT, dtype=torch.float32, device=dev) for _ in range(LAYERS)]
        t = time_graph_calls(torch, lambda: rbw.gemv_batch(layers, [X] * LAYERS, Ys, stream=stream), 5,
                             stream) / LAYERS
        out["gemv_M%d_batch96" % M] = {"us_per_layer": t * 1e6, "packed_GBps": Lp.packed_bytes() / t / 1e9,
                                       "TFLOPs": 2.0 * M * N_OUT * K_IN * K_PLANES / t / 1e12}
    X = torch.from_numpy(synth.activations(64, K_IN, seed=64).view(np.int16)).to(dev)
    Y = torch.empty(64, N_OUT, dtype=torch.float32, device=dev)
    ws = rbw.workspace(rbw.gemv_workspace_bytes(N_OUT, K_IN, K_PLANES, 64), dev)
    it64 = iter(range(10 ** 9))
    t = time_graph_calls(torch, lambda: rbw.gemv(layers[next(it64) % LAYERS], X, Y=Y, ws=ws, stream=stream),
                         2 * LAYERS, stream)
    out["gemv_M64"] = {"us": t * 1e6, "packed_GBps": Lp.packed_bytes() / t / 1e9,
                       "TFLOPs": 2.0 * 64 * N_OUT * K_IN * K_PLANES / t / 1e12,
                       "path": "tcgen05" if rbw.gemv_workspace_bytes(N_OUT, K_IN, K_PLANES, 64) else "mma.sync"}
    # backward data path: rb_transpose_planes over the 96 layers (reads and writes the
    # planes once), then the input gradient dX = dY . What of one token per layer
    # through rb_gemv_batch on the transposed layers
    tlayers = [rbw.transpose(L, stream=stream) for L in layers]
    itt = iter(range(10 ** 9))

    def tr():
        j = next(itt) % LAYERS
        rbw.transpose(layers[j], out=tlayers[j], stream=stream)
    t = time_graph_calls(torch, tr, 2 * LAYERS, stream)
    out["transpose_planes"] = {"us": t * 1e6, "GBps": 2 * Lp.packed_bytes() / t / 1e9,
                               "bytes": 2 * Lp.packed_bytes()}
    dY = torch.from_numpy(synth.activations(1, N_OUT, seed=11).view(np.int16)).to(dev)
    dXs = [torch.empty(1, K_IN, dtype=torch.float32, device=dev) for _ in range(LAYERS)]
    t = time_graph_calls(torch, lambda: rbw.gemv_batch(tlayers, [dY] * LAYERS, dXs, stream=stream), 5,
                         stream) / LAYERS
    out["input_grad_M1_batch96"] = {"us_per_layer": t * 1e6, "packed_GBps": Lp.packed_bytes() / t / 1e9}
    del layers, tlayers
    # device scale derivation: greedy SVID (20 power iterations per plane) and the
    # one-call deployment path rb_svid_pack (SVID scales, then planes + fp16 scales)
    t = time_events(torch, lambda: rbw.svid_greedy(W, K_PLANES, iters=20, stream=stream), 3, stream)
    out["svid_greedy"] = {"us": t * 1e6, "iters": 20, "planes": K_PLANES,
                          "W_passes": K_PLANES * (2 * 20 + 1), "W_bytes": 4 * N_OUT * K_IN}
    Ls = rbw.PackedLayer(N_OUT, K_IN, K_PLANES, dev)
    t = time_events(torch, lambda: rbw.svid_pack(W, K_PLANES, sweeps=0, iters=20, out=Ls, stream=stream), 3, stream)
    out["svid_pack_greedy"] = {"us": t * 1e6}
    t = time_events(torch, lambda: rbw.svid_pack(W, K_PLANES, sweeps=2, iters=20, out=Ls, stream=stream), 1, stream)
    out["svid_pack_2_sweeps"] = {"us": t * 1e6}
    # plain row-major words <-> storage layout (one read and one write of the planes)
    rm = rbw.planes_to_rowmajor(Lp, stream=stream)
    t = time_graph_calls(torch, lambda: rbw.planes_from_rowmajor(rm, N_OUT, K_IN, K_PLANES, out=Ls, stream=stream),
                         20, stream)
    out["planes_from_rowmajor"] = {"us": t * 1e6, "GBps": 2 * Lp.packed_bytes() / t / 1e9}
    # binary-codebook layer of the same planes (c = 7132, the 7B configuration: 13-bit
    # indices): the encoder once, then the LUT application over 32 copies (> L2)
    try:
        t0 = time.perf_counter()
        Bc = rbw.btc_encode(Lp, 7132, iters=10, stream=stream)
        torch.cuda.synchronize()
        t_enc = time.perf_counter() - t0
        bcs = [Bc] + [rbw.BtcLayer(N_OUT, K_IN, K_PLANES, 7132, Lp.g16, Lp.h16, dev) for _ in range(31)]
        for C in bcs[1:]:
            C.codebooks.copy_(Bc.codebooks)
            C.indices.copy_(Bc.indices)
        Xb = torch.from_numpy(synth.activations(1, K_IN, seed=5).view(np.int16)).to(dev)
        Yb = torch.empty(1, N_OUT, dtype=torch.float32, device=dev)
        wsb = rbw.workspace(int(rbw.lib().rb_btc_gemv_workspace_bytes(N_OUT, K_IN)), dev)
        itb = iter(range(10 ** 9))
        t = time_graph_calls(torch, lambda: rbw.btc_gemv(bcs[next(itb) % len(bcs)], Xb, Y=Yb, ws=wsb,
                                                         flags=rbw.RB_LAUNCH_PDL, stream=stream), 64, stream)
        out["btc_gemv_M1_c7132"] = {"us": t * 1e6, "index_GBps": Bc.index_bytes() / t / 1e9,
                                    "bits_per_weight": Bc.index_bits / 16, "index_bytes": Bc.index_bytes(),
                                    "codebook_sizes": [int(Bc.sizes[i, 0].item()) for i in range(K_PLANES)],
                                    "encode_ms_10_rounds": t_enc * 1e3}
        # the same 32 layers in one rb_btc_gemv_batch call (one launch pair)
        Ybs = [torch.empty(1, N_OUT, dtype=torch.float32, device=dev) for _ in bcs]
        wsbb = rbw.workspace(int(rbw.lib().rb_btc_gemv_batch_workspace_bytes(N_OUT, K_IN, len(bcs))), dev)
        t = time_graph_calls(torch, lambda: rbw.btc_gemv_batch(bcs, [Xb] * len(bcs), Ybs, ws=wsbb,
                                                               flags=rbw.RB_LAUNCH_PDL, stream=stream), 8,
                             stream) / len(bcs)
        out["btc_gemv_batch32_M1_c7132"] = {"us_per_layer": t * 1e6, "index_GBps": Bc.index_bytes() / t / 1e9}
        del bcs, Bc
    except rbw.RbError as e:
        out["btc_gemv_M1_c7132"] = {"unavailable": str(e)}
    # coupled-training gradients of one layer at M = 2048 tokens: G = dY^T X on tcgen05 plus dg, dh
    try:
        Mt = 2048
        Xt = torch.from_numpy(synth.activations(Mt, K_IN, seed=21).view(np.int16)).to(dev)
        dYt = torch.from_numpy(synth.activations(Mt, N_OUT, seed=22).view(np.int16)).to(dev)
        dWt = torch.empty(N_OUT, K_IN, dtype=torch.float32, device=dev)
        dgt = torch.empty(K_PLANES, N_OUT, dtype=torch.float32, device=dev)
        dht = torch.empty(K_PLANES, K_IN, dtype=torch.float32, device=dev)
        wsg = rbw.workspace(int(rbw.lib().rb_qat_backward_workspace_bytes(N_OUT, K_IN, K_PLANES)), dev)
        t = time_events(torch, lambda: rbw.qat_backward(Lp, g, h, Xt, dYt, dW=dWt, dg=dgt, dh=dht, ws=wsg,
                                                        stream=stream), 10, stream)
        fl = 2.0 * Mt * N_OUT * K_IN
        out["qat_backward_M2048"] = {"us": t * 1e6, "G_TFLOPs": fl / t / 1e12, "flops": fl,
                                     "frac_of_bf16_peak": fl / t / 1e12 / bf16_peak}
        # the matching forward: planes derived from fp32 W (pack kernel), then the tcgen05 GEMM with fp32 g
        Yt = torch.empty(Mt, N_OUT, dtype=torch.float32, device=dev)
        wsf = rbw.workspace(rbw.qat_forward_workspace_bytes(N_OUT, K_IN, K_PLANES, Mt), dev)
        t = time_events(torch, lambda: rbw.qat_forward(W, g, h, K_PLANES, Xt, Y=Yt, ws=wsf, stream=stream),
                        10, stream)
        fl = 2.0 * K_PLANES * Mt * N_OUT * K_IN
        out["qat_forward_M2048"] = {"us": t * 1e6, "TFLOPs": fl / t / 1e12, "flops": fl,
                                    "frac_of_bf16_peak": fl / t / 1e12 / bf16_peak}
        del Xt, dYt, dWt, wsg, Yt, wsf
    except rbw.RbError as e:
        out["qat_backward_M2048"] = {"unavailable": str(e)}
    # rb_gemm at M = 2048 on the prefill shape
    try:
        X = torch.from_numpy(synth.activations(2048, K_IN, seed=7).view(np.int16)).to(dev)
        Lg = rbw.PackedLayer(N_OUT, K_IN, K_PLANES, dev)
        Lg.planes.copy_(Lp.planes)
        Lg.g16.copy_(Lp.g16)
        Lg.h16.copy_(Lp.h16)
        Y = torch.empty(2048, N_OUT, dtype=torch.float32, device=dev)
        ws = rbw.workspace(rbw.gemm_workspace_bytes(N_OUT, K_IN, K_PLANES, 2048), dev)
        t = time_events(torch, lambda: rbw.gemm(Lg, X, Y=Y, ws=ws, stream=stream), 10, stream)
        fl = 2.0 * 2048 * N_OUT * K_IN * K_PLANES
        out["gemm_M2048"] = {"us": t * 1e6, "TFLOPs": fl / t / 1e12, "frac_of_bf16_peak": fl / t / 1e12 / bf16_peak,
                             "flops": fl}
    except rbw.RbError as e:
        out["gemm_M2048"] = {"unavailable": str(e)}
    # decode on the 7B MLP trio (gate/up 11008 x 4096, down 4096 x 11008, k = 2, M = 1 and 8) and
    # the 28672 x 8192 layer (k = 1 and 2, M = 1, 16, 64): rb_gemv_batch over copies of each
    # layer that together exceed 3 x L2, so every application streams its planes from HBM
    def layer_copies(layer, k, min_bytes=400e6):
        Wl = torch.from_numpy(synth.weights(layer)).to(dev)
        gl, hl = rbw.svid_greedy(Wl, k, iters=20)
        base = rbw.pack(Wl, gl, hl, k)
        del Wl
        n = max(2, int(math.ceil(min_bytes / base.packed_bytes())))
        out_l = [base]
        for _ in range(n - 1):
            Lc = rbw.PackedLayer(base.n_out, base.k_in, k, dev)
            Lc.planes.copy_(base.planes)
            Lc.g16.copy_(base.g16)
            Lc.h16.copy_(base.h16)
            out_l.append(Lc)
        return out_l

    def batch_time(ls, M, seed):
        X = torch.from_numpy(synth.activations(M, ls[0].k_in, seed=seed).view(np.int16)).to(dev)
        Ys = [torch.empty(M, ls[0].n_out, dtype=torch.float32, device=dev) for _ in ls]
        return time_graph_calls(torch, lambda: rbw.gemv_batch(ls, [X] * len(ls), Ys, stream=stream), 5,
                                stream) / len(ls)

    wl3 = synth.workload("mlp_trio_7b_k2")
    trio = {layer.name: layer_copies(layer, K_PLANES) for layer in wl3.layers}
    for M in (1, 8):
        ts = {name: batch_time(ls, M, 250 + M) for name, ls in trio.items()}
        pb = sum(ls[0].packed_bytes() for ls in trio.values())
        tt = sum(ts.values())
        out["mlp_trio_7b_M%d" % M] = {"us_per_trio": tt * 1e6, "trio_tokens_per_s": M / tt,
                                      "packed_GBps": pb / tt / 1e9,
                                      "us_per_layer": {n: t * 1e6 for n, t in ts.items()}}
    del trio
    wl4 = synth.workload("mlp_28672x8192")
    for k in (1, 2):
        ls = layer_copies(wl4.layers[0], k)
        for M in (1, 16, 64):
            t = batch_time(ls, M, 350 + M)
            out["mlp_28672x8192_k%d_M%d" % (k, M)] = {
                "us_per_layer": t * 1e6, "packed_GBps": ls[0].packed_bytes() / t / 1e9, "tokens_per_s": M / t,
                "TFLOPs": 2.0 * M * ls[0].n_out * ls[0].k_in * k / t / 1e12}
        del ls
    # rb_gemm on the prefill workload's up (14336 x 4096) and down (4096 x 14336) layers,
    # Laplace(0, 0.01) weights, activations with 1% heavy columns, M = 512 and 2048
    wl5 = synth.workload("prefill_14336x4096_k2")
    for layer in wl5.layers:
        N5, K5 = layer.n_out, layer.k_in
        W5 = torch.from_numpy(synth.weights(layer)).to(dev)
        g5, h5 = rbw.svid_greedy(W5, K_PLANES, iters=20)
        L5 = rbw.pack(W5, g5, h5, K_PLANES)
        del W5
        for M in (512, 2048):
            X = torch.from_numpy(synth.activations_for(wl5, M, K5).view(np.int16)).to(dev)
            Y = torch.empty(M, N5, dtype=torch.float32, device=dev)
            ws = rbw.workspace(rbw.gemm_workspace_bytes(N5, K5, K_PLANES, M), dev)
            t = time_events(torch, lambda: rbw.gemm(L5, X, Y=Y, ws=ws, stream=stream), 10, stream)
            fl = 2.0 * M * N5 * K5 * K_PLANES
            out["gemm_%s_%dx%d_M%d" % (layer.name, N5, K5, M)] = {
                "us": t * 1e6, "TFLOPs": fl / t / 1e12, "frac_of_bf16_peak": fl / t / 1e12 / bf16_peak}
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["rbw", "reference"], default="rbw")
    ap.add_argument("--quick", action="store_true", help="skip the extra per-row timings")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--mode", choices=["full", "gemv-kernel", "gemv-batch-kernel", "pack-kernel", "gemm-kernel",
                                       "grad-kernel", "qat-forward-kernel", "btc-kernel", "svid-kernel", "transpose-kernel",
                                       "rowmajor-kernel"],
                    default="full",
                    help="kernel-only modes run one kernel a few times (used for ncu captures)")
    ap.add_argument("--launches", type=int, default=20)
    ap.add_argument("--M", type=int, default=1)
    args = ap.parse_args(argv)
    dist = Dist()
    if args.impl == "reference":
        return run_reference(args, dist)
    if args.mode != "full":
        return run_kernel_mode(args)
    return run_rbw(args, dist)


def run_kernel_mode(args):
    """Launch one kernel `--launches` times on the workload layer (distinct buffers), no graph."""
    import torch
    from residual_binarized_weight_b200 import rbw, synth
    dev = torch.device("cuda", 0)
    wl = synth.workload(WORKLOAD)
    W = torch.from_numpy(synth.weights(wl.layers[0])).to(dev)
    g, h = rbw.svid_greedy(W, K_PLANES, iters=20)
    base = rbw.pack(W, g, h, K_PLANES)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    if args.mode == "pack-kernel":
        for _ in range(args.launches):
            rbw.pack(W, g, h, K_PLANES, out=base)
    elif args.mode == "grad-kernel":                 # rb_qat_backward at M tokens (default 2048)
        M = args.M if args.M > 1 else 2048
        X = torch.from_numpy(synth.activations(M, K_IN, seed=21).view(np.int16)).to(dev)
        dY = torch.from_numpy(synth.activations(M, N_OUT, seed=22).view(np.int16)).to(dev)
        for _ in range(args.launches):
            rbw.qat_backward(base, g, h, X, dY)
    elif args.mode == "qat-forward-kernel":          # rb_qat_forward at M tokens (default 2048)
        M = args.M if args.M > 1 else 2048
        X = torch.from_numpy(synth.activations(M, K_IN, seed=21).view(np.int16)).to(dev)
        for _ in range(args.launches):
            rbw.qat_forward(W, g, h, K_PLANES, X)
    elif args.mode == "btc-kernel":                  # rb_btc_gemv at M = 1 on the c = 7132 codebook layer
        Bc = rbw.btc_encode(base, 7132, iters=2)
        Xb = torch.from_numpy(synth.activations(1, K_IN, seed=5).view(np.int16)).to(dev)
        for _ in range(args.launches):
            rbw.btc_gemv(Bc, Xb)
    elif args.mode == "svid-kernel":                 # greedy SVID, 2 power iterations per plane
        for _ in range(args.launches):
            rbw.svid_greedy(W, K_PLANES, iters=2)
    elif args.mode == "transpose-kernel":
        t = rbw.transpose(base)
        for _ in range(args.launches):
            rbw.transpose(base, out=t)
    elif args.mode == "rowmajor-kernel":
        rm = rbw.planes_to_rowmajor(base)
        L2 = rbw.PackedLayer(N_OUT, K_IN, K_PLANES, dev)
        for _ in range(args.launches):
            rbw.planes_from_rowmajor(rm, N_OUT, K_IN, K_PLANES, out=L2)
    else:
        nl = LAYERS                         # distinct layers: 96 x 4.2 MB of planes, larger than L2
        layers = []
        for _ in range(nl):
            L = rbw.PackedLayer(N_OUT, K_IN, K_PLANES, dev)
            L.planes.copy_(base.planes)
            L.g16.copy_(base.g16)
            L.h16.copy_(base.h16)
            layers.append(L)
        M = args.M
        X = torch.from_numpy(synth.activations(M, K_IN, seed=M).view(np.int16)).to(dev)
        Y = torch.empty(M, N_OUT, dtype=torch.float32, device=dev)
        if args.mode == "gemv-kernel":
            ws = rbw.workspace(rbw.gemv_workspace_bytes(N_OUT, K_IN, K_PLANES, M), dev)
            for j in range(args.launches):
                rbw.gemv(layers[j % nl], X, Y=Y, ws=ws)
        elif args.mode == "gemv-batch-kernel":
            Ys = [torch.empty(M, N_OUT, dtype=torch.float32, device=dev) for _ in range(nl)]
            for j in range(args.launches):
                rbw.gemv_batch(layers, [X] * nl, Ys)
        else:
            ws = rbw.workspace(rbw.gemm_workspace_bytes(N_OUT, K_IN, K_PLANES, M), dev)
            for j in range(args.launches):
                rbw.gemm(layers[j % nl], X, Y=Y, ws=ws)
    torch.cuda.synchronize()
    print(json.dumps({"mode": args.mode, "launches": args.launches, "M": args.M,
                      "wall_s": time.perf_counter() - t0}), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
