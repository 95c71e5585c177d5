#!/usr/bin/env python
"""Benchmark of the MatMul-free block forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mmf|reference] [--workload NAME]

One step = one pass of the whole hot path over one batch of synthetic input:
for the default workload, the 370M-shaped stack prefill (24 MatMul-free blocks,
d=1024, GLU inner 2816, batch 8 x 2048 tokens, bf16): per block the fused
RMSNorm+absmax quantisation, the ternary contractions (f|c|g, o, gate|up, down),
the MLGRU scan and the GLU, with the recurrent state reset to zero.

Prints ONE JSON line (rank 0). `value` is whole-job tokens/s with the inputs
already resident in HBM; `e2e` is the same metric through the public API with
the step's input copied from pinned host memory and its output copied back
inside the timed region. Under torchrun each rank runs an independent replica
(sequences are independent: no collective on the data path) and the time is
the max over ranks.

`--impl reference` times the CPU oracle on a bounded sample of the same
workload on this host's cores (the baseline arm; rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "BitLinear GB/s & int8 TOPS vs roofline; MMfree block tokens/sec on 1 B200"
L2_BYTES = 126 * 1024 * 1024
# int8 dense tensor peak = measured bf16 peak x (4.5 / 2.25), the nominal int8:bf16 ratio
INT8_OVER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["mmf", "reference"], default="mmf")
    ap.add_argument("--workload", choices=["stack370m", "bitlinear", "scan", "gemv", "decode1p3b", "decode2p7b",
                                           "model2p7b"],
                    default="stack370m",
                    help="stack370m: the 370M-shaped 24-block prefill (default); bitlinear: one prefill "
                         "BitLinear of the 370M gate|up shape (16384 tokens, 1024 -> 5632); scan: one MLGRU "
                         "scan of the 370M layer shape (8 x 2048 tokens, d=1024); gemv: the decode BitLinear "
                         "sweep (2048->2048, 2048->5632, 5632->2048 at 1/4/16 tokens) over a weight pool > L2; "
                         "decode1p3b / decode2p7b: the 1.3B / 2.7B-shaped stacks, prompt prefill then decode "
                         "steps (output fed back, state carried), each step one CUDA graph; model2p7b: greedy "
                         "generation through the 2.7B-shaped model (embedding, 32 blocks, 32000-entry head, "
                         "argmax), one CUDA graph per token")
    ap.add_argument("--batch", type=int, default=None, help="decode2p7b: concurrent sequences (1, 8 or 64)")
    ap.add_argument("--decode-steps", type=int, default=None,
                    help="decode1p3b/decode2p7b: timed decode steps (default: the workload's own count)")
    ap.add_argument("--packed-only", action="store_true",
                    help="bitlinear: contract from the 2-bit codes only (no one-byte copy of the codes)")
    ap.add_argument("--layers", type=int, default=None,
                    help="stack370m: number of blocks (default 24; fewer for short profiler captures)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) pass")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip timing the CPU oracle")
    ap.add_argument("--backward", action="store_true",
                    help="scan: the scan's backward (training gradients) instead of its forward")
    ap.add_argument("--gnorm", action="store_true",
                    help="scan / stack370m: the g_norm output gate (RMSNorm of the state fused with a swish gate)")
    ap.add_argument("--no-sub", action="store_true",
                    help="stack370m: skip the decode-step and GEMV-sweep sub-measurements")
    return ap.parse_args(argv)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def int8_peak(peaks, peak_kind, clk):
    """Dense int8 tensor peak for a contraction timed in this run: 2 x the bf16 burst figure, or 2 x the
    sustained one when the sampled clocks show power capping or SM clocks well below their maximum."""
    burst = peaks["bf16_tflops"] * INT8_OVER_BF16
    sustained = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * INT8_OVER_BF16
    sm, mx = (clk or {}).get("sm_mhz"), (clk or {}).get("sm_max_mhz")
    capped = "sw_power_cap" in (clk or {}).get("reasons", []) or bool(sm and mx and sm < 0.9 * mx)
    kind = "sustained" if capped else "burst"
    return (sustained if capped else burst), burst, sustained, \
        f"{peak_kind}: bf16 {kind} x {INT8_OVER_BF16} (int8 dense : bf16 dense nominal)"


# ----------------------------------------------------------------------------- distributed plumbing

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(world, backend="nccl"):
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """Max of a per-rank value over all ranks (the whole job is as slow as its slowest rank)."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class L2Flush:
    """Between timed steps: write a buffer twice the size of L2 (the flush), then read a second one, so
    that the timed kernels start with an L2 of clean lines instead of paying for the write-back of the
    flush's dirty lines."""

    def __init__(self, dev):
        self.w = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.sink)

    NOTE = "flushed between timed steps (252 MB write, then 252 MB read, outside the step events)"


def whole_job_rate(world: int, units_per_rank_step: float, steps: int, max_total_ms: float) -> float:
    """Units per second of the whole job: every rank's units over the slowest rank's time."""
    return world * units_per_rank_step * steps / (max_total_ms / 1e3)


# ----------------------------------------------------------------------------- clocks

def wait_event(ev) -> None:
    """Wait for a CUDA event by polling with short sleeps, so the clock-sampling thread keeps running."""
    while not ev.query():
        time.sleep(0.0005)


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled during the timed region: read-only NVML queries
    every 10 ms from a thread, or nvidia-smi every 50 ms when NVML is not importable."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40}

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None
        self.thread = None
        self.rows = []

    def _nvml_handle(self, nvml):
        try:   # match the CUDA device by UUID: NVML indices ignore CUDA_VISIBLE_DEVICES
            uuid = str(torch.cuda.get_device_properties(self.idx).uuid)
            return nvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return nvml.nvmlDeviceGetHandleByIndex(self.idx)

    def start(self):
        try:
            import threading
            import pynvml as nvml
            nvml.nvmlInit()
            h = self._nvml_handle(nvml)
            reasons_fn = getattr(nvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nvml.nvmlDeviceGetCurrentClocksThrottleReasons
            mx = nvml.nvmlDeviceGetMaxClockInfo(h, nvml.NVML_CLOCK_SM)
            self.stop_flag = threading.Event()

            def run():
                while not self.stop_flag.is_set():
                    self.rows.append((nvml.nvmlDeviceGetClockInfo(h, nvml.NVML_CLOCK_SM), mx, reasons_fn(h)))
                    self.stop_flag.wait(0.01)
            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    @staticmethod
    def _summary(sm, mx, reasons, n, source):
        loaded = [v for v in sm if mx and v > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": n, "source": source}

    def stop(self) -> dict:
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            rows = self.rows
            if not rows:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
            reasons = sorted({k for _, _, r in rows for k, bit in self.REASON_BITS.items() if r & bit})
            return self._summary([float(r[0]) for r in rows], [float(r[1]) for r in rows], reasons, len(rows),
                                 "nvml, 10 ms")
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return self._summary(sm, mx, reasons, len(rows), "nvidia-smi, 50 ms")


# ----------------------------------------------------------------------------- workload

# DRAM bytes (read + write) per launch of the dominant kernel, measured by an ncu capture of the same
# kernel (mean over the four contraction launches of one 370M block, one-byte weight codes). Reported as
# the `traffic` of the headline line with the capture named in `traffic_source`; None elsewhere.
STACK370M_CONTRACTION_TRAFFIC = 69.53e6
STACK370M_TRAFFIC_SOURCE = "ncu capture, tgemm_tc at the four 370M block shapes (dram__bytes read + write)"


def stack_workload(layers=None):
    """The 370M-shaped stack; `layers` overrides the block count (a one-block run has the same
    kernel shapes, for short profiler captures), and the workload name then says so."""
    w = synth.STACK_370M
    if layers is not None and layers != w.layers:
        w = dataclasses.replace(w, layers=layers, name=f"{w.name}_layers{layers}")
    return w


def gemm_ops_per_step(w) -> float:
    """Algorithmic int8 ops (2 per weight per token) of one stack pass: 2*M*(3dd + dd + 2Id + dI) * L."""
    M = w.batch * w.seq
    per_layer = 3 * w.d * w.d + w.d * w.d + 2 * w.inner * w.d + w.d * w.inner
    return 2.0 * M * per_layer * w.layers


def build_stack(w, device, gnorm: bool = False):
    """The workload's blocks (weights from the seeded recipe); gnorm: with a seeded g_norm gain each."""
    import ternary_weight_matmul_fusedbitlinear_b200 as mmf
    shapes = {"f": (w.d, w.d), "c": (w.d, w.d), "g": (w.d, w.d), "o": (w.d, w.d),
              "gate": (w.inner, w.d), "up": (w.inner, w.d), "down": (w.d, w.inner)}
    blocks = []
    for layer in range(w.layers):
        lins = {}
        for i, name in enumerate(synth.PROJ_NAMES):
            W = synth.latent_weight(synth.sub_seed(w.seed, layer, i), *shapes[name], device=device)
            lins[name] = mmf.quantize_weights(W)
            del W
        gain = synth.gains(synth.sub_seed(w.seed, layer, 7), w.d, device=str(device)) if gnorm else None
        blocks.append(mmf.Block(lins, gain))
    torch.cuda.synchronize()
    return blocks


# ----------------------------------------------------------------------------- oracle timing

def oracle_sample(w, tokens: int, nseq: int = 1):
    """Time the CPU oracle on one block over `tokens` tokens of `nseq` sequences; returns (seconds, threads)."""
    import numpy as np
    from threadpoolctl import threadpool_info

    import oracle as O
    shapes = {"f": (w.d, w.d), "c": (w.d, w.d), "g": (w.d, w.d), "o": (w.d, w.d),
              "gate": (w.inner, w.d), "up": (w.inner, w.d), "down": (w.d, w.inner)}
    lat = {n: synth.latent_weight(synth.sub_seed(w.seed, 0, i), *shapes[n]).numpy()
           for i, n in enumerate(synth.PROJ_NAMES)}
    blk = O.make_block(lat)
    x = synth.activations(w.seed + synth.ACT_SEED_OFFSET, nseq * tokens, w.d, torch.bfloat16)
    x = x.float().numpy().astype(np.float64).reshape(nseq, tokens, w.d)
    t0 = time.perf_counter()
    O.block_forward(x, blk, np.zeros((nseq, w.d)), w.dtype)
    dt = time.perf_counter() - t0
    threads = max([int(i.get("num_threads", 1)) for i in threadpool_info()] + [1])
    return dt, threads


def cpu_baseline_entry(w, tokens: int):
    # one block over the whole batch (several seconds of CPU work), extrapolated to the stack
    dt, threads = oracle_sample(w, tokens, w.batch)
    tps = w.batch * tokens / (dt * w.layers)
    return {"value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"1 of {w.layers} blocks on {w.batch} x {tokens} tokens (the whole batch, "
                      f"{dt:.2f} s), extrapolated x{w.layers} blocks",
            "host_cores_available": len(os.sched_getaffinity(0))}


# ----------------------------------------------------------------------------- arms

def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    w = stack_workload()
    tokens = 512
    times = []
    threads = 1
    for i in range(args.warmup + args.steps):
        dt, threads = oracle_sample(w, tokens)
        if i >= args.warmup:
            times.append(dt)
    mean = sum(times) / len(times)
    value = tokens / (mean * w.layers)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "d": w.d, "inner": w.inner, "layers": w.layers, "batch": w.batch,
                   "seq": w.seq, "global_batch": w.batch, "seq_len": w.seq, "parallelism": "none (CPU oracle)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"each step: 1 of {w.layers} blocks on {tokens} tokens of 1 sequence, "
                                   f"extrapolated x{w.layers} blocks"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_mmf(args):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist_init(world)
    import ternary_weight_matmul_fusedbitlinear_b200 as mmf
    mmf.load()
    dev = torch.device("cuda", local)
    w = stack_workload(args.layers)
    peaks, peak_kind = load_peaks()

    blocks = build_stack(w, dev, gnorm=args.gnorm)
    st = mmf.State(w.layers, w.batch, w.d)
    x_host = synth.activations(w.seed + synth.ACT_SEED_OFFSET + rank, w.batch * w.seq, w.d,
                               torch.bfloat16).reshape(w.batch, w.seq, w.d)
    x = x_host.to(dev)
    y = torch.empty_like(x)
    ws = torch.empty(mmf.stack_ws_size(blocks, w.batch, w.seq), dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def step(xin, yout):
        st.reset()
        mmf.stack_forward(blocks, st, xin, ws=ws, out=yout)

    for _ in range(args.warmup):
        step(x, y)
    mmf.check()

    def timed_steps(profile: bool):
        """args.steps steps between CUDA events, L2 flushed before each (outside the events); with
        `profile` the library also brackets every kernel with events (per-kernel times), which breaks
        the programmatic launch overlap between kernels, so the headline pass runs without it."""
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        mmf.prof_reset()
        mmf.prof_enable(profile)
        barrier(world)
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush()
            starts[i].record(stream)
            step(x, y)
            ends[i].record(stream)
        wait_event(ends[-1])
        torch.cuda.synchronize()
        barrier(world)
        mmf.prof_enable(False)
        mmf.check()
        return [s.elapsed_time(e) for s, e in zip(starts, ends)], (mmf.prof_collect() if profile else {})

    # ------------------------------------------------------------ timed region (inputs resident)
    clocks = ClockSampler(local)
    clocks.start()
    step_ms, _ = timed_steps(False)
    clk = clocks.stop()
    # the same steps again with per-kernel events: kernel durations for the roofline
    prof_step_ms, prof = timed_steps(True)
    total_ms = max_over_ranks(sum(step_ms), world)
    ms_per_step = total_ms / args.steps
    tokens_per_step = w.batch * w.seq
    value = whole_job_rate(world, tokens_per_step, args.steps, total_ms)

    # dominant kernel: the ternary contraction (tensor-bound)
    gemm_names = [k for k in prof if k.startswith("tgemm")]
    gemm_ms = sum(prof[k][1] for k in gemm_names)
    gemm_launches = sum(prof[k][0] for k in gemm_names)
    ops = gemm_ops_per_step(w) * args.steps
    achieved = ops / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else 0.0
    peak, peak_burst, peak_sus, peak_src = int8_peak(peaks, peak_kind, clk)
    launches = sum(v[0] for v in prof.values())
    byte_codes = os.environ.get("MMF_PREFILL_UNPACKED", "1") != "0"
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "frac_of_sustained": achieved / peak_sus, "peak_sustained": peak_sus,
                "traffic": STACK370M_CONTRACTION_TRAFFIC if byte_codes else None,
                "traffic_note": "DRAM bytes per contraction launch, mean of one block's four",
                "traffic_source": STACK370M_TRAFFIC_SOURCE,
                "kernel": ",".join(gemm_names), "launches": gemm_launches,
                "share_of_step": gemm_ms / sum(prof_step_ms) if prof_step_ms else None,
                "kernel_times": "CUDA events around each kernel in a second pass of the same steps",
                "peak_source": peak_src,
                "per_kernel_ms": {k: round(v[1] / args.steps, 4) for k, v in prof.items()}}
    # the other kernels of the step against HBM, from the same per-kernel times
    M = w.batch * w.seq
    hbm = peaks["hbm_gbs"]
    others = {}
    if "mlgru_scan" in prof:
        scan_ms = prof["mlgru_scan"][1] / prof["mlgru_scan"][0]
        gbs = 8.0 * M * w.d / (scan_ms / 1e3) / 1e9   # 6 B read + 2 B written per channel-step (bf16)
        others["mlgru_scan"] = {"us_per_layer": round(scan_ms * 1e3, 2), "GBps": round(gbs, 1),
                                "frac": round(gbs / hbm, 4), "bytes_per_layer": 8.0 * M * w.d}
    if "mlgru_scan_gnorm" in prof:   # scan + the row kernel that forms o' and quantises it
        g_ms = prof["mlgru_scan_gnorm"][1] / prof["mlgru_scan_gnorm"][0]
        gbs = 8.0 * M * w.d / (g_ms / 1e3) / 1e9
        others["mlgru_scan_gnorm"] = {"us_per_layer": round(g_ms * 1e3, 2), "GBps": round(gbs, 1),
                                      "frac": round(gbs / hbm, 4), "bytes_per_layer": 8.0 * M * w.d,
                                      "note": "both launches; the o projection's quantiser is folded in"}
    if "rmsnorm_quant" in prof:
        q_ms = prof["rmsnorm_quant"][1] / args.steps
        qbytes = 3.0 * M * (3 * w.d + w.inner) * w.layers   # 2 B read + 1 B written per element (bf16)
        gbs = qbytes / (q_ms / 1e3) / 1e9
        others["rmsnorm_quant"] = {"ms_per_step": round(q_ms, 4), "GBps": round(gbs, 1), "frac": round(gbs / hbm, 4),
                                   "bytes_per_step": qbytes}

    # ------------------------------------------------------------ end to end through the public API
    # Every step's input is copied from pinned host memory and its output copied
    # back, all inside the timed region; the copies run on their own streams so
    # step i+1's upload and step i-1's download overlap step i's kernels
    # (double-buffered device input/output).
    e2e = None
    if not args.no_e2e:
        x_pin = [x_host.pin_memory(), x_host.clone().pin_memory()]
        y_pin = [torch.empty_like(x_host).pin_memory() for _ in range(2)]
        x_d = [x, torch.empty_like(x)]
        y_d = [y, torch.empty_like(y)]
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        up = [torch.cuda.Event() for _ in range(args.steps)]
        done = [torch.cuda.Event() for _ in range(args.steps)]
        down = [torch.cuda.Event() for _ in range(args.steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        h2d.wait_stream(stream)
        d2h.wait_stream(stream)
        with torch.cuda.stream(h2d):
            x_d[0].copy_(x_pin[0], non_blocking=True)
            up[0].record(h2d)
        for i in range(args.steps):
            b = i % 2
            if i + 1 < args.steps:
                with torch.cuda.stream(h2d):
                    if i >= 1:
                        h2d.wait_event(done[i - 1])        # step i-1 has finished reading x_d[(i+1)%2]
                    x_d[(i + 1) % 2].copy_(x_pin[(i + 1) % 2], non_blocking=True)
                    up[i + 1].record(h2d)
            stream.wait_event(up[i])
            if i >= 2:
                stream.wait_event(down[i - 2])            # y_d[b] has been copied out
            step(x_d[b], y_d[b])
            done[i].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(done[i])
                y_pin[b].copy_(y_d[b], non_blocking=True)
                down[i].record(d2h)
        stream.wait_event(down[args.steps - 1])
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(t0.elapsed_time(t1), world)
        nbytes = x_host.numel() * x_host.element_size()
        e2e = {"value": whole_job_rate(world, tokens_per_step, args.steps, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
               "note": "copies on side streams overlap neighbouring steps; all inside the timed region"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_entry(w, 2048)

    # the metric's other clauses, each its own timed measurement after the headline: the decode
    # BitLinear GEMV sweep and a 2.7B-shaped decode step (HBM-bound), on every rank like the headline
    sub = None
    if not args.no_sub:
        del blocks, ws, flush
        torch.cuda.empty_cache()
        sub = {"kernels_in_step": others}
        w27 = synth.STACK_2P7B
        blocks27 = build_stack(w27, dev)
        d27 = measure_decode(mmf, w27, 1, 128, 3, dev, peaks, prompt=False, blocks=blocks27)
        sub["decode_2p7b_b1"] = {k: d27[k] for k in ("ms_per_step", "tokens_per_s", "GBps", "frac", "bytes_per_step",
                                                      "launches_per_step", "decode_steps", "clocks")}
        m27 = measure_model_decode(mmf, w27, 1, 128, 3, dev, peaks, blocks=blocks27)
        sub["model_2p7b_greedy_b1"] = {k: m27[k] for k in ("ms_per_step", "tokens_per_s", "GBps", "frac",
                                                            "bytes_per_step", "launches_per_step", "vocab")}
        del blocks27
        torch.cuda.empty_cache()
        sub["gemv_sweep"] = measure_gemv(mmf, dev, 2, 3, peaks)
        for gn in (False, True):
            m = measure_scan(mmf, dev, 10, 3, gn)
            m["frac"] = round(m["GBps"] / peaks["hbm_gbs"], 4)
            sub["scan_gnorm" if gn else "scan"] = m

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name + ("_gnorm" if args.gnorm else ""), "d": w.d, "inner": w.inner,
                       "layers": w.layers, "batch": w.batch,
                       "seq": w.seq, "global_batch": w.batch * world, "seq_len": w.seq,
                       "parallelism": f"replicas x{world} (independent sequences)",
                       "l2": L2Flush.NOTE},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(launches), "clocks": clk, "sub": sub,
        }
        print(json.dumps(line), flush=True)
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_bitlinear(args):
    """One prefill BitLinear per step: 16384 tokens x (1024 -> 5632), bf16 (the 370M GLU gate|up shape)."""
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist_init(world)
    import ternary_weight_matmul_fusedbitlinear_b200 as mmf
    dev = torch.device("cuda", local)
    M, K, N = 16384, 1024, 5632
    peaks, peak_kind = load_peaks()
    lin = mmf.quantize_weights(synth.latent_weight(synth.sub_seed(1002, 0, synth.PROJ_GATE), N, K, device=dev))
    if not args.packed_only:   # one byte per weight as well: the prefill contraction loads it directly
        lin = mmf.unpack_codes(lin)
    x = synth.activations(1002 + rank, M, K, torch.bfloat16, device=dev)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(mmf.api.L.load().mmf_bitlinear_ws_size(M, K), dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        mmf.bitlinear(lin, x, ws=ws)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    def timed_steps(profile: bool):
        # headline pass without per-kernel events; a second pass with them gives the kernel times
        mmf.prof_reset()
        mmf.prof_enable(profile)
        barrier(world)
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush()
            starts[i].record(stream)
            mmf.bitlinear(lin, x, ws=ws)
            ends[i].record(stream)
        wait_event(ends[-1])
        torch.cuda.synchronize()
        mmf.prof_enable(False)
        return sum(s.elapsed_time(e) for s, e in zip(starts, ends)), (mmf.prof_collect() if profile else {})

    clocks = ClockSampler(local)
    clocks.start()
    step_total, _ = timed_steps(False)
    clk = clocks.stop()
    _, prof = timed_steps(True)
    total_ms = max_over_ranks(step_total, world)
    gemm = [k for k in prof if k.startswith("tgemm")]
    gemm_ms = sum(prof[k][1] for k in gemm)
    ops = 2.0 * M * N * K
    achieved = ops * args.steps / (gemm_ms / 1e3) / 1e12
    peak = peaks["bf16_tflops"] * INT8_OVER_BF16
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": world * M * args.steps / (total_ms / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"bitlinear_prefill_m{M}_k{K}_n{N}_bf16", "l2": L2Flush.NOTE,
                       "weight_codes": "2-bit packed only" if args.packed_only else "2-bit packed + one byte per weight"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None, "kernel": ",".join(gemm),
                         "peak_source": f"{peak_kind}: bf16 burst x {INT8_OVER_BF16}",
                         "per_kernel_ms": {k: round(v[1] / args.steps, 4) for k, v in prof.items()}},
            "cpu_baseline": None, "e2e": None, "gpu_launches": int(sum(v[0] for v in prof.values())),
            "clocks": clk}), flush=True)
    return 0


def measure_scan(mmf, dev, steps: int, warmup: int, gnorm: bool, flush=None) -> dict:
    """One MLGRU scan per step on the 370M layer shape (8 x 2048 tokens, d = 1024, bf16), L2 flushed
    between steps. Algorithmic bytes: 8 per channel-step (6 B of pre-activations read, 2 B of o'
    written) for either output gate; the g_norm path's own design also writes and reads v in fp32
    (16 B per channel-step in all)."""
    w = synth.STACK_370M
    B, T, d = w.batch, w.seq, w.d
    pre = synth.preacts(77, B, T, d, torch.bfloat16, scale=2.0, device=dev)
    h = torch.zeros(B, d, device=dev)
    gain = synth.gains(78, d, device=str(dev)) if gnorm else None
    flush = flush or L2Flush(dev)
    run = (lambda: mmf.mlgru_scan_gnorm(pre, h, gain)) if gnorm else (lambda: mmf.mlgru_scan(pre, h))
    key = "mlgru_scan_gnorm" if gnorm else "mlgru_scan"
    for _ in range(warmup):
        run()
    mmf.prof_reset()
    mmf.prof_enable(True)
    torch.cuda.synchronize()
    for _ in range(steps):
        flush()
        run()
    torch.cuda.synchronize()
    mmf.prof_enable(False)
    prof = mmf.prof_collect()
    ms = prof[key][1] / prof[key][0]
    nbytes = 8.0 * B * T * d
    gbs = nbytes / (ms / 1e3) / 1e9
    r = {"workload": f"mlgru_scan{'_gnorm' if gnorm else ''}_b{B}_t{T}_d{d}_bf16", "us": round(ms * 1e3, 2),
         "GBps": round(gbs, 1), "bytes": nbytes, "launches": (2 if gnorm else 1) * prof[key][0]}
    if gnorm:
        r["design_bytes"] = 16.0 * B * T * d
    return r


def measure_scan_backward(mmf, dev, steps: int, warmup: int) -> dict:
    """The scan's backward on the 370M layer shape (8 x 2048 tokens, d = 1024, bf16), L2 flushed between
    steps. Algorithmic bytes: 14 per channel-step (pre-activations 6 and dL/do' 2 read, the three
    gradients 6 written); the design also recomputes the forward states (6 B read, 4 B written) and
    reads them back (4 B): 28 B per channel-step."""
    w = synth.STACK_370M
    B, T, d = w.batch, w.seq, w.d
    pre = synth.preacts(77, B, T, d, torch.bfloat16, scale=2.0, device=dev)
    dout = synth.activations(79, B * T, d, torch.bfloat16, device=str(dev)).reshape(B, T, d)
    h0 = torch.zeros(B, d, device=dev)
    ws = torch.empty(mmf.load().mmf_mlgru_scan_backward_ws_size(B, T, d), dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    for _ in range(warmup):
        mmf.mlgru_scan_backward(pre, h0, dout, ws=ws)
    mmf.prof_reset()
    mmf.prof_enable(True)
    torch.cuda.synchronize()
    for _ in range(steps):
        flush()
        mmf.mlgru_scan_backward(pre, h0, dout, ws=ws)
    torch.cuda.synchronize()
    mmf.prof_enable(False)
    prof = mmf.prof_collect()
    key = "mlgru_scan_backward"
    ms = prof[key][1] / prof[key][0]
    nbytes = 14.0 * B * T * d
    gbs = nbytes / (ms / 1e3) / 1e9
    # a training step instead keeps the states of its forward (mmf_mlgru_scan_states): time that
    # forward and the backward given its states
    hsb = torch.empty(B, T, d, dtype=torch.float32, device=dev)
    hcur = torch.zeros(B, d, device=dev)
    lib = mmf.load()
    for _ in range(warmup):
        mmf.mlgru_scan_states(pre, hcur)
    _, hsb = mmf.mlgru_scan_states(pre, torch.zeros(B, d, device=dev))
    for _ in range(warmup):
        mmf.mlgru_scan_backward(pre, h0, dout, hs=hsb)
    mmf.prof_reset()
    mmf.prof_enable(True)
    torch.cuda.synchronize()
    for _ in range(steps):
        flush()
        mmf.mlgru_scan_states(pre, hcur)
        flush()
        mmf.mlgru_scan_backward(pre, h0, dout, hs=hsb)
    torch.cuda.synchronize()
    mmf.prof_enable(False)
    p2 = mmf.prof_collect()
    fwd_us = p2["mlgru_scan_states"][1] / p2["mlgru_scan_states"][0] * 1e3
    bwd_us = p2[key][1] / p2[key][0] * 1e3
    return {"workload": f"mlgru_scan_backward_b{B}_t{T}_d{d}_bf16", "us": round(ms * 1e3, 2), "GBps": round(gbs, 1),
            "bytes": nbytes, "design_bytes": 28.0 * B * T * d, "launches": 2 * prof[key][0],
            "with_stored_states": {"forward_states_us": round(fwd_us, 2), "backward_us": round(bwd_us, 2),
                                   "backward_GBps": round((14.0 + 4.0) * B * T * d / (bwd_us / 1e6) / 1e9, 1),
                                   "note": "backward reads the stored states (4 B per channel-step more)"}}


def run_scan(args):
    """One MLGRU scan per step on the 370M layer shape; GB/s = 8 bytes per channel-step (bf16)."""
    _, rank, local = dist_env()
    torch.cuda.set_device(local)
    import ternary_weight_matmul_fusedbitlinear_b200 as mmf
    dev = torch.device("cuda", local)
    peaks, peak_kind = load_peaks()
    m = (measure_scan_backward(mmf, dev, args.steps, args.warmup) if args.backward
         else measure_scan(mmf, dev, args.steps, args.warmup, args.gnorm))
    gbs, ms = m["GBps"], m["us"] / 1e3
    kernel = ("mlgru_scan_backward (forward states + reverse scan)" if args.backward
              else "mlgru_scan_gnorm (scan + row kernel)" if args.gnorm else "mlgru_scan")
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": {"workload": m["workload"], "l2": L2Flush.NOTE},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "traffic": None, "kernel": kernel,
                         "peak_source": peak_kind},
            "cpu_baseline": None, "e2e": None, "gpu_launches": m["launches"], "detail": m}), flush=True)
    return 0


def measure_gemv(mmf, dev, reps: int, warmup: int, peaks) -> dict:
    """Decode BitLinear sweep: per shape and token count, calls cycle through a pool of distinct packed
    matrices totalling more than 4x L2, replayed as one CUDA graph; GB/s = (N*K/4 + 4 + 2*M*K + 2*M*N)
    bytes per call / mean call time. The calls form a dependent chain on one stream."""
    rows = []
    for (K, N) in synth.GEMV_SWEEP_SHAPES:
        per = N * K // 4
        pool_n = max(8, int(4 * L2_BYTES // per) + 1)
        lins = [mmf.quantize_weights(synth.latent_weight(synth.GEMV_SWEEP_SEED * 4096 + i, N, K, device=dev))
                for i in range(pool_n)]
        for M in synth.GEMV_SWEEP_TOKENS:
            x = synth.activations(synth.GEMV_SWEEP_SEED + M, M, K, torch.bfloat16, outlier_p=synth.GEMV_OUTLIER_P,
                                  outlier_scale=synth.GEMV_OUTLIER_SCALE, device=dev)
            ws = torch.empty(mmf.api.L.load().mmf_bitlinear_ws_size(M, K), dtype=torch.uint8, device=dev)
            side = torch.cuda.Stream(dev)
            side.wait_stream(torch.cuda.current_stream(dev))
            with torch.cuda.stream(side):
                for lin in lins[:max(warmup, 3)]:
                    mmf.bitlinear(lin, x, ws=ws)
            torch.cuda.current_stream(dev).wait_stream(side)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()   # the whole pool in order: launch cost leaves the host
            with torch.cuda.graph(graph):
                for i in range(pool_n):
                    mmf.bitlinear(lins[i], x, ws=ws)
            graph.replay()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                graph.replay()
            e1.record()
            torch.cuda.synchronize()
            del graph
            us = e0.elapsed_time(e1) * 1e3 / (pool_n * reps)
            nbytes = per + 4 + 2 * M * K + 2 * M * N
            rows.append({"K": K, "N": N, "M": M, "us_per_call": round(us, 3),
                         "GBps": round(nbytes / (us * 1e-6) / 1e9, 1),
                         "frac": round(nbytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                         "TOPS": round(2.0 * M * N * K / (us * 1e-6) / 1e12, 3), "pool": pool_n})
            del ws
        del lins
        torch.cuda.empty_cache()
    mean = sum(r["GBps"] for r in rows) / len(rows)
    return {"mean_GBps": round(mean, 1), "best_GBps": max(r["GBps"] for r in rows),
            "frac_mean": round(mean / peaks["hbm_gbs"], 4), "shapes": rows,
            "note": "dependent chain of single calls (each waits for the previous one's output)"}


def run_gemv(args):
    _, rank, local = dist_env()
    torch.cuda.set_device(local)
    import ternary_weight_matmul_fusedbitlinear_b200 as mmf
    dev = torch.device("cuda", local)
    peaks, peak_kind = load_peaks()
    g = measure_gemv(mmf, dev, max(1, args.steps // 5), args.warmup, peaks)
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": g["mean_GBps"], "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "bitlinear_decode_gemv_sweep", "l2": "weight pool > 4x L2, cycled"},
            "roofline": {"bound": "hbm", "achieved": g["mean_GBps"], "best": g["best_GBps"], "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": g["frac_mean"], "traffic": None, "kernel": "rmsnorm_quant+tgemm_mma",
                         "peak_source": peak_kind, "sweep": g["shapes"]},
            "cpu_baseline": None, "e2e": None, "gpu_launches": None}), flush=True)
    return 0


def decode_bytes_per_step(w, B) -> float:
    """Algorithmic bytes of one decode step: the packed weights (0.25 B/weight) + the state read and written."""
    weights = w.layers * (4 * w.d * w.d + 3 * w.d * w.inner) / 4.0
    return weights + 2.0 * w.layers * B * w.d * 4


def measure_decode(mmf, w, B: int, steps: int, warmup: int, dev, peaks, prompt: bool = True, blocks=None) -> dict:
    """Optional prompt prefill, then `steps` decode steps; each decode step (all layers, T=1) is one CUDA
    graph replay whose output is copied back to its input. Returns the timings and the HBM GB/s of the
    step's algorithmic bytes (packed weights + state)."""
    blocks = blocks if blocks is not None else build_stack(w, dev)
    st = mmf.State(w.layers, B, w.d)
    out = {"batch": B, "layers": w.layers, "d": w.d, "inner": w.inner}
    if prompt:
        xp = synth.activations(w.seed + synth.ACT_SEED_OFFSET, B * w.seq, w.d, torch.bfloat16,
                               device=dev).reshape(B, w.seq, w.d)
        ws_p = torch.empty(mmf.stack_ws_size(blocks, B, w.seq), dtype=torch.uint8, device=dev)
        y_p = torch.empty_like(xp)
        mmf.stack_forward(blocks, st, xp, ws=ws_p, out=y_p)   # warm-up
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        st.reset()
        e0.record()
        mmf.stack_forward(blocks, st, xp, ws=ws_p, out=y_p)
        e1.record()
        torch.cuda.synchronize()
        out["prompt"] = w.seq
        out["prefill_ms"] = e0.elapsed_time(e1)
        out["prefill_tokens_per_s"] = B * w.seq / (out["prefill_ms"] / 1e3)
        x = y_p[:, -1:, :].contiguous()
        del ws_p, xp, y_p
    else:
        x = synth.activations(w.seed + synth.ACT_SEED_OFFSET, B, w.d, torch.bfloat16, device=dev).reshape(B, 1, w.d)
    y = torch.empty_like(x)
    ws = torch.empty(mmf.stack_ws_size(blocks, B, 1), dtype=torch.uint8, device=dev)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):   # eager steps first: they also allocate the state's decode buffers
        for _ in range(3):
            mmf.stack_forward(blocks, st, x, ws=ws, out=y)
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    mmf.check()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        mmf.stack_forward(blocks, st, x, ws=ws, out=y)
        x.copy_(y)
    for _ in range(max(warmup, 3)):
        graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        graph.replay()
    e1.record()
    wait_event(e1)
    torch.cuda.synchronize()
    clk = clocks.stop()
    del graph
    mmf.check()
    step_ms = e0.elapsed_time(e1) / steps
    # per-kernel device time of a decode step (eager launches, outside the timed region)
    mmf.prof_reset()
    mmf.prof_enable(True)
    for _ in range(5):
        mmf.stack_forward(blocks, st, x, ws=ws, out=y)
    torch.cuda.synchronize()
    mmf.prof_enable(False)
    prof = mmf.prof_collect()
    nbytes = decode_bytes_per_step(w, B)
    gbs = nbytes / (step_ms / 1e3) / 1e9
    out.update({"decode_steps": steps, "ms_per_step": step_ms, "tokens_per_s": B / (step_ms / 1e3),
                "GBps": gbs, "frac": gbs / peaks["hbm_gbs"], "bytes_per_step": nbytes,
                "launches_per_step": sum(v[0] for v in prof.values()) // 5,
                "per_kernel_ms_eager_step": {k: round(v[1] / 5, 4) for k, v in prof.items()}, "clocks": clk})
    return out


VOCAB = 32000   # the embedding size of the default configuration (hysenlabs review, "Install and model initialisation")


def measure_model_decode(mmf, w, B: int, steps: int, warmup: int, dev, peaks, blocks=None) -> dict:
    """Greedy generation through the whole model: per token the embedding lookup, every block's decode
    step, the LM head (BitLinear d -> 32000) and the argmax, the token fed back on the device; one CUDA
    graph replay per token. Algorithmic bytes per token: the packed weights of the blocks and the head,
    the state read and written, the embedding rows and the logits written and read."""
    blocks = blocks if blocks is not None else build_stack(w, dev)
    head = mmf.quantize_weights(synth.latent_weight(synth.sub_seed(w.seed, w.layers, 7), VOCAB, w.d, device=dev))
    table = synth.activations(w.seed + 7, VOCAB, w.d, torch.bfloat16, device=str(dev))
    st = mmf.State(w.layers, B, w.d)
    ids = torch.randint(0, VOCAB, (B,), dtype=torch.int32, device=dev)
    x = torch.empty(B, 1, w.d, dtype=torch.bfloat16, device=dev)
    y = torch.empty_like(x)
    ws = torch.empty(mmf.stack_ws_size(blocks, B, 1), dtype=torch.uint8, device=dev)
    ws_h = torch.empty(mmf.load().mmf_bitlinear_ws_size(B, w.d), dtype=torch.uint8, device=dev)

    def token():
        mmf.embed(table, ids, out=x.view(B, w.d))
        mmf.stack_forward(blocks, st, x, ws=ws, out=y)
        logits = mmf.bitlinear(head, y.view(B, w.d), ws=ws_h)
        mmf.argmax(logits, out=ids)

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):   # eager tokens first: they also allocate the state's decode buffers
        for _ in range(3):
            token()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    mmf.check()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        token()
    for _ in range(max(warmup, 3)):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        graph.replay()
    e1.record()
    wait_event(e1)
    torch.cuda.synchronize()
    del graph
    mmf.check()
    step_ms = e0.elapsed_time(e1) / steps
    mmf.prof_reset()
    mmf.prof_enable(True)
    for _ in range(5):
        token()
    torch.cuda.synchronize()
    mmf.prof_enable(False)
    prof = mmf.prof_collect()
    nbytes = decode_bytes_per_step(w, B) + VOCAB * w.d / 4.0 + B * w.d * 2 + 2.0 * B * VOCAB * 2
    gbs = nbytes / (step_ms / 1e3) / 1e9
    return {"batch": B, "layers": w.layers, "d": w.d, "inner": w.inner, "vocab": VOCAB, "decode_steps": steps,
            "ms_per_step": step_ms, "tokens_per_s": B / (step_ms / 1e3), "GBps": gbs, "frac": gbs / peaks["hbm_gbs"],
            "bytes_per_step": nbytes, "launches_per_step": sum(v[0] for v in prof.values()) // 5,
            "per_kernel_ms_eager_step": {k: round(v[1] / 5, 4) for k, v in prof.items()}}


def run_model(args):
    """Greedy generation tokens/s of the 2.7B-shaped model (embedding, 32 blocks, head, argmax)."""
    _, rank, local = dist_env()
    torch.cuda.set_device(local)
    import ternary_weight_matmul_fusedbitlinear_b200 as mmf
    dev = torch.device("cuda", local)
    w = synth.STACK_2P7B
    B = args.batch or w.batch
    peaks, peak_kind = load_peaks()
    steps = args.decode_steps or w.decode_steps
    r = measure_model_decode(mmf, w, B, steps, args.warmup, dev, peaks)
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": r["tokens_per_s"], "unit": "tokens/s", "n_gpus": 1, "steps": steps,
            "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"model2p7b_greedy_v{VOCAB}_b{B}", "batch": B, "layers": w.layers, "d": w.d,
                       "inner": w.inner, "vocab": VOCAB, "decode_steps": steps,
                       "l2": "weight stream per token > L2"},
            "roofline": {"bound": "hbm", "achieved": r["GBps"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": r["frac"], "traffic": None, "kernel": "greedy token (all kernels)",
                         "bytes_per_step": r["bytes_per_step"], "peak_source": peak_kind,
                         "per_kernel_ms_eager_step": r["per_kernel_ms_eager_step"]},
            "cpu_baseline": None, "e2e": None, "gpu_launches": r["launches_per_step"] * steps}), flush=True)
    return 0


def run_decode(args):
    _, rank, local = dist_env()
    torch.cuda.set_device(local)
    import ternary_weight_matmul_fusedbitlinear_b200 as mmf
    dev = torch.device("cuda", local)
    w = synth.STACK_1P3B if args.workload == "decode1p3b" else synth.STACK_2P7B
    B = args.batch or w.batch
    peaks, peak_kind = load_peaks()
    steps = args.decode_steps or w.decode_steps
    r = measure_decode(mmf, w, B, steps, args.warmup, dev, peaks, prompt=True)
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": r["tokens_per_s"], "unit": "tokens/s", "n_gpus": 1, "steps": steps,
            "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{w.name}_b{B}", "batch": B, "layers": w.layers, "d": w.d, "inner": w.inner,
                       "prompt": w.seq, "decode_steps": steps, "prefill_ms": r["prefill_ms"],
                       "prefill_tokens_per_s": r["prefill_tokens_per_s"], "l2": "weight stream per step > L2"},
            "roofline": {"bound": "hbm", "achieved": r["GBps"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": r["frac"], "traffic": None, "kernel": "decode step (all kernels)",
                         "bytes_per_step": r["bytes_per_step"], "peak_source": peak_kind,
                         "per_kernel_ms_eager_step": r["per_kernel_ms_eager_step"]},
            "cpu_baseline": None, "e2e": None, "gpu_launches": r["launches_per_step"] * steps,
            "clocks": r["clocks"]}), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "bitlinear":
        return run_bitlinear(args)
    if args.workload == "scan":
        return run_scan(args)
    if args.workload == "model2p7b":
        return run_model(args)
    if args.workload == "gemv":
        return run_gemv(args)
    if args.workload in ("decode1p3b", "decode2p7b"):
        return run_decode(args)
    return run_mmf(args)


if __name__ == "__main__":
    sys.exit(main())
