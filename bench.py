"""Benchmark: W4A16-g128 fused-dequant decode product on B200.

One step = one decode token through the three weight shapes of a 7B layer
([4096,4096], [11008,4096], [4096,11008]; INT4 symmetric, g = 128) at M = 1:
three calls of the W4A16 product, each on its own weight.  `value` is HBM
GB/s of algorithmic bytes (packed codes + fp16 scales + X + Y) over the timed
steps, all ranks together.  Inputs are resident in HBM; L2 reuse is defeated
by rotating ROT copies of the quantized weights (ROT x 55 MB > 4x L2).

Secondary measurements on the same line (`extra`): the prefill W4A16 GEMM
(M = 2048, TFLOPS), the W8A8 GEMM (4096^3, TOPS), quantize/pack GB/s, and
the decode product at M = 4 and 16.

--impl reference times the CPU oracle (the only reference this method has) on
a bounded sample of the same workload and prints the same metric.

Launch: python bench.py --gpus N --steps K --warmup W
        (N > 1: under torch.distributed.run, one rank per GPU; each rank runs
        its own replica -- the decode product has no exchange step).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, bf16_bits, make_activation  # noqa: E402

METRIC = "W4A16-g128 dequant-GEMM: HBM GB/s at M=1, TFLOPS at M=2048, % of roofline"
ROT = 10  # rotating weight copies (10 x 55 MB = 550 MB > 4 x 126 MB L2)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def decode_bytes(N, K, M, asym=False):
    """Algorithmic bytes of one W4A16 decode product: packed codes, fp16
    scales (and zeros), X and Y, each read or written once."""
    G = K // 128
    return N * K // 2 + N * G * 2 * (2 if asym else 1) + 2 * M * K + 2 * M * N


# ------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def mark(self):
        return len(self.lines)

    def stop(self):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, start_mark=0):
        rows = []
        for ln in self.lines[start_mark:]:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"],
                    "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i] == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------ device setup

def setup_decode(wq, wl, M, dev, rot):
    """Quantize each shape's weight on the device and make `rot` copies."""
    sets = []
    for i, (N, K) in enumerate(wl.shapes):
        W = wl.weight(i).to(dev)
        codes, scales, zeros = wq.quantize_pack(W, 128, 4, wl.sym)
        del W
        copies = [(codes, scales, zeros)]
        for _ in range(rot - 1):
            copies.append((codes.clone(), scales.clone(),
                           None if zeros is None else zeros.clone()))
        X = wl.activation(M, K).to(dev)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = wq.w4a16_workspace(M, N, K, dev)
        sets.append({"N": N, "K": K, "copies": copies, "X": X, "Y": Y, "ws": ws})
    return sets


def capture_shape_graph(wq, s, sym, count, start):
    """CUDA graph of `count` back-to-back decode products of one shape, each
    on the next rotating copy of its weight."""
    g = torch.cuda.CUDAGraph()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for j in range(count):
                c, sc, z = s["copies"][(start + j) % len(s["copies"])]
                wq.wq_gemm_w4a16(s["X"], c, sc, z, s["N"], 128, sym, s["Y"], s["ws"])
    torch.cuda.current_stream().wait_stream(stream)
    return g


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gemv_cc_kernel_7b_decode_step.txt")
DECODE_SRC = os.path.join(ROOT, "bit_gemm_group_b200", "csrc", "gemv_w4a16_cc.cu")


def recorded_traffic():
    """DRAM bytes (read + write) of one 7B decode step (its three decode
    launches) from the committed ncu capture, or None when the decode kernel's
    source has changed since that capture (or there is none)."""
    import hashlib
    try:
        fields = {}
        with open(TRAFFIC_FILE) as f:
            for line in f:
                if ":" in line:
                    k, v = line.split(":", 1)
                    fields[k.strip()] = v.strip()
        with open(DECODE_SRC, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
        if fields.get("kernel_source_sha256") != sha:
            return None
        return int(fields["dram_bytes_per_step"])
    except (OSError, KeyError, ValueError):
        return None


def time_graph(g, reps):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g.replay()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps  # ms per replay


def flush_l2(buf):
    buf.add_(1)


def time_flushed(fn, flush, reps=10, warm=3):
    """Median device time (ms) of fn() with the L2 flushed before each run."""
    for _ in range(warm):
        fn()
    ts = []
    for _ in range(reps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.median(ts)


# ----------------------------------------------------------------- our arm

def job_time_ms(local_ms, world, device):
    """The job's time: the slowest rank's device time (all ranks take part)."""
    if world <= 1:
        return float(local_ms)
    tt = torch.tensor([float(local_ms)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
    return float(tt.item())


def job_throughput_gbs(world, steps, step_bytes, ms):
    """Whole-job GB/s: every rank streams its own replica's bytes each step."""
    return world * steps * step_bytes / (ms * 1e-3) / 1e9


def run_ours(args, rank, world, local_rank):
    import bit_gemm_group_b200 as wq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wq.lib()
    wl = WORKLOADS["7b-decode"]
    M = 1
    sets = setup_decode(wq, wl, M, dev, ROT)
    step_bytes = sum(decode_bytes(s["N"], s["K"], M) for s in sets)

    # graphs: per shape, ROT launches (one per rotating copy) = ROT steps
    graphs = [capture_shape_graph(wq, s, wl.sym, ROT, 0) for s in sets]
    stream = torch.cuda.current_stream()

    def run_steps(nsteps, events=None):
        full, rem = divmod(nsteps, ROT)
        for _ in range(full):
            for j, g in enumerate(graphs):
                if events is not None:
                    events[j].append(torch.cuda.Event(enable_timing=True))
                    events[j][-1].record(stream)
                g.replay()
                if events is not None:
                    events[j].append(torch.cuda.Event(enable_timing=True))
                    events[j][-1].record(stream)
        for r in range(rem):
            for s in sets:
                c, sc, z = s["copies"][r % ROT]
                wq.wq_gemm_w4a16(s["X"], c, sc, z, s["N"], 128, wl.sym, s["Y"], s["ws"])

    warm = max(3, args.warmup)
    run_steps(warm)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()

    sampler = ClockSampler(local_rank)
    sampler.start()
    mark = sampler.mark()
    events = [[] for _ in sets]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    t0.record(stream)
    run_steps(args.steps, events)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    sampler.stop()
    ms = job_time_ms(t0.elapsed_time(t1), world, dev)
    clocks = sampler.summary(mark)

    # kernel time per shape from the events around each graph replay
    kern_ms = [sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(len(ev) // 2))
               for ev in events]
    launches_timed = (args.steps // ROT) * ROT
    kernel_total_ms = sum(kern_ms)
    pk = peaks()
    value = job_throughput_gbs(world, args.steps, step_bytes, ms)
    achieved = (launches_timed * step_bytes / (kernel_total_ms * 1e-3) / 1e9
                if kernel_total_ms > 0 else None)

    extra = {}
    if not args.quick:
        extra = secondary(wq, dev, args)
    e2e = measure_e2e(wq, sets, wl, M, dev)
    cpu = cpu_baseline(wl, M) if (rank == 0 and world == 1 and not args.no_cpu) else None

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": warm, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "7b-decode: W4A16 g128 sym, M=1, W [4096,4096]+[11008,4096]"
                               "+[4096,11008] bf16 N(0,0.02) 0.1% cols x30, X N(0,1)",
                   "M": 1, "group_size": 128, "bytes_per_step": step_bytes,
                   "l2": f"{ROT} rotating weight copies ({ROT * step_bytes / 1e6:.0f} MB) > 4x L2",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2) if achieved else None,
                     "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / pk["hbm_gbs"], 4) if achieved else None,
                     "traffic": recorded_traffic(), "traffic_unit": "bytes per step",
                     "kernel": "wq W4A16 decode product",
                     "peak_source": pk["source"],
                     "per_shape_us": [round(1e3 * k / max(1, launches_timed), 3)
                                      for k in kern_ms]},
        "e2e": e2e,
        "gpu_launches": args.steps * len(sets),
        "clocks": clocks,
        "extra": extra,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)


def measure_e2e(wq, sets, wl, M, dev, steps=200):
    """Same metric through the public API with host buffers: each step copies
    X from pinned host memory, runs the three products and reads Y back."""
    host_x = [s["X"].cpu().pin_memory() for s in sets]
    host_y = [torch.empty_like(s["Y"], device="cpu").pin_memory() for s in sets]
    stream = torch.cuda.current_stream()
    h2d = sum(x.numel() * 2 for x in host_x)
    d2h = sum(y.numel() * 2 for y in host_y)
    step_bytes = sum(decode_bytes(s["N"], s["K"], M) for s in sets)

    def one(i):
        for j, s in enumerate(sets):
            s["X"].copy_(host_x[j], non_blocking=True)
            c, sc, z = s["copies"][i % len(s["copies"])]
            wq.wq_gemm_w4a16(s["X"], c, sc, z, s["N"], 128, wl.sym, s["Y"], s["ws"])
            host_y[j].copy_(s["Y"], non_blocking=True)

    for i in range(5):
        one(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        one(i)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    return {"value": round(steps * step_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms / steps}


def secondary(wq, dev, args):
    """Other rows of the path, timed with CUDA events (one line each)."""
    out = {}
    pk = peaks()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    # quantize + pack of the 7B weights (bf16 in, codes + scales out)
    wl = WORKLOADS["7b-decode"]
    W = wl.weight(1).to(dev)
    N, K = W.shape
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((N, K // 128), dtype=torch.float16, device=dev)
    for _ in range(3):
        wq.wq_quantize_pack(W, 128, 4, True, codes, scales, None)
    ts = []
    for _ in range(10):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        wq.wq_quantize_pack(W, 128, 4, True, codes, scales, None)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    qbytes = N * K * 2 + N * K // 2 + N * (K // 128) * 2
    t = statistics.median(ts)
    out["quantize_pack_11008x4096_gbs"] = round(qbytes / (t * 1e-3) / 1e9, 1)
    out["quantize_pack_frac_hbm"] = round(qbytes / (t * 1e-3) / 1e9 / pk["hbm_gbs"], 3)
    del W

    # decode product at M = 4 and 16 (same rotation scheme, one graph per shape)
    for M in (4, 16):
        sets = setup_decode(wq, wl, M, dev, ROT)
        tot_ms = 0.0
        for s in sets:
            g = capture_shape_graph(wq, s, True, ROT, 0)
            tot_ms += time_graph(g, 20) / ROT
        b = sum(decode_bytes(s["N"], s["K"], M) for s in sets)
        out[f"decode_M{M}_gbs"] = round(b / (tot_ms * 1e-3) / 1e9, 1)
        del sets
    torch.cuda.empty_cache()

    # 70B decode shapes at M = 1 (asymmetric, fp16 scale + zero), 3 rotating copies
    wl70 = WORKLOADS["70b-decode"]
    sets = setup_decode(wq, wl70, 1, dev, 3)
    tot_ms = 0.0
    for s in sets:
        g = capture_shape_graph(wq, s, False, 3, 0)
        tot_ms += time_graph(g, 10) / 3
    b = sum(decode_bytes(s["N"], s["K"], 1, asym=True) for s in sets)
    out["decode_70b_M1_gbs"] = round(b / (tot_ms * 1e-3) / 1e9, 1)
    del sets
    torch.cuda.empty_cache()

    # prefill W4A16 GEMM, X [2048, 4096] x W [11008, 4096]^T (L2 flushed between runs)
    wlp = WORKLOADS["prefill"]
    Wp = wlp.weight(0).to(dev)
    N, K = Wp.shape
    codes, scales, _ = wq.quantize_pack(Wp, 128, 4, True)
    del Wp
    Xp = wlp.activation(2048, K).to(dev)
    Yp = torch.empty((2048, N), dtype=torch.bfloat16, device=dev)
    t = time_flushed(lambda: wq.wq_gemm_w4a16(Xp, codes, scales, None, N, 128, True, Yp), flush)
    flops = 2.0 * 2048 * N * K
    out["prefill_w4a16_tflops"] = round(flops / (t * 1e-3) / 1e12, 1)
    out["prefill_w4a16_us"] = round(t * 1e3, 1)
    out["prefill_frac_bf16_peak"] = round(flops / (t * 1e-3) / 1e12 / pk["bf16_tflops"], 3)
    del codes, scales, Xp, Yp

    # W8A8: per-token act quant + int8 tensor-core GEMM, 4096^3
    wl8 = WORKLOADS["w8a8"]
    W8 = wl8.weight(0).to(dev)
    qw, sw, _ = wq.quantize_pack(W8, W8.shape[1], 8, True)
    del W8
    X8 = wl8.activation(4096, 4096).to(dev)
    Y8 = torch.empty((4096, 4096), dtype=torch.bfloat16, device=dev)
    ws8 = torch.empty((wq.wq_w8a8_workspace_bytes(4096, 4096),), dtype=torch.uint8, device=dev)
    t = time_flushed(lambda: wq.wq_gemm_w8a8(X8, qw, sw, Y8, ws8), flush)
    ops = 2.0 * 4096 ** 3
    int8_peak = 2.0 * pk["bf16_tflops"]  # measured bf16 peak x the nominal int8/bf16 ratio
    out["w8a8_tops"] = round(ops / (t * 1e-3) / 1e12, 1)
    out["w8a8_us"] = round(t * 1e3, 1)
    out["w8a8_frac_int8_peak"] = round(ops / (t * 1e-3) / 1e12 / int8_peak, 3)
    out["int8_peak_tops"] = int8_peak

    # SmoothQuant (alpha = 0.5) in front of the same W8A8 product: statistics,
    # factors and the smoothed weight are offline; the timed call quantizes X/s
    # per token and runs the int8 GEMM.  The accuracy of both variants is taken
    # against the fp64 product of the same bf16 inputs on the first 256 rows.
    W8 = wl8.weight(0).to(dev)
    s8 = wq.smooth_scales(wq.channel_absmax(X8), wq.channel_absmax(W8), 0.5)
    qws, sws = wq.quantize_i8_smooth(W8, s8)
    t = time_flushed(lambda: wq.wq_gemm_w8a8_smooth(X8, qws, sws, s8, Y8, ws8), flush)
    out["w8a8_smooth_tops"] = round(ops / (t * 1e-3) / 1e12, 1)
    out["w8a8_smooth_us"] = round(t * 1e3, 1)
    ref = X8[:256].double().cpu().numpy() @ W8.double().cpu().numpy().T
    y_plain = wq.gemm_w8a8(X8[:256].contiguous(), qw, sw).double().cpu().numpy()
    y_smooth = wq.gemm_w8a8_smooth(X8[:256].contiguous(), qws, sws, s8).double().cpu().numpy()
    nrm = np.linalg.norm(ref)
    out["w8a8_rel_err_plain"] = float(f"{np.linalg.norm(y_plain - ref) / nrm:.3e}")
    out["w8a8_rel_err_smooth"] = float(f"{np.linalg.norm(y_smooth - ref) / nrm:.3e}")
    del qw, sw, X8, Y8, ws8, W8, s8, qws, sws
    torch.cuda.empty_cache()

    # FP8 E4M3 W8A8 on the same workload (tcgen05.mma kind::f8f6f4)
    W8 = wl8.weight(0).to(dev)
    X8 = wl8.activation(4096, 4096).to(dev)
    Y8 = torch.empty((4096, 4096), dtype=torch.bfloat16, device=dev)
    ws8 = torch.empty((wq.wq_w8a8_workspace_bytes(4096, 4096),), dtype=torch.uint8, device=dev)
    fw, fsw = wq.quantize_fp8_rows(W8)
    t = time_flushed(lambda: wq.wq_gemm_fp8(X8, fw, fsw, Y8, ws8), flush)
    fp8_peak = 2.0 * pk["bf16_tflops"]  # measured bf16 peak x the nominal fp8/bf16 ratio
    out["fp8_tflops"] = round(ops / (t * 1e-3) / 1e12, 1)
    out["fp8_us"] = round(t * 1e3, 1)
    out["fp8_frac_peak"] = round(ops / (t * 1e-3) / 1e12 / fp8_peak, 3)
    ref = X8[:256].double().cpu().numpy() @ W8.double().cpu().numpy().T
    y8 = wq.gemm_fp8(X8[:256].contiguous(), fw, fsw).double().cpu().numpy()
    out["fp8_rel_err"] = float(f"{np.linalg.norm(y8 - ref) / np.linalg.norm(ref):.3e}")
    del W8, X8, Y8, ws8, fw, fsw
    torch.cuda.empty_cache()

    # W8A16 (int8 and E4M3 per-channel weights, bf16 activations): decode
    # M = 1 on the 7B [11008, 4096] weight (HBM GB/s of codes + scales + X + Y)
    # and prefill M = 2048 on the same weight (TFLOPS), L2 flushed between runs
    W16 = WORKLOADS["7b-decode"].weight(1).to(dev)
    N, K = W16.shape
    Xd = WORKLOADS["7b-decode"].activation(1, K).to(dev)
    Xp = WORKLOADS["prefill"].activation(2048, K).to(dev)
    Yd = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
    Yp = torch.empty((2048, N), dtype=torch.bfloat16, device=dev)
    for name, (q16, s16) in (("int8", wq.quantize_pack(W16, K, 8, True)[:2]),
                             ("e4m3", wq.quantize_fp8_rows(W16))):
        fmt = wq.WQ_W8_INT8 if name == "int8" else wq.WQ_W8_E4M3
        t = time_flushed(lambda: wq.wq_gemm_w8a16(Xd, q16, fmt, s16, Yd), flush)
        b = N * K + 4 * N + 2 * K + 2 * N
        out[f"w8a16_{name}_decode_gbs"] = round(b / (t * 1e-3) / 1e9, 1)
        out[f"w8a16_{name}_decode_frac_hbm"] = round(b / (t * 1e-3) / 1e9 / pk["hbm_gbs"], 3)
        t = time_flushed(lambda: wq.wq_gemm_w8a16(Xp, q16, fmt, s16, Yp), flush)
        f = 2.0 * 2048 * N * K
        out[f"w8a16_{name}_prefill_tflops"] = round(f / (t * 1e-3) / 1e12, 1)
        out[f"w8a16_{name}_prefill_frac_bf16_peak"] = round(
            f / (t * 1e-3) / 1e12 / pk["bf16_tflops"], 3)
    del W16, Xd, Xp, Yd, Yp, q16, s16
    torch.cuda.empty_cache()

    # GPTQ of a [4096, 4096] bf16 weight (the 7B square projection), factor
    # from 8192 synthetic correlated calibration tokens (numpy, not timed)
    K = 4096
    rng = np.random.default_rng(12)
    Xc = rng.standard_normal((8192, K // 8)) @ rng.standard_normal((K // 8, K))
    Xc += 0.2 * rng.standard_normal((8192, K))
    H = 2.0 * Xc.T @ Xc
    H += 0.01 * np.mean(np.diag(H)) * np.eye(K)
    Ucpu = np.linalg.cholesky(np.linalg.inv(H)).T.copy()   # upper, H^-1 = U^T U
    del Xc, H
    Ug = torch.from_numpy(Ucpu).to(dev)
    Wg = WORKLOADS["7b-decode"].weight(0).to(dev)
    ws_g = torch.empty((int(wq.lib().wq_gptq_workspace_bytes(K, K)),), dtype=torch.uint8,
                       device=dev)
    cg = torch.empty((K, K // 2), dtype=torch.uint8, device=dev)
    sg = torch.empty((K, K // 128), dtype=torch.float16, device=dev)
    t = time_flushed(lambda: wq.wq_gptq_quantize(Wg, Ug, 128, True, cg, sg, None, ws_g), flush,
                     reps=3, warm=1)
    out["gptq_4096x4096_ms"] = round(t, 3)
    out["gptq_4096x4096_fp64_tflops"] = round(2.0 * K * K * K / 2 / (t * 1e-3) / 1e12, 2)
    del Ug, Wg, ws_g, cg, sg
    torch.cuda.empty_cache()

    # KV-cache INT8 (K per channel, V per token), bf16 cache of 8 kv heads x 8
    # sequences x 8192 tokens x 128 dims (2 x 134 MB, larger than L2).  The
    # algorithmic bytes count one read of K and V, the int8 writes and the
    # scales; K is read a second time for its channel maxima.
    BH, S, D = 64, 8192, 128
    gen = torch.Generator(device=dev)
    gen.manual_seed(6)
    Kc = torch.randn((BH, S, D), generator=gen, device=dev).to(torch.bfloat16)
    Vc = torch.randn((BH, S, D), generator=gen, device=dev).to(torch.bfloat16)
    qk = torch.empty((BH, S, D), dtype=torch.int8, device=dev)
    qv = torch.empty_like(qk)
    sk = torch.empty((BH, D), dtype=torch.float32, device=dev)
    sv = torch.empty((BH, S), dtype=torch.float32, device=dev)
    t = time_flushed(lambda: wq.wq_quant_kv(Kc, Vc, qk, sk, qv, sv), flush)
    kv_bytes = 2 * BH * S * D * (2 + 1) + BH * D * 4 + BH * S * 4
    out["kv_quant_gbs"] = round(kv_bytes / (t * 1e-3) / 1e9, 1)
    out["kv_quant_frac_hbm"] = round(kv_bytes / (t * 1e-3) / 1e9 / pk["hbm_gbs"], 3)
    del Kc, Vc, qk, qv, sk, sv
    torch.cuda.empty_cache()
    return out


def cpu_baseline(wl, M, budget_s=12.0):
    """The oracle as it stands, single-threaded on this host, on the same
    decode step (three 7B shapes at M = 1), repeated until ~budget_s."""
    import oracle
    prepared = []
    for i, (N, K) in enumerate(wl.shapes):
        W = wl.weight(i)
        c, s, z, _ = oracle.quantize_int4(bf16_bits(W), 128, True, oracle.BF16)
        prepared.append((bf16_bits(wl.activation(M, K)), c, s, z, N, K))
    step_bytes = sum(decode_bytes(N, K, M) for *_, N, K in prepared)
    t0 = time.perf_counter()
    steps = 0
    while True:
        for x, c, s, z, N, K in prepared:
            oracle.gemm_w4a16(x, c, s, z, 128, True)
        steps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(steps * step_bytes / dt / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle",
            "sample": f"{steps} full decode steps (3 shapes, M=1) of the fp64 C oracle in "
                      f"{dt:.1f} s on one host thread ({os.cpu_count()} cores present)"}


# ----------------------------------------------------------- reference arm

def run_reference(args, rank, world, budget_s=60.0):
    """The oracle as it stands, one host thread.  Each of the K steps runs the
    decode step on the first `frac` of every shape's output rows, with frac
    chosen so the K timed steps take about budget_s; the metric counts the
    bytes of the rows actually computed."""
    if rank != 0:
        return
    wl = WORKLOADS["7b-decode"]
    M = 1
    import oracle
    prepared = []
    for i, (N, K) in enumerate(wl.shapes):
        W = wl.weight(i)
        c, s, z, _ = oracle.quantize_int4(bf16_bits(W), 128, True, oracle.BF16)
        prepared.append((bf16_bits(wl.activation(M, K)), c, s, z, N, K))

    def step(frac):
        b = 0
        for x, c, s, z, N, K in prepared:
            n1 = max(8, int(N * frac))
            oracle.gemm_w4a16(x, c, s, z, 128, True, 0, n1)
            b += decode_bytes(n1, K, M)
        return b

    t0 = time.perf_counter()
    step(1.0)                                       # warm-up: one full step
    t_full = time.perf_counter() - t0
    frac = min(1.0, budget_s / max(1, args.steps) / t_full)
    for _ in range(max(0, args.warmup - 1)):
        step(frac)
    total = 0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        total += step(frac)
    dt = time.perf_counter() - t0
    value = total / dt / 1e9
    sample = (f"{args.steps} steps, each the decode step (3 shapes, M=1) on the first "
              f"{100 * frac:.1f}% of output rows, fp64 C oracle on one host thread")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "7b-decode: W4A16 g128 sym, M=1, W [4096,4096]+[11008,4096]"
                               "+[4096,11008] bf16 N(0,0.02) 0.1% cols x30, X N(0,1)",
                   "M": 1, "group_size": 128},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def profile_case(case):
    """Launches of one kernel on its workload, nothing else timed:
    decode = W4A16 decode product on [11008, 4096] at M = 1 (three launches),
    decode-large = the same on [57344, 8192] (a fused gate/up projection of a
    70B model, 235 MB of codes, larger than L2; three launches), decode-step =
    two warm-up steps then one step of the 7B decode workload (its three
    shapes), prefill = W4A16 GEMM 2048 x 11008 x 4096, w8a8 = W8A8 GEMM 4096^3
    (per-token activation quantization + int8 GEMM), fp8 = the same product in
    FP8 E4M3, decode-m16 = W4A16 decode product on [11008, 4096] at M = 16
    (tensor-core kernel), quantize = INT4 g128 quantize + pack of the bf16
    [11008, 4096] weight, kv = KV-cache INT8 of a bf16 cache [64, 8192, 128]
    (three launches each); gptq = GPTQ of a bf16 [4096, 4096] weight with a
    synthetic inverse-Hessian factor (one launch); w8a16 = int8 W8A16 on the
    [11008, 4096] weight at M = 1 then M = 2048 (three launches each)."""
    import bit_gemm_group_b200 as wq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if case == "decode-large":
        N, K = 57344, 8192
        gen = torch.Generator(device=dev)
        gen.manual_seed(7)
        W = (torch.randn((N, K), generator=gen, device=dev) * 0.02).to(torch.bfloat16)
        c, s, z = wq.quantize_pack(W, 128, 4, True)
        del W
        X = make_activation(1, K, seed=7).to(dev)
        Y = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
        ws = wq.w4a16_workspace(1, N, K, dev)
        for _ in range(3):
            wq.wq_gemm_w4a16(X, c, s, None, N, 128, True, Y, ws)
    elif case == "decode-step":
        wl = WORKLOADS["7b-decode"]
        sets = []
        for i, (N, K) in enumerate(wl.shapes):
            c, s, z = wq.quantize_pack(wl.weight(i).to(dev), 128, 4, True)
            sets.append((N, K, c, s, wl.activation(1, K).to(dev),
                         torch.empty((1, N), dtype=torch.bfloat16, device=dev),
                         wq.w4a16_workspace(1, N, K, dev)))
        for _ in range(3):
            for N, K, c, s, X, Y, ws in sets:
                wq.wq_gemm_w4a16(X, c, s, None, N, 128, True, Y, ws)
    elif case == "decode":
        wl = WORKLOADS["7b-decode"]
        W = wl.weight(1).to(dev)
        N, K = W.shape
        c, s, z = wq.quantize_pack(W, 128, 4, True)
        X = wl.activation(1, K).to(dev)
        Y = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
        ws = wq.w4a16_workspace(1, N, K, dev)
        for _ in range(3):
            wq.wq_gemm_w4a16(X, c, s, None, N, 128, True, Y, ws)
    elif case == "decode-m16":
        wl = WORKLOADS["7b-decode"]
        W = wl.weight(1).to(dev)
        N, K = W.shape
        c, s, z = wq.quantize_pack(W, 128, 4, True)
        X = wl.activation(16, K).to(dev)
        Y = torch.empty((16, N), dtype=torch.bfloat16, device=dev)
        ws = wq.w4a16_workspace(16, N, K, dev)
        for _ in range(3):
            wq.wq_gemm_w4a16(X, c, s, None, N, 128, True, Y, ws)
    elif case == "quantize":
        W = WORKLOADS["7b-decode"].weight(1).to(dev)
        N, K = W.shape
        c = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
        s = torch.empty((N, K // 128), dtype=torch.float16, device=dev)
        for _ in range(3):
            wq.wq_quantize_pack(W, 128, 4, True, c, s, None)
    elif case == "kv":
        BH, S, D = 64, 8192, 128
        gen = torch.Generator(device=dev)
        gen.manual_seed(6)
        Kc = torch.randn((BH, S, D), generator=gen, device=dev).to(torch.bfloat16)
        Vc = torch.randn((BH, S, D), generator=gen, device=dev).to(torch.bfloat16)
        for _ in range(3):
            wq.quant_kv(Kc, Vc)
    elif case == "gptq":
        K = 4096
        gen = torch.Generator(device=dev)
        gen.manual_seed(12)
        A = torch.randn((K, K), generator=gen, device=dev, dtype=torch.float64) / K ** 0.5
        H = A.T @ A + 0.01 * torch.eye(K, device=dev, dtype=torch.float64)
        U = torch.linalg.cholesky(torch.linalg.inv(H)).T.contiguous()  # upper, H^-1 = U^T U
        del A, H
        W = WORKLOADS["7b-decode"].weight(0).to(dev)
        wq.gptq_quantize(W, U, True)
    elif case == "w8a16":
        W = WORKLOADS["7b-decode"].weight(1).to(dev)
        N, K = W.shape
        q, s, _ = wq.quantize_pack(W, K, 8, True)
        Xd = WORKLOADS["7b-decode"].activation(1, K).to(dev)
        Xp = WORKLOADS["prefill"].activation(2048, K).to(dev)
        for _ in range(3):
            wq.gemm_w8a16(Xd, q, s)
        for _ in range(3):
            wq.gemm_w8a16(Xp, q, s)
    elif case == "fp8":
        wl = WORKLOADS["w8a8"]
        W = wl.weight(0).to(dev)
        fw, fsw = wq.quantize_fp8_rows(W)
        X = wl.activation(4096, 4096).to(dev)
        Y = torch.empty((4096, 4096), dtype=torch.bfloat16, device=dev)
        ws = torch.empty((wq.wq_w8a8_workspace_bytes(4096, 4096),), dtype=torch.uint8, device=dev)
        for _ in range(3):
            wq.wq_gemm_fp8(X, fw, fsw, Y, ws)
    elif case == "prefill":
        wl = WORKLOADS["prefill"]
        W = wl.weight(0).to(dev)
        N, K = W.shape
        c, s, z = wq.quantize_pack(W, 128, 4, True)
        X = wl.activation(2048, K).to(dev)
        Y = torch.empty((2048, N), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            wq.wq_gemm_w4a16(X, c, s, None, N, 128, True, Y)
    else:
        wl = WORKLOADS["w8a8"]
        W = wl.weight(0).to(dev)
        qw, sw, _ = wq.quantize_pack(W, W.shape[1], 8, True)
        X = wl.activation(4096, 4096).to(dev)
        Y = torch.empty((4096, 4096), dtype=torch.bfloat16, device=dev)
        ws = torch.empty((wq.wq_w8a8_workspace_bytes(4096, 4096),), dtype=torch.uint8, device=dev)
        for _ in range(3):
            wq.wq_gemm_w8a8(X, qw, sw, Y, ws)
    torch.cuda.synchronize()
    print(case, "status", wq.wq_status_str(wq.wq_get_device_status()))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--quick", action="store_true", help="skip the secondary rows")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-baseline leg")
    ap.add_argument("--profile-case",
                    choices=["decode", "decode-large", "decode-step", "decode-m16", "prefill",
                             "w8a8", "fp8", "quantize", "kv", "gptq", "w8a16"],
                    help="run one kernel 3 times on its workload (for ncu captures) and exit")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
