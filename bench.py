"""Benchmark: W4A16-g128 fused-dequant products on B200.

Headline step = one decode token through the two weight shapes of a 70B
layer's MLP ([28672, 8192] and [8192, 28672]; INT4 asymmetric, g = 128, fp16
scale and zero) at M = 1: two calls of the W4A16 product, each on its own
weight and its own X.  `value` is HBM GB/s of algorithmic bytes (packed codes
+ fp16 scales and zeros + X + Y) over the timed steps, all ranks together.
Inputs are resident in HBM; L2 reuse is defeated by rotating ROT copies of the
quantized weights (ROT x 250 MB > 4x L2).

Secondary measurements on the same line (`extra`): the 7B decode step
([4096,4096], [11008,4096], [4096,11008], symmetric) with its own roofline,
decode at M = 2..16, the prefill W4A16 GEMM (M = 2048, TFLOPS), the W8A8 GEMM
(4096^3, TOPS) with SmoothQuant and in FP8, W8A16, quantize/pack, GPTQ and
the KV-cache quantizer, each timed as a CUDA graph of at least 100
back-to-back launches over rotating buffers larger than L2, and the measured
int8 / fp8 tensor-core peaks the 8-bit fractions divide by.

--impl reference times the CPU oracle (the only reference this method has) on
a bounded sample of the same workload and prints the same metric.

Launch: python bench.py --gpus N --steps K --warmup W
        (N > 1: under torch.distributed.run, one rank per GPU; each rank runs
        its own replica -- the decode product has no exchange step).
"""
import argparse
import concurrent.futures as cf
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
ROT_70B = 3   # rotating weight copies of the 70B step (3 x 250 MB > 4 x 126 MB L2)
ROT_7B = 10   # of the 7B step (10 x 55 MB)

# Parameters of the models whose layers the steps come from (the quantization
# guide's 7B / 70B examples); model bytes at a format = params x bytes/param.
MODEL_PARAMS = {"70b-decode": 70e9, "7b-decode": 7e9}

WORKLOAD_DESC = {
    "70b-decode": "70b-decode: W4A16 g128 asym (fp16 scale+zero), M=1, W [28672,8192]+"
                  "[8192,28672] bf16 N(0,0.015) 0.1% cols x50, X N(0,1)",
    "7b-decode": "7b-decode: W4A16 g128 sym, M=1, W [4096,4096]+[11008,4096]+[4096,11008] "
                 "bf16 N(0,0.02) 0.1% cols x30, X N(0,1)",
}


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


def bytes_per_param(asym):
    """INT4 g128 storage per weight: half a byte of code plus the fp16 scale
    (and zero) shared by 128 weights."""
    return 0.5 + (4.0 if asym else 2.0) / 128


def tokens_per_s_equiv(gbs, M, wl_name, asym):
    """Upper bound on decode tokens/s if every weight of the model streamed at
    this rate: M tokens per pass over params x bytes/param."""
    model_bytes = MODEL_PARAMS[wl_name] * bytes_per_param(asym)
    return M * gbs * 1e9 / model_bytes


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

def setup_decode(wq, wl, M, dev, rot, keep_cpu=False):
    """Quantize each shape's weight on the device and make `rot` copies.
    With keep_cpu, the bf16 CPU weights are returned too (for the CPU leg)."""
    sets, cpu_w = [], []
    for i, (N, K) in enumerate(wl.shapes):
        Wc = wl.weight(i)
        if keep_cpu:
            cpu_w.append(Wc)
        W = Wc.to(dev)
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
    return (sets, cpu_w) if keep_cpu else sets


def capture(fn, count):
    """CUDA graph of fn(j) for j in range(count), captured on a side stream."""
    g = torch.cuda.CUDAGraph()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for j in range(count):
                fn(j)
    torch.cuda.current_stream().wait_stream(stream)
    return g


def decode_call(wq, s, sym, j):
    c, sc, z = s["copies"][j % len(s["copies"])]
    wq.wq_gemm_w4a16(s["X"], c, sc, z, s["N"], 128, sym, s["Y"], s["ws"])


def step_graph(wq, sets, sym, nsteps):
    """Graph of nsteps decode steps; step j runs every shape on copy j % rot."""
    def one(j):
        for s in sets:
            decode_call(wq, s, sym, j)
    return capture(one, nsteps)


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


def per_shape_us(wq, sets, sym, rot, reps=10):
    """Diagnostic: device time of one launch of each shape alone (a graph of
    back-to-back launches of that shape over its rotating copies)."""
    out = []
    for s in sets:
        g = capture(lambda j, s=s: decode_call(wq, s, sym, j), 10 * rot)
        out.append(round(1e3 * time_graph(g, reps) / (10 * rot), 3))
        del g
    return out


TRAFFIC = {
    "70b-decode": os.path.join(ROOT, "profiles", "gemv_cc_kernel_70b_decode_step.txt"),
    "7b-decode": os.path.join(ROOT, "profiles", "gemv_cc_kernel_7b_decode_step.txt"),
}
DECODE_SRC = os.path.join(ROOT, "bit_gemm_group_b200", "csrc", "gemv_w4a16_cc.cu")


def recorded_traffic(path):
    """DRAM bytes (read + write) of one decode step from a committed ncu
    capture, or None when the decode kernel's source has changed since that
    capture (or there is none)."""
    import hashlib
    try:
        fields = {}
        with open(path) as f:
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


def flush_l2(buf):
    buf.add_(1)


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


def timed_steps(wq, sets, sym, rot, steps):
    """Graphs covering exactly `steps` decode steps: full rotations in one
    graph replayed, the remainder in a second graph.  Returns a callable that
    launches them."""
    full, rem = divmod(steps, rot)
    g_full = step_graph(wq, sets, sym, rot) if full else None
    g_rem = step_graph(wq, sets, sym, rem) if rem else None

    def run():
        for _ in range(full):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()
    return run, (g_full, g_rem)


def measure_step(wq, wl_name, M, rot, steps, warm, dev, world, keep_cpu=False, sampler=None):
    """Device time of `steps` decode steps of a workload (max over ranks);
    with a clock sampler, the clocks seen during the timed region."""
    wl = WORKLOADS[wl_name]
    if keep_cpu:
        sets, cpu_w = setup_decode(wq, wl, M, dev, rot, keep_cpu=True)
    else:
        sets, cpu_w = setup_decode(wq, wl, M, dev, rot), None
    asym = not wl.sym
    step_bytes = sum(decode_bytes(s["N"], s["K"], M, asym) for s in sets)
    run_warm, _gw = timed_steps(wq, sets, wl.sym, rot, warm)
    run_warm()
    torch.cuda.synchronize()
    run, graphs = timed_steps(wq, sets, wl.sym, rot, steps)
    run()   # one untimed pass of the same graphs
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    mark = sampler.mark() if sampler is not None else 0
    t0.record(stream)
    run()
    t1.record(stream)
    torch.cuda.synchronize()
    if sampler is not None:
        time.sleep(0.15)   # the sampler reads nvidia-smi's lines with a short lag
    clocks = sampler.summary(mark) if sampler is not None else None
    if world > 1:
        torch.distributed.barrier()
    ms = job_time_ms(t0.elapsed_time(t1), world, dev)
    return {"sets": sets, "cpu_w": cpu_w, "wl": wl, "ms": ms, "step_bytes": step_bytes,
            "asym": asym, "launches": steps * len(sets), "clocks": clocks}


def step_summary(r, M, steps, world, pk, wl_name):
    """Throughput, roofline and tokens/s-equivalent of a measured step."""
    value = job_throughput_gbs(world, steps, r["step_bytes"], r["ms"])
    # the region holds only decode launches, back to back: the average launch
    # moves step_bytes / len(sets) algorithmic bytes in ms / launches
    achieved = job_throughput_gbs(1, steps, r["step_bytes"], r["ms"])
    return value, {
        "bound": "hbm", "achieved": round(achieved, 2), "peak": pk["hbm_gbs"], "unit": "GB/s",
        "frac": round(achieved / pk["hbm_gbs"], 4),
        "traffic": recorded_traffic(TRAFFIC[wl_name]), "traffic_unit": "bytes per step",
        "kernel": "wq W4A16 decode product (gemv_cc_kernel)",
        "peak_source": pk["source"],
    }, round(tokens_per_s_equiv(achieved, M, wl_name, r["asym"]), 1)


def run_ours(args, rank, world, local_rank):
    import bit_gemm_group_b200 as wq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wq.lib()
    pk = peaks()
    M = 1
    warm = max(3, args.warmup)
    want_cpu = rank == 0 and world == 1 and not args.no_cpu

    sampler = ClockSampler(local_rank)
    sampler.start()
    r = measure_step(wq, "70b-decode", M, ROT_70B, args.steps, warm, dev, world,
                     keep_cpu=want_cpu, sampler=sampler)
    sampler.stop()
    clocks = r["clocks"]
    value, roof, tps = step_summary(r, M, args.steps, world, pk, "70b-decode")
    roof["per_shape_us"] = per_shape_us(wq, r["sets"], r["wl"].sym, ROT_70B)
    ms_per_step = r["ms"] / args.steps
    step_bytes = r["step_bytes"]
    e2e = measure_e2e(wq, r["sets"], r["wl"], M, r["asym"])
    cpu = cpu_baseline(r["wl"], r["cpu_w"], M) if want_cpu else None
    del r
    torch.cuda.empty_cache()

    extra = {}
    if not args.quick:
        extra = secondary(wq, dev, args, pk)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": warm, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC["70b-decode"], "M": 1, "group_size": 128,
                   "bytes_per_step": step_bytes,
                   "l2": f"{ROT_70B} rotating weight copies ({ROT_70B * step_bytes / 1e6:.0f} MB)"
                         " > 4x L2",
                   "parallelism": f"replicas x{world}"},
        "roofline": roof,
        "tokens_per_s_equiv": {"value": tps, "unit": "tokens/s",
                               "model": "70B params x 0.53125 B/param (INT4 g128 asym)",
                               "note": "upper bound: every weight streamed at the "
                                       "achieved rate"},
        "e2e": e2e,
        "gpu_launches": args.steps * 2,
        "clocks": clocks,
        "extra": extra,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


def measure_e2e(wq, sets, wl, M, asym, steps=200):
    """Same metric through the public API with host buffers: each step copies
    X from pinned host memory, runs the products and reads Y back.  `value`
    is the direct call sequence; `graph_value` the same sequence captured in a
    CUDA graph (copies included)."""
    host_x = [s["X"].cpu().pin_memory() for s in sets]
    host_y = [torch.empty_like(s["Y"], device="cpu").pin_memory() for s in sets]
    stream = torch.cuda.current_stream()
    h2d = sum(x.numel() * 2 for x in host_x)
    d2h = sum(y.numel() * 2 for y in host_y)
    step_bytes = sum(decode_bytes(s["N"], s["K"], M, asym) for s in sets)

    def one(i):
        for j, s in enumerate(sets):
            s["X"].copy_(host_x[j], non_blocking=True)
            decode_call(wq, s, wl.sym, i)
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
    g = capture(one, steps)
    gms = time_graph(g, 3)
    del g
    return {"value": round(steps * step_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms / steps,
            "graph_value": round(steps * step_bytes / (gms * 1e-3) / 1e9, 2),
            "graph_ms_per_step": gms / steps}


def time_rotating(calls, launches=100, reps=3):
    """Median device time (ms) of one call in a CUDA graph of `launches`
    back-to-back calls, rotating through `calls` (each on its own buffers,
    together larger than L2)."""
    for c in calls:
        c()
    torch.cuda.synchronize()
    g = capture(lambda j: calls[j % len(calls)](), launches)
    ts = [time_graph(g, 1) for _ in range(reps)]
    del g
    return statistics.median(ts) / launches


def measure_int8_fp8_peaks(dev):
    """Dense tensor-core peaks on this GPU, measured as a library GEMM at
    8192^3: torch._int_mm (int8 -> int32) and torch._scaled_mm (E4M3 -> bf16).
    Best of 10 back-to-back runs after warm-up."""
    n = 8192
    out = {}
    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
    b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev).t()
    try:
        for _ in range(3):
            torch._int_mm(a, b)
        ts = []
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(a, b)
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        out["int8_tops"] = round(2.0 * n ** 3 / (min(ts) * 1e-3) / 1e12, 1)
    except RuntimeError as e:  # noqa: PERF203
        out["int8_error"] = str(e)[:120]
    del a, b
    fa = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn)
    fb = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn).t()
    one = torch.tensor(1.0, device=dev)
    try:
        for _ in range(3):
            torch._scaled_mm(fa, fb, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        ts = []
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(fa, fb, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        out["fp8_tflops"] = round(2.0 * n ** 3 / (min(ts) * 1e-3) / 1e12, 1)
    except RuntimeError as e:  # noqa: PERF203
        out["fp8_error"] = str(e)[:120]
    del fa, fb
    torch.cuda.empty_cache()
    out["how"] = "library GEMM 8192^3 (torch._int_mm, torch._scaled_mm E4M3 -> bf16), best of 10"
    return out


def secondary(wq, dev, args, pk):
    """Other rows of the path, each a CUDA graph of >= 100 launches."""
    out = {}
    mp = measure_int8_fp8_peaks(dev)
    out["peaks_measured"] = mp
    int8_peak = mp.get("int8_tops") or 2.0 * pk["bf16_tflops"]
    fp8_peak = mp.get("fp8_tflops") or 2.0 * pk["bf16_tflops"]
    int8_src = "measured" if "int8_tops" in mp else "2x bf16 (nominal ratio)"
    fp8_src = "measured" if "fp8_tflops" in mp else "2x bf16 (nominal ratio)"

    # the 7B decode step (three shapes, symmetric), its own roofline
    steps7 = 20 * ROT_7B
    r = measure_step(wq, "7b-decode", 1, ROT_7B, steps7, 3 * ROT_7B, dev, 1)
    v7, roof7, tps7 = step_summary(r, 1, steps7, 1, pk, "7b-decode")
    roof7["per_shape_us"] = per_shape_us(wq, r["sets"], True, ROT_7B)
    out["decode_7b_step"] = {"value": round(v7, 2), "unit": "GB/s", "roofline": roof7,
                             "tokens_per_s_equiv": tps7, "ms_per_step": r["ms"] / steps7,
                             "bytes_per_step": r["step_bytes"], "workload": WORKLOAD_DESC["7b-decode"]}
    del r
    torch.cuda.empty_cache()

    # decode at more activation rows (same step structure)
    for wl_name, rot, Ms in (("7b-decode", ROT_7B, (2, 4, 8, 16)), ("70b-decode", ROT_70B, (2, 4, 8, 16))):
        for M in Ms:
            steps = 10 * rot
            r = measure_step(wq, wl_name, M, rot, steps, rot, dev, 1)
            v, roof, tps = step_summary(r, M, steps, 1, pk, wl_name)
            key = f"decode_{wl_name.split('-')[0]}_M{M}"
            out[key] = {"gbs": round(v, 1), "frac_hbm": roof["frac"], "tokens_per_s_equiv": tps}
            del r
            torch.cuda.empty_cache()

    # quantize + pack of the 7B [11008, 4096] bf16 weight (5 sets > 4x L2)
    wl = WORKLOADS["7b-decode"]
    W = wl.weight(1).to(dev)
    N, K = W.shape
    qsets = []
    for _ in range(5):
        qsets.append((W.clone(), torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                      torch.empty((N, K // 128), dtype=torch.float16, device=dev)))
    del W
    t = time_rotating([lambda s=s: wq.wq_quantize_pack(s[0], 128, 4, True, s[1], s[2], None)
                       for s in qsets])
    qbytes = N * K * 2 + N * K // 2 + N * (K // 128) * 2
    out["quantize_pack_11008x4096_gbs"] = round(qbytes / (t * 1e-3) / 1e9, 1)
    out["quantize_pack_frac_hbm"] = round(qbytes / (t * 1e-3) / 1e9 / pk["hbm_gbs"], 3)
    del qsets
    torch.cuda.empty_cache()

    # prefill W4A16 GEMM, X [2048, 4096] x W [11008, 4096]^T (6 rotating sets)
    wlp = WORKLOADS["prefill"]
    Wp = wlp.weight(0).to(dev)
    N, K = Wp.shape
    codes, scales, _ = wq.quantize_pack(Wp, 128, 4, True)
    del Wp
    Xp = wlp.activation(2048, K).to(dev)
    psets = [(Xp.clone(), codes.clone(), scales.clone(),
              torch.empty((2048, N), dtype=torch.bfloat16, device=dev)) for _ in range(6)]
    t = time_rotating([lambda s=s: wq.wq_gemm_w4a16(s[0], s[1], s[2], None, N, 128, True, s[3])
                       for s in psets])
    flops = 2.0 * 2048 * N * K
    out["prefill_w4a16_tflops"] = round(flops / (t * 1e-3) / 1e12, 1)
    out["prefill_w4a16_us"] = round(t * 1e3, 1)
    out["prefill_frac_bf16_peak"] = round(flops / (t * 1e-3) / 1e12 / pk["bf16_tflops"], 3)
    del psets, codes, scales, Xp
    torch.cuda.empty_cache()

    # W8A8: per-token act quant + int8 tensor-core GEMM, 4096^3 (5 rotating sets)
    wl8 = WORKLOADS["w8a8"]
    W8 = wl8.weight(0).to(dev)
    qw, sw, _ = wq.quantize_pack(W8, W8.shape[1], 8, True)
    X8 = wl8.activation(4096, 4096).to(dev)
    nws = wq.wq_w8a8_workspace_bytes(4096, 4096)
    wsets = [(X8.clone(), qw.clone(), sw.clone(),
              torch.empty((4096, 4096), dtype=torch.bfloat16, device=dev),
              torch.empty((nws,), dtype=torch.uint8, device=dev)) for _ in range(5)]
    t = time_rotating([lambda s=s: wq.wq_gemm_w8a8(s[0], s[1], s[2], s[3], s[4]) for s in wsets])
    ops = 2.0 * 4096 ** 3
    out["w8a8_tops"] = round(ops / (t * 1e-3) / 1e12, 1)
    out["w8a8_us"] = round(t * 1e3, 1)
    out["w8a8_frac_int8_peak"] = round(ops / (t * 1e-3) / 1e12 / int8_peak, 3)
    out["int8_peak_tops"] = int8_peak
    out["int8_peak_source"] = int8_src

    # SmoothQuant (alpha = 0.5) in front of the same W8A8 product: statistics,
    # factors and the smoothed weight are offline; the timed call quantizes X/s
    # per token and runs the int8 GEMM.  The accuracy of both variants is taken
    # against the fp64 product of the same bf16 inputs on the first 256 rows.
    s8 = wq.smooth_scales(wq.channel_absmax(X8), wq.channel_absmax(W8), 0.5)
    qws, sws = wq.quantize_i8_smooth(W8, s8)
    ssets = [(s[0], qws.clone(), sws.clone(), s8.clone(), s[3], s[4]) for s in wsets]
    t = time_rotating([lambda s=s: wq.wq_gemm_w8a8_smooth(s[0], s[1], s[2], s[3], s[4], s[5])
                       for s in ssets])
    out["w8a8_smooth_tops"] = round(ops / (t * 1e-3) / 1e12, 1)
    out["w8a8_smooth_us"] = round(t * 1e3, 1)
    ref = X8[:256].double().cpu().numpy() @ W8.double().cpu().numpy().T
    y_plain = wq.gemm_w8a8(X8[:256].contiguous(), qw, sw).double().cpu().numpy()
    y_smooth = wq.gemm_w8a8_smooth(X8[:256].contiguous(), qws, sws, s8).double().cpu().numpy()
    nrm = np.linalg.norm(ref)
    out["w8a8_rel_err_plain"] = float(f"{np.linalg.norm(y_plain - ref) / nrm:.3e}")
    out["w8a8_rel_err_smooth"] = float(f"{np.linalg.norm(y_smooth - ref) / nrm:.3e}")
    del ssets, qws, sws, s8

    # FP8 E4M3 W8A8 on the same workload (tcgen05.mma kind::f8f6f4)
    fw, fsw = wq.quantize_fp8_rows(W8)
    fsets = [(s[0], fw.clone(), fsw.clone(), s[3], s[4]) for s in wsets]
    t = time_rotating([lambda s=s: wq.wq_gemm_fp8(s[0], s[1], s[2], s[3], s[4]) for s in fsets])
    out["fp8_tflops"] = round(ops / (t * 1e-3) / 1e12, 1)
    out["fp8_us"] = round(t * 1e3, 1)
    out["fp8_frac_peak"] = round(ops / (t * 1e-3) / 1e12 / fp8_peak, 3)
    out["fp8_peak_tflops"] = fp8_peak
    out["fp8_peak_source"] = fp8_src
    y8 = wq.gemm_fp8(X8[:256].contiguous(), fw, fsw).double().cpu().numpy()
    out["fp8_rel_err"] = float(f"{np.linalg.norm(y8 - ref) / np.linalg.norm(ref):.3e}")
    del fsets, wsets, W8, X8, qw, sw, fw, fsw
    torch.cuda.empty_cache()

    # W8A16 (int8 and E4M3 per-channel weights, bf16 activations): decode
    # M = 1 on the 7B [11008, 4096] weight (HBM GB/s of codes + scales + X + Y,
    # 12 rotating copies) and prefill M = 2048 on the same weight (TFLOPS)
    W16 = WORKLOADS["7b-decode"].weight(1).to(dev)
    N, K = W16.shape
    Xd = WORKLOADS["7b-decode"].activation(1, K).to(dev)
    Xp = WORKLOADS["prefill"].activation(2048, K).to(dev)
    Yd = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
    Yp = [torch.empty((2048, N), dtype=torch.bfloat16, device=dev) for _ in range(4)]
    for name, (q16, s16) in (("int8", wq.quantize_pack(W16, K, 8, True)[:2]),
                             ("e4m3", wq.quantize_fp8_rows(W16))):
        fmt = wq.WQ_W8_INT8 if name == "int8" else wq.WQ_W8_E4M3
        cps = [(q16.clone(), s16.clone()) for _ in range(12)]
        t = time_rotating([lambda c=c: wq.wq_gemm_w8a16(Xd, c[0], fmt, c[1], Yd) for c in cps],
                          launches=120)
        b = N * K + 4 * N + 2 * K + 2 * N
        out[f"w8a16_{name}_decode_gbs"] = round(b / (t * 1e-3) / 1e9, 1)
        out[f"w8a16_{name}_decode_frac_hbm"] = round(b / (t * 1e-3) / 1e9 / pk["hbm_gbs"], 3)
        t = time_rotating([lambda i=i, c=c: wq.wq_gemm_w8a16(Xp, c[0], fmt, c[1], Yp[i])
                           for i, c in enumerate(cps[:4])])
        f = 2.0 * 2048 * N * K
        out[f"w8a16_{name}_prefill_tflops"] = round(f / (t * 1e-3) / 1e12, 1)
        out[f"w8a16_{name}_prefill_frac_bf16_peak"] = round(
            f / (t * 1e-3) / 1e12 / pk["bf16_tflops"], 3)
        del cps
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
    t = time_rotating([lambda: wq.wq_gptq_quantize(Wg, Ug, 128, True, cg, sg, None, ws_g)],
                      launches=100, reps=1)
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
    kvs = []
    for _ in range(2):
        Kc = torch.randn((BH, S, D), generator=gen, device=dev).to(torch.bfloat16)
        Vc = torch.randn((BH, S, D), generator=gen, device=dev).to(torch.bfloat16)
        kvs.append((Kc, Vc, torch.empty((BH, S, D), dtype=torch.int8, device=dev),
                    torch.empty((BH, D), dtype=torch.float32, device=dev),
                    torch.empty((BH, S, D), dtype=torch.int8, device=dev),
                    torch.empty((BH, S), dtype=torch.float32, device=dev)))
    t = time_rotating([lambda s=s: wq.wq_quant_kv(*s) for s in kvs])
    kv_bytes = 2 * BH * S * D * (2 + 1) + BH * D * 4 + BH * S * 4
    out["kv_quant_gbs"] = round(kv_bytes / (t * 1e-3) / 1e9, 1)
    out["kv_quant_frac_hbm"] = round(kv_bytes / (t * 1e-3) / 1e9 / pk["hbm_gbs"], 3)
    del kvs
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------- CPU oracle

def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def prepare_oracle(wl, cpu_w, M, frac):
    """Oracle inputs for the first `frac` of each shape's rows (INT4 codes
    from the oracle's own quantizer)."""
    import oracle
    prepared = []
    for i, (N, K) in enumerate(wl.shapes):
        W = cpu_w[i] if cpu_w is not None else wl.weight(i)
        n = max(8, int(N * frac)) // 8 * 8
        c, s, z, _ = oracle.quantize_int4(bf16_bits(W[:n].contiguous()), 128, wl.sym, oracle.BF16)
        prepared.append((bf16_bits(wl.activation(M, K)), c, s, z, n, K))
    return prepared


def oracle_step(prepared, sym, threads, pool=None):
    """One decode step of the oracle over the prepared rows; with threads > 1
    the rows are sharded into blocks over a thread pool (the oracle's code
    stays single-threaded; ctypes releases the GIL during each call)."""
    import oracle
    b = 0
    for x, c, s, z, n, K in prepared:
        if threads <= 1:
            oracle.gemm_w4a16(x, c, s, z, 128, sym)
        else:
            blk = max(8, (n // (4 * threads)) // 8 * 8)
            futs = [pool.submit(oracle.gemm_w4a16, x, c, s, z, 128, sym, a, min(n, a + blk))
                    for a in range(0, n, blk)]
            for f in futs:
                f.result()
        b += decode_bytes(n, K, x.shape[0], not sym)
    return b


def cpu_baseline(wl, cpu_w, M, budget_s=12.0, frac=1 / 32):
    """The oracle as it stands on this host, on the first `frac` of the rows
    of the same decode step: all cores (row blocks over a thread pool) for the
    reported value, one thread for context."""
    prepared = prepare_oracle(wl, cpu_w, M, frac)
    ncores = os.cpu_count() or 1
    res = {}
    for threads, budget in ((1, budget_s / 3), (ncores, budget_s)):
        with cf.ThreadPoolExecutor(threads) as pool:
            t0 = time.perf_counter()
            total, steps = 0, 0
            while True:
                total += oracle_step(prepared, wl.sym, threads, pool)
                steps += 1
                if time.perf_counter() - t0 >= budget:
                    break
            dt = time.perf_counter() - t0
        res[threads] = (total / dt / 1e9, steps, dt)
    v, steps, dt = res[ncores]
    v1 = res[1][0]
    return {"value": round(v, 4), "unit": "GB/s", "cores": ncores, "kind": "oracle",
            "sample": f"{steps} decode steps of the 70B MLP pair at M=1 on the first "
                      f"{100 * frac:.1f}% of each shape's rows, fp64 C oracle, {ncores} host "
                      f"threads over row blocks in {dt:.1f} s ({cpu_model()})",
            "single_thread_value": round(v1, 4)}


# ----------------------------------------------------------- reference arm

def run_reference(args, rank, world, budget_s=60.0):
    """The oracle as it stands on the host's cores (row blocks over a thread
    pool).  Each of the K steps runs the 70B decode step on the first `frac`
    of every shape's output rows, with frac chosen so that the K timed steps
    take about budget_s; the metric counts the bytes of the rows computed."""
    if rank != 0:
        return
    wl = WORKLOADS["70b-decode"]
    M = 1
    ncores = os.cpu_count() or 1
    probe = prepare_oracle(wl, None, M, 1 / 64)
    with cf.ThreadPoolExecutor(ncores) as pool:
        t0 = time.perf_counter()
        oracle_step(probe, wl.sym, ncores, pool)          # warm-up and rate probe
        t_full = 64 * (time.perf_counter() - t0)          # one full step, estimated
        frac = min(1.0, budget_s / max(1, args.steps) / max(t_full, 1e-6))
        prepared = prepare_oracle(wl, None, M, frac)      # at least 8 rows per shape
        for _ in range(max(0, args.warmup - 1)):
            oracle_step(prepared, wl.sym, ncores, pool)
        total = 0
        t0 = time.perf_counter()
        for _ in range(args.steps):
            total += oracle_step(prepared, wl.sym, ncores, pool)
        dt = time.perf_counter() - t0
    value = total / dt / 1e9
    sample = (f"{args.steps} steps, each the 70B MLP decode pair (M=1) on the first "
              f"{100 * frac:.2f}% of output rows, fp64 C oracle on {ncores} host threads "
              f"({cpu_model()})")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC["70b-decode"], "M": 1, "group_size": 128},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": ncores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ ncu targets

def profile_case(case):
    """Launches of one kernel on its workload, nothing else timed:
    decode-70b-step = two warm-up steps then one step of the 70B decode
    workload (its two shapes; the traffic record of the headline);
    decode-step = the same for the 7B decode workload (three shapes);
    decode = W4A16 decode product on [11008, 4096] at M = 1 (three launches);
    decode-large = the same on [57344, 8192] (235 MB of codes, three
    launches); decode-m16 = [11008, 4096] at M = 16 (tensor-core kernel);
    prefill = W4A16 GEMM 2048 x 11008 x 4096; w8a8 = W8A8 GEMM 4096^3
    (per-token activation quantization + int8 GEMM); fp8 = the same product in
    FP8 E4M3; quantize = INT4 g128 quantize + pack of the bf16 [11008, 4096]
    weight; kv = KV-cache INT8 of a bf16 cache [64, 8192, 128] (three launches
    each); gptq = GPTQ of a bf16 [4096, 4096] weight with a synthetic
    inverse-Hessian factor (one launch); w8a16 = int8 W8A16 on the [11008,
    4096] weight at M = 1 then M = 2048 (three launches each)."""
    import bit_gemm_group_b200 as wq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if case in ("decode-step", "decode-70b-step"):
        wl = WORKLOADS["7b-decode" if case == "decode-step" else "70b-decode"]
        sets = []
        for i, (N, K) in enumerate(wl.shapes):
            c, s, z = wq.quantize_pack(wl.weight(i).to(dev), 128, 4, wl.sym)
            sets.append((N, K, c, s, z, wl.activation(1, K).to(dev),
                         torch.empty((1, N), dtype=torch.bfloat16, device=dev),
                         wq.w4a16_workspace(1, N, K, dev)))
        for _ in range(3):
            for N, K, c, s, z, X, Y, ws in sets:
                wq.wq_gemm_w4a16(X, c, s, z, N, 128, wl.sym, Y, ws)
    elif case == "decode-large":
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
    elif case in ("decode", "decode-m16"):
        M = 1 if case == "decode" else 16
        wl = WORKLOADS["7b-decode"]
        W = wl.weight(1).to(dev)
        N, K = W.shape
        c, s, z = wq.quantize_pack(W, 128, 4, True)
        X = wl.activation(M, K).to(dev)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = wq.w4a16_workspace(M, N, K, dev)
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
    ap.add_argument("--warmup", type=int, default=30)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--quick", action="store_true", help="skip the secondary rows")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-baseline leg")
    ap.add_argument("--profile-case",
                    choices=["decode", "decode-large", "decode-step", "decode-70b-step",
                             "decode-m16", "prefill", "w8a8", "fp8", "quantize", "kv", "gptq",
                             "w8a16"],
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
        line = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
