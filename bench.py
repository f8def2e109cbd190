"""Benchmark: batch-1 decode through a Llama-2-7B-shaped stack of rotated 2-bit linears.

One step = one decode token through 32 blocks of seven rotated low-bit linears
(q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008; 256-wide butterfly blocks
on the 11008 side) with RMSNorm, residual adds, SiLU*up and the one-key attention
stand-in between them -- every step of the hot path, in the library's kernels.
Weights are random-initialised on the device (N(0, 0.02^2), 0.1% outlier columns x20)
and rotated/quantized by the library; inputs are seeded N(0,1) bf16 vectors.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). With N > 1 (torchrun) every rank runs an independent
replica (the path has no exchange step); the time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on the host cores on a bounded sample of
the same workload (one block of the stack per step), in the same metric.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

N_LAYERS = 32
HIDDEN, FFN, NH, NKV, HD = 4096, 11008, 32, 32, 128
BITS, GROUP, BATCH = 2, 64, 1
WORKLOAD = 4
METRIC = "rotated 2-bit linear: decode tokens/s (7B-shaped, batch 1) and HBM GB/s vs roofline"
CONFIG_NAME = "llama2-7b-shaped 32-layer rotated 2-bit linear stack, batch-1 decode"
# with --rht every butterfly is the fixed randomized Hadamard transform (Theta = 0): the
# baseline the HARP pages compare against (same codes budget, no learned angles)
CONFIG_NAME_RHT = "llama2-7b-shaped 32-layer 2-bit linear stack with fixed randomized Hadamard rotations, batch-1 decode"
# with --int8-angles every butterfly keeps its angles in int8 (one step per stage), as the
# HARP pages' storage option; the layers are built from the dequantized angles
CONFIG_NAME_Q8 = "llama2-7b-shaped 32-layer rotated 2-bit linear stack with int8 butterfly angles, batch-1 decode"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=N_LAYERS)
    ap.add_argument("--cpu-sample-layers", type=int, default=1)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rht", action="store_true",
                    help="fixed randomized Hadamard rotations (Theta = 0) instead of the learned-angle butterflies")
    ap.add_argument("--int8-angles", action="store_true",
                    help="learned angles stored in int8 with a per-stage step (decoded in the kernels)")
    ap.add_argument("--config", type=int, default=4, choices=[1, 2, 3, 4, 5],
                    help="4 (default): the 7B 32-block decode stack; 1: one 1024x1024 layer; 2: the seven 7B "
                         "linears; 3: the batch sweep; 5: the 70B 80-block stack at 2/3/4 bits, batch 1 and 16. "
                         "Configs other than 4 print one JSON line per measured cell")
    ap.add_argument("--distinct-blocks", type=int, default=8,
                    help="config 5: distinct seeded blocks cycled over the 80 layers")
    args = ap.parse_args()
    if args.rht and args.int8_angles:
        ap.error("--rht and --int8-angles exclude each other")
    return args


def shapes():
    from rotated_bit_matmul_b200 import synth
    return synth.llama7b_linears()


def algorithmic_bytes_per_step(n_layers, batch=BATCH, bits=BITS):
    """Packed codes + fp16 scale/zero + fp32 activations in and out, per linear."""
    tot = 0
    for s in shapes():
        tot += s.n_out * s.n_in * bits // 8 + s.n_out * (s.n_in // GROUP) * 4 + 4 * batch * (s.n_in + s.n_out)
    return tot * n_layers


# DRAM bytes (read + write) of one fused decode launch per transformer block, from an
# ncu capture of the 4-block stack (dram__bytes_read.sum + dram__bytes_write.sum, scaled
# by blocks): 278.45 MB per 4-block launch with fp32 cos/sin tables, 270.19 MB with int8
# angles. With them, a hash of the kernel's sources at capture time: the figures are
# reported only while those sources are unchanged.
TRAFFIC_PER_BLOCK = {"bytes": {"fp32": 278_446_336 // 4, "int8": 270_192_384 // 4},
                     "sources_sha256_16": "dbd501af0bd7bebb"}
KERNEL_SOURCES = ("decode.cu", "decode.h", "common.cuh", "gemv_core.cuh", "bfly_engine.cuh")


def traffic_per_step(n_layers, angles="fp32"):
    import hashlib
    csrc = os.path.join(ROOT, "rotated_bit_matmul_b200", "csrc")
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest()[:16] != TRAFFIC_PER_BLOCK["sources_sha256_16"]:
        return None
    b = TRAFFIC_PER_BLOCK["bytes"][angles]
    return None if b is None else b * n_layers


def measured_tc_peak():
    """Dense bf16 tensor-core TFLOP/s from MEASURED_PEAKS.json (burst), else the fallback."""
    try:
        d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(d["bf16_tflops"])
    except Exception:
        return 1590.0


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks sampling
class ClockSampler:
    def __init__(self, index=0):
        self.index = index
        self.samples = []
        self._stop = threading.Event()
        self._th = None

    def _run(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                     "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            return
        try:
            while not self._stop.is_set():
                line = proc.stdout.readline()
                if not line:
                    break
                self.samples.append([t.strip() for t in line.split(",")])
        finally:
            proc.terminate()

    def __enter__(self):
        self._th = threading.Thread(target=self._run, daemon=True)
        self._th.start()
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._th.join(timeout=3)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4) if len(s) > 5 + i and s[5 + i] == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------ CPU oracle sample
def _oracle_block(sample_layers, rht=False, q8=False):
    import oracle
    from rotated_bit_matmul_b200 import synth
    lays = []
    for l in range(sample_layers):
        for i, s in enumerate(shapes()):
            W = synth.weights(s.n_out, s.n_in, WORKLOAD, l, i)
            thV, sV = synth.butterfly_params(s.n_in, s.w_in, WORKLOAD, l, i, "V")
            thU, sU = synth.butterfly_params(s.n_out, s.w_out, WORKLOAD, l, i, "U")
            if rht:
                thV, thU = np.zeros_like(thV), np.zeros_like(thU)
            if q8:
                thV = oracle.dequantize_angles(*oracle.quantize_angles(thV))
                thU = oracle.dequantize_angles(*oracle.quantize_angles(thU))
            lays.append(oracle.prepare_layer(W, BITS, s.w_in, s.w_out, thV, sV, thU, sU)[0])
    return lays


def cpu_oracle_sample(sample_layers=1, min_seconds=10.0, steps=None, warmup=0, rht=False, q8=False):
    """Times the fp64 oracle on `sample_layers` blocks of the 7B stack for one token per
    pass and scales to the 32-block step. Without `steps` it repeats passes until
    `min_seconds` of CPU work have been timed; with `steps` it runs `warmup` untimed and
    `steps` timed passes. Returns (tokens_per_s, seconds_per_block, threads, passes)."""
    import oracle
    from rotated_bit_matmul_b200 import synth
    threads = len(os.sched_getaffinity(0))
    oracle.set_threads(threads)
    lays = _oracle_block(sample_layers, rht, q8)
    for w in range(warmup):
        oracle.stack_step(lays, HIDDEN, FFN, NH, NKV, HD, synth.activations(BATCH, HIDDEN, WORKLOAD, step=w).astype(np.float64))
    passes, dt = 0, 0.0
    while (steps is not None and passes < steps) or (steps is None and (passes == 0 or dt < min_seconds)):
        x = synth.activations(BATCH, HIDDEN, WORKLOAD, step=warmup + passes).astype(np.float64)
        t0 = time.perf_counter()
        oracle.stack_step(lays, HIDDEN, FFN, NH, NKV, HD, x)
        dt += time.perf_counter() - t0
        passes += 1
    per_block = dt / (passes * sample_layers)
    return 1.0 / (per_block * N_LAYERS), per_block, threads, passes


# ------------------------------------------------------------------ GPU path
def build_stack(n_layers, device, rht=False, q8=False):
    import torch
    import rotated_bit_matmul_b200 as rb
    from rotated_bit_matmul_b200 import synth
    layers = []
    for l in range(n_layers):
        for i, s in enumerate(shapes()):
            W = synth.device_weights(s.n_out, s.n_in, WORKLOAD, l, i, device=device)
            thV, sV = synth.butterfly_params(s.n_in, s.w_in, WORKLOAD, l, i, "V")
            thU, sU = synth.butterfly_params(s.n_out, s.w_out, WORKLOAD, l, i, "U")
            thV, thU = torch.from_numpy(thV).to(device), torch.from_numpy(thU).to(device)
            if rht:  # Theta = 0 on both sides: no angles reach the library
                thV = thU = None
            sV, sU = torch.from_numpy(sV).to(device), torch.from_numpy(sU).to(device)
            if q8:  # int8 angles; W is rotated with the angles they stand for
                qV, dV = rb.harp_quantize_angles(thV)
                qU, dU = rb.harp_quantize_angles(thU)
                thV, thU = dV[:, None] * qV.float(), dU[:, None] * qU.float()
            Wr = rb.rotate_weights_device(W, thV, sV, s.w_in, thU, sU, s.w_out)
            del W
            codes, sz = rb.harp_quantize_weights(Wr, BITS, GROUP)
            del Wr
            if q8:
                layers.append(rb.HarpLayer.int8_angles(s.n_in, s.n_out, BITS, s.w_in, s.w_out, qV, dV, sV, qU, dU, sU,
                                                       codes, sz))
            else:
                layers.append(rb.HarpLayer(s.n_in, s.n_out, BITS, s.w_in, s.w_out, thV, sV, thU, sU, codes, sz))
    torch.cuda.synchronize()
    return rb.HarpStack(layers, HIDDEN, FFN, NH, NKV, HD)


def launches_per_step(n_layers, fused):
    if fused:
        return 1  # the fused decode-step kernel (its counter reset is a cudaMemsetAsync)
    # one convert + per block: 2 RMSNorm, 7 x (input butterfly, GEMV, output butterfly),
    # 2 residual adds, 1 SiLU*up (no repeat: 32 query heads over 32 kv heads) + one store
    return 1 + n_layers * (2 + 7 * 3 + 2 + 1) + 1


def run_ours(args, rk):
    import torch
    from rotated_bit_matmul_b200 import replicas, synth
    device = torch.device("cuda", rk.local_rank)
    torch.cuda.set_device(device)
    stack = build_stack(args.layers, device, args.rht, args.int8_angles)
    K, Wm = args.steps, args.warmup
    xs = torch.stack([torch.from_numpy(synth.activations(BATCH, HIDDEN, WORKLOAD, step=s)).to(torch.bfloat16)
                      for s in range(K + Wm)]).to(device)
    x_in = torch.empty((BATCH, HIDDEN), dtype=torch.bfloat16, device=device)
    y = torch.empty((BATCH, HIDDEN), dtype=torch.float32, device=device)
    ws = stack.workspace(BATCH)
    stream = torch.cuda.Stream(device)

    # warm-up (also first-use allocations), then capture one step into a CUDA graph
    with torch.cuda.stream(stream):
        for s in range(Wm):
            x_in.copy_(xs[s])
            stack.step(x_in, out=y, workspace=ws)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        stack.step(x_in, out=y, workspace=ws)
    stream.synchronize()
    with torch.cuda.stream(stream):  # the first replays upload the graph: keep them untimed
        for s in range(max(Wm, 3)):
            x_in.copy_(xs[s])
            g.replay()
    stream.synchronize()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    replicas.barrier(rk)
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for s in range(K):
                x_in.copy_(xs[Wm + s], non_blocking=True)
                g.replay()
            e1.record(stream)
        e1.synchronize()
    torch.cuda.synchronize()
    replicas.barrier(rk)
    ms = replicas.max_over_ranks(rk, e0.elapsed_time(e1), device)
    ms_step = ms / K
    value = replicas.whole_job_rate(rk, BATCH * K, ms)

    # end to end through the public API with host buffers: pinned H2D of the step's
    # input, the stack step, D2H of its output, every step
    xh = torch.stack([torch.from_numpy(synth.activations(BATCH, HIDDEN, WORKLOAD, step=s)).to(torch.bfloat16)
                      for s in range(K)]).pin_memory()
    yh = torch.empty((K, BATCH, HIDDEN), dtype=torch.float32).pin_memory()
    replicas.barrier(rk)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for s in range(K):
            x_in.copy_(xh[s], non_blocking=True)
            stack.step(x_in, out=y, workspace=ws)
            yh[s].copy_(y, non_blocking=True)
        e1.record(stream)
    e1.synchronize()
    replicas.barrier(rk)
    ms_e2e = replicas.max_over_ranks(rk, e0.elapsed_time(e1), device)
    e2e = {"value": replicas.whole_job_rate(rk, BATCH * K, ms_e2e), "unit": "tokens/s",
           "h2d_bytes_per_step": int(xh[0].numel() * xh.element_size()),
           "d2h_bytes_per_step": int(yh[0].numel() * yh.element_size())}

    nbytes = algorithmic_bytes_per_step(args.layers)
    peak, peak_kind = measured_peak()
    achieved = nbytes / (ms_step * 1e-3) / 1e9
    fused = stack.uses_fused_step(BATCH)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": (traffic_per_step(args.layers, "int8" if args.int8_angles else "fp32")
                            if fused and not args.rht else None),
                "kernel": "decode_kernel (one launch per step)" if fused else "whole decode step (graph of kernels)",
                "peak_kind": peak_kind, "algorithmic_bytes_per_step": nbytes}
    del g
    return dict(value=value, ms_step=ms_step, e2e=e2e, roofline=roofline, clocks=clk.summary(),
                launches=launches_per_step(args.layers, fused) * K, fused=fused)


# ------------------------------------------------------------------ configs 1, 2, 3, 5
def _line(metric, value, unit, higher, config, roofline, cpu=None, launches=None, clocks=None, dtype=None, extra=None):
    d = {"metric": metric, "value": value, "unit": unit, "n_gpus": 1, "higher_is_better": higher,
         "scaling": "weak", "vs_baseline": None, "dtype": dtype or "u2/u3/u4 codes x i16 or f16 activations",
         "data": "synthetic (seeded N(0,1) activations; random-init N(0,0.02^2) weights with 0.1% outlier columns)",
         "config": config, "roofline": roofline, "cpu_baseline": cpu, "gpu_launches": launches, "clocks": clocks}
    if extra:
        d.update(extra)
    print(json.dumps(d), flush=True)


def _oracle_linear_us(n_out, n_in, w_in, w_out, bits, batch, threads, seconds=10.0):
    """Times oracle.linear_fwd on one seeded layer (host-prepared) for about `seconds`."""
    import oracle
    from rotated_bit_matmul_b200 import synth
    oracle.set_threads(threads)
    W = synth.weights(n_out, n_in, 1, 0, 0)
    thV, sV = synth.butterfly_params(n_in, w_in, 1, 0, 0, "V")
    thU, sU = synth.butterfly_params(n_out, w_out, 1, 0, 0, "U")
    lay = oracle.prepare_layer(W, bits, w_in, w_out, thV, sV, thU, sU)[0]
    x = synth.activations(batch, n_in, 1, step=0, bf16=False).astype(np.float64)
    n, t0 = 0, time.perf_counter()
    while n == 0 or time.perf_counter() - t0 < seconds:
        oracle.linear_fwd(lay, x)
        n += 1
    return (time.perf_counter() - t0) / n * 1e6, n


def run_linear_configs(args):
    """Configs 1-3: single rotated linears through harp_linear_fwd, graph-replayed over
    enough distinct layers that each call streams its weights from HBM (cold L2)."""
    import torch
    from rotated_bit_matmul_b200 import linear_timing as lt
    peak, peak_kind = measured_peak()
    tc_peak = measured_tc_peak()
    threads = len(os.sched_getaffinity(0))
    if args.config == 1:
        with ClockSampler(0) as clk:
            r = lt.time_shape(1024, 1024, 1024, 1024, 2, [1], xdtype=torch.float32, min_layers=64)[0]
        us = r["us_per_call"]
        cpu = None
        if not args.no_cpu_baseline:
            o_us, n = _oracle_linear_us(1024, 1024, 1024, 1024, 2, 1, threads)
            o1, n1 = _oracle_linear_us(1024, 1024, 1024, 1024, 2, 1, 1, seconds=5.0)
            cpu = {"value": round(o_us, 1), "unit": "us/call", "cores": threads, "kind": "oracle",
                   "sample": f"{n} calls of the whole layer on {threads} threads; 1 thread: {o1:.1f} us ({n1} calls)"}
        ach = r["alg_bytes"] / us / 1e3
        _line("single 1024x1024 rotated 2-bit linear, batch 1: latency per call", us, "us/call", False,
              {"workload": "config 1: one 1024x1024 rotated 2-bit linear, fp32 x [1,1024], w 1024 both sides",
               "distinct_layers": r["layers"], "l2": "each call reads another of the layer copies (cold L2)"},
              {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s", "frac": round(ach / peak, 4),
               "traffic": None, "peak_kind": peak_kind, "algorithmic_bytes_per_call": r["alg_bytes"],
               "kernel": "whole harp_linear_fwd (3 launches)"},
              cpu=cpu, launches=3, clocks=clk.summary(), dtype="u2 codes x i16 activations -> i32 dot")
        return
    shapes = lt.SHAPES if args.config == 2 else lt.SHAPES[:2]
    batches = [1] if args.config == 2 else [1, 4, 16, 64, 256]
    names = {0: "q/k/v/o 4096x4096", 1: "gate/up 11008x4096", 2: "down 4096x11008"}
    mult = {0: 4, 1: 2, 2: 1}
    total_us, total_bytes = 0.0, 0
    for i, shp in enumerate(shapes):
        with ClockSampler(0) as clk:
            rows = lt.time_shape(*shp, 2, batches)
        fused = {}
        if args.config == 3 and shp[3] <= 256:
            # the output blocks of 256 finished inside the tensor-core kernel (opt-in)
            os.environ["HARP_MMA_FUSE"] = "1"
            try:
                fused = {r["batch"]: r["us_per_call"] for r in lt.time_shape(*shp, 2, [b for b in batches if b >= 16])}
            finally:
                del os.environ["HARP_MMA_FUSE"]
        for r in rows:
            us, B = r["us_per_call"], r["batch"]
            ach = r["alg_bytes"] / us / 1e3
            tf = r["tflops"]
            bound = "tensor" if B >= 64 else "hbm"
            roof = {"bound": bound, "achieved": round(ach, 1) if bound == "hbm" else tf,
                    "peak": peak if bound == "hbm" else tc_peak, "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
                    "frac": round((ach / peak) if bound == "hbm" else (tf / tc_peak), 4), "traffic": None,
                    "hbm_frac": round(ach / peak, 4), "tensor_frac": round(tf / tc_peak, 4),
                    "algorithmic_bytes_per_call": r["alg_bytes"], "peak_kind": peak_kind,
                    "kernel": "whole harp_linear_fwd: " + ("GEMV path" if B < 16 else "tcgen05 path")}
            _line(f"rotated 2-bit linear {names[i]}, batch {B}: time per call", us, "us/call", False,
                  {"workload": f"config {args.config}: {names[i]} rotated 2-bit linear, bf16 x [{B},{shp[1]}]",
                   "batch": B, "distinct_layers": r["layers"], "l2": "cold L2: distinct layer copies per call"},
                  roof, launches=3 if B < 16 else 4, clocks=clk.summary(),
                  extra={"fused_epilogue_us_per_call": fused[B]} if B in fused else None)
            if args.config == 2:
                total_us += mult[i] * us
                total_bytes += mult[i] * r["alg_bytes"]
    if args.config == 2:
        # the FFN side as one mixed-radix butterfly (11008 = 2^8 * 43) against 43 blocks of 256
        for side, nm in (("U", "gate/up 11008x4096, output side 2^8*43"), ("V", "down 4096x11008, input side 43*2^8")):
            with ClockSampler(0) as clk:
                m = lt.time_mixed_radix(side)
            ach = m["alg_bytes"] / m["us_mixed_radix"] / 1e3
            _line(f"rotated 2-bit linear {nm} mixed-radix, batch 1: time per call", m["us_mixed_radix"], "us/call",
                  False, {"workload": f"config 2: {nm} as one mixed-radix butterfly, bf16 x [1,{m['n_in']}]",
                          "batch": 1, "distinct_layers": m["layers"], "l2": "cold L2: distinct layer copies per call"},
                  {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                   "frac": round(ach / peak, 4), "traffic": None, "peak_kind": peak_kind,
                   "algorithmic_bytes_per_call": m["alg_bytes"], "kernel": "whole harp_linear_fwd, mixed-radix sides"},
                  launches=None, clocks=clk.summary(),
                  extra={"block_diagonal_us_per_call": m["us_block_diagonal"],
                         "mixed_radix_over_block_diagonal": round(m["us_mixed_radix"] / m["us_block_diagonal"], 3)})
        ach = total_bytes / total_us / 1e3
        _line("the seven linears of a 7B-shaped block, batch 1: time per block", round(total_us, 2), "us/block",
              False, {"workload": "config 2: q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008, batch 1",
                      "sum_of": "4 x q/k/v/o + 2 x gate/up + 1 x down calls"},
              {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s", "frac": round(ach / peak, 4),
               "traffic": None, "peak_kind": peak_kind, "kernel": "21 launches (3 per linear)"},
              launches=21)


def run_70b(args):
    """Config 5: the Llama-70B-shaped 80-block stack at 2, 3 and 4 bits, batch 1 and 16.
    Weights of `--distinct-blocks` seeded blocks are drawn on the device, rotated once and
    quantized at each bit width; the 80 layers cycle through them, so every step streams
    all 80 blocks' codes (a block is 0.27-0.48 GB, and the same weights come back only
    after distinct_blocks - 1 other blocks, far more than the 126 MB L2)."""
    import torch
    import rotated_bit_matmul_b200 as rb
    from rotated_bit_matmul_b200 import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hidden, ffn, nh, nkv, hd = synth.STACK_DIMS["70b"]
    shapes = synth.llama70b_linears()
    nl = 80
    D = max(1, min(args.distinct_blocks, nl))
    per_bits = {b: [] for b in (2, 3, 4)}  # bits -> list over distinct blocks of 7 HarpLayers
    for d in range(D):
        blk = {b: [] for b in per_bits}
        for i, s in enumerate(shapes):
            W = synth.device_weights(s.n_out, s.n_in, 5, d, i, device=dev)
            thV, sV = synth.butterfly_params(s.n_in, s.w_in, 5, d, i, "V")
            thU, sU = synth.butterfly_params(s.n_out, s.w_out, 5, d, i, "U")
            thV, thU = torch.from_numpy(thV).to(dev), torch.from_numpy(thU).to(dev)
            sV, sU = torch.from_numpy(sV).to(dev), torch.from_numpy(sU).to(dev)
            Wr = rb.rotate_weights_device(W, thV, sV, s.w_in, thU, sU, s.w_out)
            del W
            for b in per_bits:
                codes, sz = rb.harp_quantize_weights(Wr, b, GROUP)
                blk[b].append(rb.HarpLayer(s.n_in, s.n_out, b, s.w_in, s.w_out, thV, sV, thU, sU, codes, sz))
            del Wr
        for b in per_bits:
            per_bits[b].append(blk[b])
    torch.cuda.synchronize()
    peak, peak_kind = measured_peak()
    K, Wm = args.steps, args.warmup
    for bits, blocks in per_bits.items():
        handles = [blocks[l % D][i] for l in range(nl) for i in range(7)]
        S = rb.HarpStack(handles, hidden, ffn, nh, nkv, hd)
        for B in (1, 16):
            wbytes = sum(s.n_out * s.n_in * bits // 8 + s.n_out * (s.n_in // GROUP) * 4 for s in shapes) * nl
            abytes = sum(4 * B * (s.n_in + s.n_out) for s in shapes) * nl
            xs = torch.from_numpy(synth.activations(B, hidden, 5, step=0)).to(dev, torch.bfloat16)
            y = torch.empty((B, hidden), dtype=torch.float32, device=dev)
            ws = S.workspace(B)
            st = torch.cuda.Stream(dev)
            with torch.cuda.stream(st):
                for _ in range(Wm):
                    S.step(xs, out=y, workspace=ws)
            st.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st):
                S.step(xs, out=y, workspace=ws)
            with torch.cuda.stream(st):
                for _ in range(3):
                    g.replay()
            st.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with ClockSampler(0) as clk:
                with torch.cuda.stream(st):
                    e0.record(st)
                    for _ in range(K):
                        g.replay()
                    e1.record(st)
                e1.synchronize()
            ms = e0.elapsed_time(e1) / K
            del g
            ach = (wbytes + abytes) / (ms * 1e-3) / 1e9
            fused = S.uses_fused_step(B)
            _line(f"rotated {bits}-bit linear stack, Llama-70B-shaped, batch {B}: decode tokens/s", B / (ms * 1e-3),
                  "tokens/s", True,
                  {"workload": f"config 5: Llama-70B-shaped 80-block rotated {bits}-bit linear stack, batch-{B} decode",
                   "layers": nl, "distinct_blocks": D, "hidden": hidden, "ffn": ffn, "bits": bits, "batch": B,
                   "l2": "inputs larger than L2"},
                  {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s", "frac": round(ach / peak, 4),
                   "traffic": None, "peak_kind": peak_kind, "algorithmic_bytes_per_step": wbytes + abytes,
                   "kernel": "fused decode step" if fused else "per-linear path (graph of kernels)"},
                  launches=None, clocks=clk.summary(), extra={"ms_per_step": ms, "steps": K, "warmup": Wm})
        S.close()
    for blocks in per_bits.values():
        for blk in blocks:
            for L in blk:
                L.close()


def main():
    args = parse()
    if args.config != 4 and args.impl == "ours":
        if args.config == 5:
            run_70b(args)
        else:
            run_linear_configs(args)
        return
    from rotated_bit_matmul_b200 import replicas
    rk = replicas.from_env()
    # the reference arm is the CPU oracle: its ranks meet over gloo
    replicas.init(rk, "gloo" if args.impl == "reference" else "nccl")
    world = rk.world

    workload = CONFIG_NAME_RHT if args.rht else (CONFIG_NAME_Q8 if args.int8_angles else CONFIG_NAME)
    config = {"workload": workload, "layers": args.layers, "hidden": HIDDEN, "ffn": FFN, "bits": BITS,
              "group": GROUP, "batch": BATCH, "global_batch": BATCH * world, "parallelism": f"replicas{world}",
              "l2": "inputs larger than L2: each step streams ~2.03 GB of packed codes and scales (L2 126 MB)"}
    base = {"metric": METRIC, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "data": "synthetic (seeded N(0,1) bf16 inputs; random-init N(0,0.02^2) weights with 0.1% outlier columns)",
            "config": config}

    if args.impl == "reference":
        # rank 0 alone times the oracle; the other ranks leave without work
        if rk.rank == 0:
            tps, per_block, threads, passes = cpu_oracle_sample(args.cpu_sample_layers, steps=args.steps,
                                                                warmup=args.warmup, rht=args.rht,
                                                                q8=args.int8_angles)
            ms = per_block * N_LAYERS * 1e3
            line = dict(base, impl="reference", value=tps, unit="tokens/s", ms_per_step=ms, dtype="f64",
                        cpu_baseline={"value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                      "sample": f"each step: {args.cpu_sample_layers} of {N_LAYERS} blocks of one "
                                                f"decode token, scaled to {N_LAYERS} blocks"},
                        e2e={"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0})
            print(json.dumps(line), flush=True)
        replicas.finish(rk)
        return

    r = run_ours(args, rk)
    cpu = None
    if rk.rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, per_block, threads, passes = cpu_oracle_sample(args.cpu_sample_layers, rht=args.rht, q8=args.int8_angles)
        cpu = {"value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{passes} passes of {args.cpu_sample_layers} of {N_LAYERS} blocks of one decode token "
                         f"(about 10 s of CPU work), scaled to {N_LAYERS} blocks"}
    if rk.rank == 0:
        line = dict(base, value=r["value"], unit="tokens/s", ms_per_step=r["ms_step"],
                    dtype="u2 codes x i16 activations -> i32 dot, f32 elsewhere", roofline=r["roofline"],
                    cpu_baseline=cpu, e2e=r["e2e"], gpu_launches=r["launches"], clocks=r["clocks"])
        print(json.dumps(line), flush=True)
    replicas.finish(rk)


if __name__ == "__main__":
    main()
