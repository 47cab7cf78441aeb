#!/usr/bin/env python3
"""Benchmark of the block-scaled quantization hot path on B200.

One step is one pass of every hot-path operation over synthetic inputs that
are resident in HBM:
  1. mx_quantize     expert weights bf16 [64, 2048, 7168] -> packed + E8M0 scales
  2. grouped GEMM    forward  x bf16 [32768, 7168] . deq(W)^T, W [32, 2048, 7168]
  3. grouped GEMM    backward grad_out bf16 [32768, 2048] . deq(W)
  4. quantize_cache  KV-like bf16 [4, 8192, 512]: fp8 (block 128), mxfp4 (32), nvfp4 (16)
  5. mx_dequantize   the packed weights of step 1 back to bf16 [64, 2048, 7168]
Every kernel reads inputs last touched more than L2's 126 MB of traffic
earlier (the 2.4 GB pack/unpack passes and the GEMMs sit between reuses).

Printed metric: quant/dequant HBM GB/s = algorithmic bytes of steps 1, 4, 5
over their summed device time (CUDA events on the launching stream), with
the grouped-GEMM TFLOP/s beside it.  `--impl reference` times the scalar
CPU oracle instead, on a bounded sample of the same workload.

Multi-GPU (torchrun): every rank runs the same per-GPU workload (weak
scaling, no data exchange); timings are the max over ranks.
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "quant/dequant HBM GB/s (% of ~8 TB/s); MXFP4 grouped-GEMM TFLOPS (% of peak)"

# Workload sizes.
W_SHAPE = (64, 2048, 7168)
KV_SHAPE = (4, 8192, 512)
CACHE_RUNS = (("fp8", 128), ("mxfp4", 32), ("nvfp4", 16))
T, E, N, K = 32768, 32, 2048, 7168
WORKLOAD = ("mx_quantize + mx_dequantize of expert weights bf16 [64,2048,7168]; "
            "quantize_cache fp8/128, mxfp4/32, nvfp4/16 of KV bf16 [4,8192,512]; "
            "MXFP4 grouped GEMM fwd + dgrad, x [32768,7168], W [32,2048,7168], "
            "multinomial expert counts")


def algorithmic_bytes():
    w = W_SHAPE[0] * W_SHAPE[1] * W_SHAPE[2]
    kv = KV_SHAPE[0] * KV_SHAPE[1] * KV_SHAPE[2]
    return {
        # read bf16, write packed nibbles + one scale byte per 32
        "mx_quantize": w * 2 + w // 2 + w // 32,
        "mx_dequantize": w // 2 + w // 32 + w * 2,
        # read and write bf16
        "quantize_cache": kv * 4,
    }


def gemm_flops():
    return 2.0 * T * N * K


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(name):
    """Hash of a kernel's translation unit and every header beside it (the
    device helpers it includes), so that a profile taken before a change to
    either no longer counts."""
    csrc = os.path.join(ROOT, "nvfp4_quantization_amax_b200", "csrc")
    h = hashlib.sha256()
    headers = sorted(f for f in os.listdir(csrc) if f.endswith((".cuh", ".h")))
    for f in [name] + headers:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key, src):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel's source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    ent = t.get(kernel_key)
    if not ent or ent.get("source_sha") != source_hash(src):
        return None
    return ent.get("dram_bytes_per_launch")


# --------------------------------------------------------------- clocks

REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


def gpu_id(torch, dev):
    """nvidia-smi -i selector for a torch device (its UUID)."""
    u = str(torch.cuda.get_device_properties(dev).uuid)
    return u if u.startswith("GPU-") else "GPU-" + u


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while running."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        cmd = ["nvidia-smi", "-i", str(self.index),
               "--query-gpu=timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
               "--format=csv,noheader,nounits", "-lms", "20"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0=None, t1=None):
        """Clocks while the GPU ran the timed region: the samples whose
        nvidia-smi timestamp falls in [t0, t1] (host wall-clock seconds of
        the region's start and of its closing synchronize)."""
        samples = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 5:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, mx, mask = float(parts[1]), float(parts[2]), int(parts[4], 16)
            except ValueError:
                continue
            try:
                watts = float(parts[3])
            except ValueError:  # "[N/A]"
                watts = None
            samples.append((ts, sm, mx, watts, mask))
        if not samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        window = [x for x in samples if t0 is not None and t0 <= x[0] <= t1]
        used = window if window else samples
        reasons = set()
        for x in used:
            for bit, name in REASON_BITS.items():
                if x[4] & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(x[1] for x in used),
                "sm_min_mhz": min(x[1] for x in used), "sm_max_mhz": used[-1][2],
                "power_w_median": (round(statistics.median(w), 1)
                                   if (w := [x[3] for x in used if x[3] is not None]) else None),
                "reasons": sorted(reasons), "samples": len(used),
                "window": "timed region" if window else "whole sampler run (no sample in the region)"}


# ------------------------------------------------------------ GPU arm

class Step:
    """Device-resident inputs and outputs of one step, and the step itself."""

    def __init__(self, torch, mxq, gen, dev):
        self.torch, self.mxq = torch, mxq
        self.W = gen.expert_weights(*W_SHAPE, device=dev)
        self.P, self.S = mxq.mx_quantize(self.W)
        self.Wout = torch.empty_like(self.W)
        self.kv = [gen.kv_cache(KV_SHAPE, device=dev, seed_base=10 * i) for i in range(3)]
        self.kv_out = [torch.empty_like(k) for k in self.kv]
        W5 = gen.expert_weights(E, N, K, device=dev, workload=5)
        self.P5, self.S5 = mxq.mx_quantize(W5)
        del W5
        self.x = gen.normal_bf16(gen.seed_for(5, 3), (T, K), device=dev)
        self.g = gen.normal_bf16(gen.seed_for(5, 4), (T, N), device=dev)
        counts = gen.expert_counts(T, E, device=dev)
        self.offs = torch.cumsum(counts, 0).to(torch.int32)
        self.y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
        self.gx = torch.empty((T, K), dtype=torch.bfloat16, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.names = ["mx_quantize", "gemm_fwd", "gemm_dgrad", "qc_fp8", "qc_mxfp4", "qc_nvfp4",
                      "mx_dequantize"]

    def run(self, ev=None):
        m = self.mxq
        calls = [
            lambda: m.mx_quantize(self.W, self.P, self.S),
            lambda: m.mxfp4_grouped_mm(self.x, self.P5, self.S5, self.offs, False, self.y,
                                       self.status),
            lambda: m.mxfp4_grouped_mm(self.g, self.P5, self.S5, self.offs, True, self.gx,
                                       self.status),
        ] + [
            (lambda i=i, f=f, b=b: m.quantize_cache(self.kv[i], f, b, self.kv_out[i]))
            for i, (f, b) in enumerate(CACHE_RUNS)
        ] + [lambda: m.mx_dequantize(self.P, self.S, self.torch.bfloat16, self.Wout)]
        for i, c in enumerate(calls):
            if ev is not None:
                ev[i][0].record()
            c()
            if ev is not None:
                ev[i][1].record()


def time_next_rows(torch, mxq, step, dev, reps=3):
    """Device time (ms, mean over reps, max over ranks) of the next-row
    kernels: NVFP4 two-level quantize (max and mse block-scale rules) and
    dequantize on the expert weights; packed cache quantize / unpack on the
    three KV-cache tensors; the W4A4 GEMMs.  Timed after, and outside, the
    main step, each call on an L2 flushed before it."""
    packed, bscales, g = mxq.nvfp4_quantize(step.W)
    packed2, bscales2, g2 = mxq.nvfp4_quantize(step.W)
    ws = torch.empty(16, dtype=torch.uint8, device=dev)
    calls = {
        "nvfp4_quantize": lambda: mxq.nvfp4_quantize(step.W, packed, bscales, g, ws),
        "nvfp4_quantize_mse": lambda: mxq.nvfp4_quantize(step.W, packed2, bscales2, g2, ws,
                                                         rule="mse"),
        "nvfp4_dequantize": lambda: mxq.nvfp4_dequantize(packed, bscales, g, torch.bfloat16,
                                                         step.Wout),
    }
    for i, (f, b) in enumerate(CACHE_RUNS):
        codes, sc = mxq.quantize_cache_packed(step.kv[i], f, b)
        calls["cache_pack_" + f] = (
            lambda i=i, f=f, b=b, c=codes, s=sc: mxq.quantize_cache_packed(step.kv[i], f, b, c, s))
        calls["cache_unpack_" + f] = (
            lambda i=i, f=f, b=b, c=codes, s=sc: mxq.dequantize_cache_packed(
                c, s, f, b, torch.bfloat16, step.kv_out[i]))
    # W4A4: the benchmark GEMM with MXFP4 activations (quantized inside the call)
    xq, xs = mxq.mx_quantize(step.x)
    calls["w4a4_grouped_mm"] = lambda: mxq.w4a4_grouped_mm(step.x, step.P5, step.S5, step.offs,
                                                           step.y, step.status, xq, xs)
    # ... and in NVFP4 (each expert's weight quantized as its own tensor)
    import synthetic as gen
    W5 = gen.expert_weights(E, N, K, device=dev, workload=5)
    nvq = [mxq.nvfp4_quantize(W5[e]) for e in range(E)]
    del W5
    nvp = torch.stack([q[0] for q in nvq])
    nvs = torch.stack([q[1] for q in nvq])
    nvg = torch.cat([q[2] for q in nvq])
    del nvq
    calls["nvfp4_w4a4_grouped_mm"] = lambda: mxq.nvfp4_w4a4_grouped_mm(
        step.x, nvp, nvs, nvg, step.offs, step.y, step.status)
    # the block-scaled GEMMs alone, on activations quantized beforehand
    calls["_w4a4_gemm"] = lambda: mxq.w4a4_grouped_mm(None, step.P5, step.S5, step.offs, step.y,
                                                      step.status, x_quantized=(xq, xs))
    nx = mxq.nvfp4_quantize(step.x)
    calls["_nvfp4_w4a4_gemm"] = lambda: mxq.nvfp4_w4a4_grouped_mm(
        None, nvp, nvs, nvg, step.offs, step.y, step.status, x_quantized=nx)
    # Before each timed call a 256 MB write flushes L2 (126 MB) and keeps the
    # GPU busy while the host queues the call, so each event pair holds the
    # call's own kernels on cold inputs and no host launch overhead.
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = {}
    for name, fn in calls.items():
        for _ in range(2):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        torch.cuda.synchronize()
        for a, b in ev:
            flush.zero_()
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        out[name] = sum(a.elapsed_time(b) for a, b in ev) / reps
    names = list(out)
    vals = max_over_ranks([out[n] for n in names], dev)
    times = dict(zip(names, vals))
    # work of the mse sweep: evaluations of expert 0's blocks under the
    # tensor's g (the same i.i.d. weights in every expert)
    blocks0 = W_SHAPE[1] * W_SHAPE[2] // 16
    times["_mse_evals_per_block"] = mse_evaluations(torch, step.W[0], float(g2.item())) / blocks0
    return times


E4M3_POS_CODES = 126  # positive finite E4M3 bytes 0x01 .. 0x7E


def mse_evaluations(torch, w, g, lanes=1):
    """(candidate, weight) evaluations the mse-rule kernel performs on the
    16-blocks of w (bf16 [rows, K]) under the global scale g, replaying its
    pruning (the measurement's work unit, not a result): each block's codes
    are visited from the top (the first code whose quotient amax / d_c is at
    most 0.25, by binary search, else 126) downwards, `lanes` interleaved
    slots (the kernel's lanes per block: one) each stopping at the first code
    whose d underflows to 0 or whose clipping error (amax - 6 d)^2 alone
    exceeds the slot's best sum so far.
    Each visit evaluates 16 weights.  Error sums are formed in float64 from
    float32 quotients as in the kernel; a sum that differs from the kernel's
    in its last bits can move a stop by one code, so the count is exact up to
    such margins."""
    f32, f64 = torch.float32, torch.float64
    dev = w.device
    x = w.reshape(-1, 16).to(f32)
    ax = x.abs()
    amax = ax.amax(1)
    codes = torch.arange(E4M3_POS_CODES + 1, device=dev)
    # E4M3 value of each code byte: exponent field (bits 3-6), mantissa bits 0-2
    e, m = (codes >> 3) & 15, codes & 7
    s_c = torch.where(e == 0, m.to(f32) * 2.0 ** -9, (1.0 + m.to(f32) / 8.0) * torch.pow(
        torch.tensor(2.0, device=dev), (e - 7).to(f32)))
    d_c = (s_c * torch.tensor(g, dtype=f32, device=dev)).to(f32)

    def all_zero(c):
        dc = d_c[c]
        return (dc != 0) & ((amax / dc) <= 0.25)
    # c_top: binary search for the first all-zero code where code 126 is all-zero
    lo = torch.ones_like(amax, dtype=torch.int64)
    hi = torch.full_like(lo, E4M3_POS_CODES)
    top_zero = all_zero(hi)
    for _ in range(8):
        mid = (lo + hi) >> 1
        z = all_zero(mid)
        hi = torch.where(z & (lo < hi), mid, hi)
        lo = torch.where(~z & (lo < hi), mid + 1, lo)
    c_top = torch.where(top_zero, lo, torch.full_like(lo, E4M3_POS_CODES))
    mids = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=f32, device=dev)
    table = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=f64, device=dev)
    amax64, ax64 = amax.to(f64), ax.to(f64)
    total = 0
    for slot in range(lanes):
        best = torch.full_like(amax64, float("inf"))
        alive = torch.ones_like(amax, dtype=torch.bool)
        for k in range(E4M3_POS_CODES):
            c = c_top - slot - lanes * k
            alive &= c >= 1
            if not bool(alive.any()):
                break
            cc = c.clamp(min=1)
            d = d_c[cc]
            alive &= d != 0
            t = amax64 - 6.0 * d.to(f64)
            alive &= ~((t > 0) & (t * t * (1.0 - 2.0 ** -40) > best))
            total += int(alive.sum()) * 16
            v = ax / d[:, None]
            idx = torch.bucketize(v, mids)
            idx += ((v == 0.75) | (v == 1.75) | (v == 3.5)).to(idx.dtype)
            err = ((table[idx] * d.to(f64)[:, None] - ax64) ** 2).sum(1)
            better = alive & (err <= best)
            best = torch.where(better, err, best)
    return total


def mse_roofline(evals_s, clocks):
    """Issue-rate roofline of the mse sweep.  Unit: one (candidate, weight)
    evaluation.  The kernel's thread instructions per evaluation come from
    an ncu count (profiles/mse_issue.json: smsp__thread_inst_executed.sum of
    one launch over the evaluations the replay counts for that launch); the
    peak is every SM sub-partition issuing one full warp instruction per
    clock: 148 x 4 x 32 thread instructions per cycle at the maximum SM
    clock (the sweep runs outside the timed step, whose sampled clock may
    sit lower under the power cap)."""
    path = os.path.join(ROOT, "profiles", "mse_issue.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        prof = json.load(f)
    if prof.get("source_sha") != source_hash("nvfp4_mse.cu"):
        return None
    mhz = (clocks or {}).get("sm_max_mhz") or 1965.0
    per_eval = prof["thread_inst_per_eval"]
    peak = 148 * 4 * 32 * mhz * 1e6 / per_eval
    return {"bound": "issue", "unit": "G evaluations/s", "achieved": round(evals_s / 1e9, 2),
            "peak": round(peak / 1e9, 2), "frac": round(evals_s / peak, 4),
            "thread_inst_per_eval": per_eval, "sm_mhz": mhz,
            "peak_source": "148 SMs x 4 schedulers x 32 lanes per clock"}


def next_row_bytes():
    """Algorithmic HBM bytes of each next-row call (bf16 inputs/outputs)."""
    w = W_SHAPE[0] * W_SHAPE[1] * W_SHAPE[2]
    n = KV_SHAPE[0] * KV_SHAPE[1] * KV_SHAPE[2]
    # NVFP4 quantize: the per-tensor scale needs the whole tensor's maximum
    # first, so x is read twice; packed codes + E4M3 scales written once
    nb = {"nvfp4_quantize": 2 * 2 * w + w // 2 + w // 16,
          "nvfp4_quantize_mse": 2 * 2 * w + w // 2 + w // 16,
          "nvfp4_dequantize": w // 2 + w // 16 + 2 * w}
    for f, b in CACHE_RUNS:
        stored = (n if f == "fp8" else n // 2) + n // b
        nb["cache_pack_" + f] = 2 * n + stored
        nb["cache_unpack_" + f] = stored + 2 * n
    return nb


def time_e2e(torch, mxq, step, steps):
    """Same metric through the public API with host buffers: every call
    copies its inputs from pinned host memory to the device and its results
    back into pinned host outputs that the caller passed.  One untimed step
    first, so that no allocation is timed."""
    def pinned(t):
        return torch.empty(t.shape, dtype=t.dtype, pin_memory=True)

    hW = step.W.cpu().pin_memory()
    hP, hS = step.P.cpu().pin_memory(), step.S.cpu().pin_memory()
    hkv = [k.cpu().pin_memory() for k in step.kv]
    oP, oS, oW = pinned(hP), pinned(hS), pinned(hW)
    okv = [pinned(k) for k in hkv]
    h2d = hW.numel() * 2 + hP.numel() + hS.numel() + sum(k.numel() * 2 for k in hkv)
    d2h = oP.numel() + oS.numel() + oW.numel() * 2 + sum(k.numel() * 2 for k in okv)

    def one_step():
        mxq.mx_quantize(hW, oP, oS)
        for k, o, (f, b) in zip(hkv, okv, CACHE_RUNS):
            mxq.quantize_cache(k, f, b, o)
        mxq.mx_dequantize(hP, hS, torch.bfloat16, oW)

    one_step()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(steps):
        one_step()
    torch.cuda.synchronize()
    dt = (time.perf_counter() - t0) / steps
    return dt, h2d, d2h


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings (identity on one process)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def run_gpu(args, rank, world):
    import torch
    import torch.distributed as dist

    import nvfp4_quantization_amax_b200 as mxq
    import synthetic as gen

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        # a short limit: a rank that never arrives ends the others' barrier
        # or all-reduce with an error instead of a long hang
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(minutes=3))
    step = Step(torch, mxq, gen, dev)
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    if int(step.status.item()) != 0:
        raise RuntimeError("grouped GEMM reported status %d" % int(step.status.item()))

    # One pair of events per kernel and step, read after the closing
    # synchronize: the host queues the steps back to back, so no kernel
    # starts on an idle GPU and no event pair spans host launch overhead.
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in step.names]
          for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_id(torch, dev)) as clk:
        t_region = time.time()
        start.record()
        for k in range(args.steps):
            step.run(ev[k])
        stop.record()
        torch.cuda.synchronize()
        t_region = (t_region, time.time())
    if world > 1:
        dist.barrier()
    if int(step.status.item()) != 0:
        raise RuntimeError("grouped GEMM reported status %d" % int(step.status.item()))
    total_ms = start.elapsed_time(stop)
    kern_ms = {n: sum(ev[k][i][0].elapsed_time(ev[k][i][1]) for k in range(args.steps)) / args.steps
               for i, n in enumerate(step.names)}
    red = max_over_ranks([total_ms] + [kern_ms[n] for n in step.names], dev)
    total_ms = red[0]
    kern_ms = dict(zip(step.names, red[1:]))

    e2e_dt, h2d, d2h = time_e2e(torch, mxq, step, max(1, min(args.steps, 3)))
    e2e_dt = max_over_ranks([e2e_dt], dev)[0]
    next_ms = time_next_rows(torch, mxq, step, dev)
    extra = {}
    if world == 1:
        # the small-workload latency and the mixed-block sweep, outside the
        # timed step (the sweep needs ~68 GB, so the step's tensors go first)
        extra["config1_latency"] = time_config1(torch, mxq, gen, dev)
        del step
        torch.cuda.empty_cache()
        if not args.no_sweep:
            extra["sweep"] = time_sweep(torch, mxq, gen, dev, args.sweep_max_log2)

    if rank == 0:
        report(args, world, total_ms, kern_ms, e2e_dt, h2d, d2h, clk.summary(*t_region), next_ms,
               extra)
    if world > 1:
        dist.destroy_process_group()


def report(args, world, total_ms, kern_ms, e2e_dt, h2d, d2h, clocks, next_ms=None, extra=None):
    peaks, peak_src = load_peaks()
    ab = algorithmic_bytes()
    qd_bytes = ab["mx_quantize"] + ab["mx_dequantize"] + 3 * ab["quantize_cache"]
    qd_ms = kern_ms["mx_quantize"] + kern_ms["mx_dequantize"] + \
        sum(kern_ms[n] for n in ("qc_fp8", "qc_mxfp4", "qc_nvfp4"))
    gbs = qd_bytes / (qd_ms * 1e-3) / 1e9 * world
    gemm_ms = kern_ms["gemm_fwd"] + kern_ms["gemm_dgrad"]
    tflops = 2 * gemm_flops() / (gemm_ms * 1e-3) / 1e12 * world
    kernels = {}
    for n, ms in kern_ms.items():
        if n.startswith("gemm"):
            tf = gemm_flops() / (ms * 1e-3) / 1e12
            kernels[n] = {"ms": round(ms, 4), "tflops": round(tf, 1),
                          "frac": round(tf / peaks["bf16_tflops"], 4)}
        else:
            b = ab["quantize_cache"] if n.startswith("qc_") else ab[n]
            g = b / (ms * 1e-3) / 1e9
            kernels[n] = {"ms": round(ms, 4), "gbs": round(g, 1),
                          "frac": round(g / peaks["hbm_gbs"], 4)}
    dominant = max(kern_ms, key=kern_ms.get)
    if dominant.startswith("gemm"):
        ach = gemm_flops() / (kern_ms[dominant] * 1e-3) / 1e12
        roof = {"kernel": dominant, "bound": "tensor", "achieved": round(ach, 1),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(ach / peaks["bf16_tflops"], 4),
                "traffic": profiled_traffic(dominant, "grouped_mm_tc.cu"),
                "peak_source": peak_src + " bf16 burst"}
    else:
        b = ab["quantize_cache"] if dominant.startswith("qc_") else ab[dominant]
        ach = b / (kern_ms[dominant] * 1e-3) / 1e9
        roof = {"kernel": dominant, "bound": "hbm", "achieved": round(ach, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                "traffic": profiled_traffic(dominant, "elementwise.cu"),
                "peak_source": peak_src + " copy"}
    e2e_gbs = qd_bytes / e2e_dt / 1e9 * world
    line = {
        "metric": METRIC,
        "value": round(gbs, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64 / Box-Muller inputs of the configured shapes)",
        "config": {
            "workload": WORKLOAD,
            "hbm_fraction_nominal_8tbs": round(gbs / world / 8000.0, 4),
            "l2": "no flush; every kernel's inputs were last touched >126 MB of traffic earlier",
            "parallelism": "replicas" if world > 1 else "single GPU",
        },
        "gemm": {"value": round(tflops, 1), "unit": "TFLOP/s",
                 "frac_of_measured_burst": round(tflops / world / peaks["bf16_tflops"], 4),
                 "frac_of_measured_sustained":
                     round(tflops / world / peaks["bf16_tflops_sustained"], 4),
                 "frac_of_nominal_2250": round(tflops / world / 2250.0, 4)},
        "kernels": kernels,
        "roofline": roof,
        "e2e": {"value": round(e2e_gbs, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": 7 * args.steps,
        "clocks": clocks,
    }
    if next_ms:
        evals_per_block = next_ms.pop("_mse_evals_per_block", None)
        nb = next_row_bytes()
        w = W_SHAPE[0] * W_SHAPE[1] * W_SHAPE[2]
        rows = {}
        w4 = next_ms.pop("w4a4_grouped_mm", None)
        nv4 = next_ms.pop("nvfp4_w4a4_grouped_mm", None)
        w4g = next_ms.pop("_w4a4_gemm", None)
        nv4g = next_ms.pop("_nvfp4_w4a4_gemm", None)
        fp4_peak = 4.0 * peaks["bf16_tflops"]

        def gemm_alone(ms):
            tf = gemm_flops() / (ms * 1e-3) / 1e12
            return {"ms": round(ms, 4), "tflops": round(tf, 1),
                    "frac_of_fp4_peak": round(tf / fp4_peak, 4),
                    "includes": "the block-scaled GEMM on activations quantized beforehand"}
        for n, ms in next_ms.items():
            gbs = nb[n] / (ms * 1e-3) / 1e9
            rows[n] = {"ms": round(ms, 4), "gbs": round(gbs, 1),
                       "frac": round(gbs / peaks["hbm_gbs"], 4),
                       "workload": ("bf16 [64,2048,7168] expert weights" if n.startswith("nvfp4")
                                    else "bf16 [4,8192,512] KV cache")}
        # the sweep is arithmetic: at most 126 candidate scales x 16 weights
        # per block, of which the kernel evaluates only those that can win
        mse = rows["nvfp4_quantize_mse"]
        mse["bound"] = "issue"
        mse["g_candidates_per_s"] = round(126 * w / (next_ms["nvfp4_quantize_mse"] * 1e-3) / 1e9, 1)
        if evals_per_block is not None:
            evals_s = evals_per_block * (w // 16) / (next_ms["nvfp4_quantize_mse"] * 1e-3)
            mse["evaluations_per_block"] = round(evals_per_block, 3)
            mse["g_evaluations_per_s"] = round(evals_s / 1e9, 2)
            mse["roofline"] = mse_roofline(evals_s, clocks)
        if w4 is not None:
            # fp4 peak: the measured bf16 burst x the nominal fp4 / bf16 ratio (9 / 2.25)
            tf = gemm_flops() / (w4 * 1e-3) / 1e12
            rows["w4a4_grouped_mm"] = {
                "ms": round(w4, 4), "tflops": round(tf, 1),
                "frac_of_fp4_peak": round(tf / (4.0 * peaks["bf16_tflops"]), 4),
                "includes": "mx_quantize of the activations + the block-scaled GEMM",
                "workload": "x bf16 [32768,7168], W MXFP4 [32,2048,7168], multinomial counts"}
            if w4g is not None:
                rows["w4a4_grouped_mm"]["gemm"] = gemm_alone(w4g)
        if nv4 is not None:
            tf = gemm_flops() / (nv4 * 1e-3) / 1e12
            rows["nvfp4_w4a4_grouped_mm"] = {
                "ms": round(nv4, 4), "tflops": round(tf, 1),
                "frac_of_fp4_peak": round(tf / (4.0 * peaks["bf16_tflops"]), 4),
                "includes": "nvfp4_quantize of the activations (two passes) + the block-scaled GEMM",
                "workload": "x bf16 [32768,7168], W NVFP4 [32,2048,7168], multinomial counts"}
            if nv4g is not None:
                rows["nvfp4_w4a4_grouped_mm"]["gemm"] = gemm_alone(nv4g)
        line["next_rows"] = rows
    if extra:
        line.update(extra)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    print(json.dumps(line), flush=True)


# ------------------------------------------------------ CPU oracle arm

def host_cpu():
    """Host cores this process may use and the CPU model, read at run time."""
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return int(cores or 1), model


def sampled_rows(offs, per_expert=16, seed=8):
    """Every expert's first and last row plus `per_expert` seeded rows."""
    import numpy as np

    rng = np.random.default_rng(seed)
    starts = np.concatenate([[0], offs[:-1]])
    rows = []
    for lo, hi in zip(starts, offs):
        if hi > lo:
            rows += [lo, hi - 1] + list(rng.integers(lo, hi, per_expert))
    return np.unique(np.array(rows, np.int64))


def cpu_baseline(budget_s):
    """The scalar oracle, as it stands, timed on the host cores on bounded
    samples of the same workload: single-threaded, and the same source built
    with OpenMP on every core this process may use.  GB/s over the same
    algorithmic bytes per element as the GPU metric; the grouped GEMM as
    GFLOP/s of the exact double sums over every expert's first and last row
    plus 16 seeded rows (the oracle dequantizes each expert it touches)."""
    import numpy as np
    import torch

    import oracle
    import synthetic as gen

    cores, model = host_cpu()
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"  # input generation only
    per = max(budget_s / 8.0, 0.4)

    def timed(fn, bytes_per_call):
        n, t0 = 0, time.perf_counter()
        while True:
            fn()
            n += 1
            dt = time.perf_counter() - t0
            if dt >= per:
                return n * bytes_per_call, dt, n

    def bf16_bits(t):
        return t.cpu().view(torch.int16).numpy().view(np.uint16)

    def quant_dequant_cache(w_rows, kv_rows):
        W = gen.expert_weights(1, w_rows, 7168).view(w_rows, 7168)
        wb = bf16_bits(W)
        pk, sc = oracle.mx_quantize(wb)
        kv = bf16_bits(gen.kv_cache((1, kv_rows, 512)).view(kv_rows, 512))
        e_w, e_kv = w_rows * 7168, kv_rows * 512
        b1, t1, n1 = timed(lambda: oracle.mx_quantize(wb), e_w * 2 + e_w // 2 + e_w // 32)
        b2, t2, n2 = timed(lambda: oracle.mx_dequantize(pk, sc), e_w // 2 + e_w // 32 + e_w * 2)

        def qc():
            for f, b in CACHE_RUNS:
                oracle.quantize_cache(kv, f, b)
        b3, t3, n3 = timed(qc, 3 * e_kv * 4)
        return (b1 + b2 + b3) / (t1 + t2 + t3) / 1e9, (n1, n2, n3), t1 + t2 + t3

    gbs1, n_1, t_1 = quant_dequant_cache(16, 64)
    with oracle.all_cores():
        gbs_all, n_all, t_all = quant_dequant_cache(max(16, 8 * cores), max(64, 32 * cores))

    # grouped GEMM forward on the benchmark's inputs (W packed by the oracle)
    counts = gen.expert_counts(T, E).numpy()
    offs = np.cumsum(counts).astype(np.int32)
    rows = sampled_rows(offs)
    W5 = gen.expert_weights(E, N, K, device=gen_dev, workload=5)
    with oracle.all_cores():
        p5, s5 = oracle.mx_quantize(bf16_bits(W5.view(E * N, K)))
    del W5
    p5, s5 = p5.reshape(E, N, K // 2), s5.reshape(E, N, K // 32)
    a = bf16_bits(gen.normal_bf16(gen.seed_for(5, 3), (T, K), device=gen_dev))
    first = rows[rows < offs[0]]  # one expert's rows, single-threaded
    t0 = time.perf_counter()
    oracle.grouped_mm(a, p5, s5, offs, rows=first)
    g1 = 2.0 * first.size * N * K / (time.perf_counter() - t0) / 1e9
    with oracle.all_cores():
        t0 = time.perf_counter()
        oracle.grouped_mm(a, p5, s5, offs, rows=rows)
        g_all = 2.0 * rows.size * N * K / (time.perf_counter() - t0) / 1e9
    return {"value": round(gbs1, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "gbs_all_cores": round(gbs_all, 4), "cores_all": cores, "cpu_model": model,
            "gemm_gflops": round(g1, 4), "gemm_rows": int(first.size),
            "gemm_gflops_all_cores": round(g_all, 4), "gemm_rows_all_cores": int(rows.size),
            "sample": ("single thread: mx_quantize %dx and mx_dequantize %dx of [16,7168] weight "
                       "rows, quantize_cache (3 formats) %dx of [64,512] KV rows, %.1f s; "
                       "all %d cores (OpenMP build of the same source): %dx/%dx of [%d,7168] and "
                       "%dx of [%d,512], %.1f s; grouped GEMM forward of the benchmark inputs "
                       "(T=32768, E=32, N=2048, K=7168): first and last row plus 16 seeded rows "
                       "per expert (%d rows) on all cores, expert 0's %d of them single-threaded"
                       % (n_1[0], n_1[1], n_1[2], t_1, cores, n_all[0], n_all[1],
                          max(16, 8 * cores), n_all[2], max(64, 32 * cores), t_all,
                          rows.size, first.size))}


def time_config1(torch, mxq, gen, dev, reps=20):
    """Latency of the small MXFP4 workload (bf16 [64,256] with its four forced
    rows): mx_quantize and mx_dequantize, microseconds, median of `reps`
    calls after 5 warm-up calls, L2 flushed before each call."""
    x = gen.mx_small(dev)
    p, s = mxq.mx_quantize(x)
    y = torch.empty_like(x)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = {}
    for name, fn in (("mx_quantize", lambda: mxq.mx_quantize(x, p, s)),
                     ("mx_dequantize", lambda: mxq.mx_dequantize(p, s, torch.bfloat16, y))):
        for _ in range(5):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) * 1e3)
        out[name] = round(statistics.median(ts), 2)
    return {"unit": "us", "workload": "bf16 [64,256], 4 forced rows",
            "timing": "median of %d, L2 flushed before each call" % reps, **out}


def time_sweep(torch, mxq, gen, dev, max_log2=21, min_log2=10):
    """Bandwidth sweep over row counts of the mixed-block workload x bf16
    [R, 7168] (normal, subnormal-range, zero and single-spike 32-blocks):
    mx_quantize, mx_dequantize and quantize_cache in the three formats, device
    time per call (CUDA events, median of 5 after 2 warm-up calls; L2 is
    flushed before each timed call).  R = 2^10, 2^12, ..., 2^20, 2^21 (those
    from 2^min_log2 to 2^max_log2)."""
    C = 7168
    r_max = 1 << max_log2
    x = gen.mixed_blocks(r_max, C, device=dev)
    out = torch.empty_like(x)
    packed = torch.empty((r_max, C // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((r_max, C // 32), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    rows_out = []
    logs = sorted(set(list(range(10, min(max_log2, 20) + 1, 2)) + [max_log2]))
    logs = [lg for lg in logs if lg >= min_log2] or [max_log2]
    for lg in logs:
        R = 1 << lg
        xr, outr, pr, sr = x[:R], out[:R], packed[:R], scales[:R]
        mxq.mx_quantize(xr, pr, sr)
        n = R * C
        calls = {
            "mx_quantize": (lambda: mxq.mx_quantize(xr, pr, sr), n * 2 + n // 2 + n // 32),
            "mx_dequantize": (lambda: mxq.mx_dequantize(pr, sr, torch.bfloat16, outr),
                              n // 2 + n // 32 + n * 2),
        }
        for f, b in CACHE_RUNS:
            calls["qc_" + f] = ((lambda f=f, b=b: mxq.quantize_cache(xr, f, b, outr)), n * 4)
        row = {"rows": R}
        for name, (fn, nbytes) in calls.items():
            for _ in range(2):
                fn()
            ts = []
            for _ in range(5):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b.record()
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b))
            ms = sorted(ts)[2]
            row[name] = {"ms": round(ms, 4), "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1)}
        rows_out.append(row)
    del x, out, packed, scales, flush
    torch.cuda.empty_cache()
    return {"workload": "mixed blocks bf16 [R, 7168]", "unit": "GB/s",
            "timing": "median of 5, L2 flushed before each call", "rows": rows_out}


def run_sweep(args):
    """The mixed-block sweep alone, as one JSON line."""
    import torch

    import nvfp4_quantization_amax_b200 as mxq
    import synthetic as gen

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    sw = time_sweep(torch, mxq, gen, dev, min(args.sweep_max_log2, 21), args.sweep_min_log2)
    sw["peak_hbm_gbs"] = load_peaks()[0]["hbm_gbs"]
    print(json.dumps(sw), flush=True)


def run_reference(args, rank, world):
    """The reference arm: the scalar CPU oracle, as it stands, single-threaded
    on the host.  One step is one bounded sample of the quant/dequant part of
    the workload (the same generators, so the same values): mx_quantize and
    mx_dequantize of the first 16 expert-weight rows of [64,2048,7168] and
    quantize_cache in the three formats of the first 64 KV rows of
    [4,8192,512]; W untimed steps, then K timed ones.  Rank 0 alone runs."""
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle
    import synthetic as gen

    def bf16_bits(t):
        return t.cpu().view(torch.int16).numpy().view(np.uint16)

    w_rows, kv_rows = 16, 64
    wb = bf16_bits(gen.expert_weights(1, w_rows, 7168).view(w_rows, 7168))
    kv = bf16_bits(gen.kv_cache((1, kv_rows, 512)).view(kv_rows, 512))
    e_w, e_kv = w_rows * 7168, kv_rows * 512
    step_bytes = 2 * (e_w * 2 + e_w // 2 + e_w // 32) + len(CACHE_RUNS) * e_kv * 4

    def one_step():
        pk, sc = oracle.mx_quantize(wb)
        oracle.mx_dequantize(pk, sc)
        for f, b in CACHE_RUNS:
            oracle.quantize_cache(kv, f, b)

    for _ in range(args.warmup):
        one_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_step()
    dt = time.perf_counter() - t0
    value = round(step_bytes * args.steps / dt / 1e9, 4)
    sample = ("each step: mx_quantize and mx_dequantize of [16,7168] expert-weight rows and "
              "quantize_cache (fp8/128, mxfp4/32, nvfp4/16) of [64,512] KV rows, %d bytes of the "
              "GPU metric's algorithmic traffic; %d timed steps after %d untimed, one thread"
              % (step_bytes, args.steps, args.warmup))
    cores, model = host_cpu()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": sample, "cpu_model": model, "cores_available": cores},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["mxq", "reference"], default="mxq")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--sweep", action="store_true",
                    help="instead of the step: the mixed-block bandwidth sweep over row counts")
    ap.add_argument("--sweep-max-log2", type=int, default=21, choices=range(10, 22))
    ap.add_argument("--sweep-min-log2", type=int, default=10, choices=range(10, 22),
                    help="with --sweep: leave out the row counts below 2^N")
    ap.add_argument("--no-sweep", action="store_true",
                    help="leave the mixed-block sweep out of the default run")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.sweep:
        if rank == 0:
            run_sweep(args)
    elif args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_gpu(args, rank, world)


if __name__ == "__main__":
    main()
