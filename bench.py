#!/usr/bin/env python
"""Benchmark of the NVFP4 hot path on B200: one step = one autoregressive chunk through the QKV
projection of a 5B-class video DiT layer with every NVFP4 operation of the path:

  a4  weight quantize        W [9216 x 3072] BF16 -> NVFP4 (re-quantized each step, as in training)
  a1-a3 activation quantize  A [4680 x 3072] (3 latent frames x 30 x 52 patches): amax, row-wise
                             (GEMM operand) and column-wise (token-dim blocks, the wgrad operand)
                             from one read of A
  a5+a6 NVFP4 GEMM + bias    Y [4680 x 9216] = gA*gB * A.W^T + bias, BF16
  a7  KV append              K = Y[:, 3072:6144], V = Y[:, 6144:] (strided) -> cache slot (in place);
                             their amax comes from the GEMM epilogue (no amax pass)
  a8  KV restore             the 12-slot window (56160 tokens, 24 heads x 128) -> BF16 K and V

The weight quantization is independent of the rest of the step: it runs on a second stream as
soon as the previous step's GEMM has read the previous Wq, overlapping that step's KV append and
restore and this step's activation quantization; everything else is ordered on the main stream.
`value` = NVFP4 GEMM FLOPs per step / device time per step (TFLOP/s), summed over ranks; the
per-op times (each on its own stream), throughputs and roofline fractions are in `kernels`.  An
op's `share` is its part of the main stream's ordered ops (the critical path); the side-stream op
has `share` null, since its stream time includes the time it shares the GPU with the ops it
overlaps.  `roofline` is that of the main-stream op with the largest share.  Per-op times come
from a separate pass (up to 300 steps) with events around every op; the timed region records
events only around the dominant op, whose per-launch time there feeds the roofline.  Inputs rotate over
three input sets (~300 MB) and each step streams ~1.1 GB, so no step finds its inputs in the
126 MB L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs an independent replica (the path has no exchange step);
timing is the max over ranks of the device time.  `--impl reference` times the CPU oracle on a
bounded row sample of the same step (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 GEMM TFLOP/s (% FP4 peak); quantize/KV-dequant GB/s (% HBM peak)"
UNIT = "TFLOP/s"
M_TOK, HID, NQKV = 4680, 3072, 9216
HEADS, HEAD_DIM, SLOTS = 24, 128, 12
GEMM_FLOP = 2.0 * M_TOK * NQKV * HID
FP4_OVER_BF16 = 9.0 / 2.25          # nominal dense FP4 : BF16 tensor throughput on B200
PEAK_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None, help="timed steps (default 3000; 200 for --op attention)")
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--e2e-steps", type=int, default=40)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-large-gemms", action="store_true",
                   help="skip the standalone FFN and training-shape GEMM timings of the default run")
    p.add_argument("--cpu-seconds", type=float, default=15.0)
    p.add_argument("--attn-slots", type=int, default=SLOTS,
                   help="--op attention: cache slots in the window (default 12 = 56160 tokens; 1 gives the "
                        "small case used for ncu captures)")
    p.add_argument("--op", choices=["step", "attention", "appends", "kernels"], default="step",
                   help="step: the QKV chunk step (default); attention: kv_attention over the step's KV "
                        "window; appends: one chunk's KV append into all 30 layers, as a CUDA graph; "
                        "kernels: every kernel standalone on every workload shape (cold L2)")
    a = p.parse_args(argv)
    if a.steps is None:
        a.steps = {"attention": 200, "appends": 300, "kernels": 20}.get(a.op, 3000)
    return a


# ---------------------------------------------------------------------------------- plumbing

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def init_dist(world, backend):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def reduce_max(value: float, dist, device) -> float:
    """Max over ranks of a per-rank time (timing plumbing only; no data-path collective)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(per_rank_units: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput of independent replicas: all ranks' units / the slowest rank's time."""
    return per_rank_units * world / max_seconds


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(PEAK_FALLBACK), "fallback"


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.lines = []
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, RuntimeError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


def kernel_source_digest(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "bit_kv_cache_24_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(name, digest):
    """DRAM bytes per launch from a committed ncu summary (profiles/<name>.md), or None when the
    summary is missing or was taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", f"{name}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_digest") != digest:
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ------------------------------------------------------------------------ standalone timing

NOMINAL = {"fp4_tflops": 9000.0, "hbm_gbs": 7700.0}   # B200 dense FP4 and HGX HBM3e, context only


def standalone_timer(dev, reps):
    """Device time of one call, L2 flushed (a 256 MB read) before every launch and the host
    enqueue hidden behind a device sleep; median of `reps` launches after 3 warm-up calls."""
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def timeit(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.max()
            torch.cuda._sleep(2_000_000)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) / 1e3)
        ts.sort()
        return ts[len(ts) // 2]
    return timeit


def cublaslt_nvfp4(timeit, A, B, y_ref):
    """cuBLASLt's NVFP4 GEMM through torch (scaled_mm, block-16 E4M3 scales in the same tensor-core
    layout) on our codes and scales: library context beside our kernel, not part of the path.
    Returns its time, or why it is unavailable."""
    import torch.nn.functional as F
    M, N, K = A.rows, B.rows, A.cols
    try:
        a = A.codes.view(torch.float4_e2m1fn_x2)
        b = B.codes.view(torch.float4_e2m1fn_x2).t()
        sa = A.sf.view(torch.float8_e4m3fn).view(128 * ((M + 127) // 128), -1)
        sb = B.sf.view(torch.float8_e4m3fn).view(128 * ((N + 127) // 128), -1)
        ST, SW = F.ScalingType, F.SwizzleType
        call = lambda: F.scaled_mm(a, b, [sa, A.g], [ST.BlockWise1x16, ST.TensorWise], [sb, B.g],
                                   [ST.BlockWise1x16, ST.TensorWise], swizzle_a=[SW.SWIZZLE_32_4_4, SW.NO_SWIZZLE],
                                   swizzle_b=[SW.SWIZZLE_32_4_4, SW.NO_SWIZZLE], output_dtype=torch.bfloat16)
        y = call()
        torch.cuda.synchronize()
        rel = float((y.float() - y_ref.float()).norm() / y_ref.float().norm().clamp_min(1e-30))
        if not rel < 1e-2:
            return {"unavailable": f"result differs from ours (rel. Frobenius {rel:.3g})"}
        t = timeit(call)
        return {"us": round(t * 1e6, 1), "tflops": round(2 * M * N * K / t / 1e12, 1), "rel_frobenius_vs_ours": rel}
    except Exception as e:                                # library context only
        return {"unavailable": f"{type(e).__name__}: {str(e).splitlines()[0][:160]}"}


def time_gemm(nv, timeit, dev, A, B, fp4_peak, bias=None, resid=None, library=True):
    """One NVFP4 GEMM standalone: our kernel (with the workload's epilogue) and, as context,
    cuBLASLt's on the same operands (no epilogue term)."""
    y = torch.empty(A.rows, B.rows, dtype=torch.bfloat16, device=dev)
    t = timeit(lambda: nv.nvfp4_gemm(A, B, bias=bias, resid=resid, out=y))
    tf = 2 * A.rows * B.rows * A.cols / t / 1e12
    e = {"shape": [A.rows, B.rows, A.cols], "bound": "tensor", "us_per_launch": round(t * 1e6, 1),
         "achieved": round(tf, 1), "unit": "TFLOP/s", "peak": round(fp4_peak, 1), "frac": round(tf / fp4_peak, 4),
         "frac_nominal_9pf": round(tf / NOMINAL["fp4_tflops"], 4)}
    if library:
        e["cublaslt_nvfp4"] = cublaslt_nvfp4(timeit, A, B, nv.nvfp4_gemm(A, B))
    del y
    return e


def large_gemms(nv, dev, fp4_peak, reps=20, library=True):
    """The FFN (one chunk) and training-shape GEMMs, each standalone with L2 flushed: FFN up
    4680x14336x3072, FFN down 4680x3072x14336 (+R), fprop 37440x3072x3072, dgrad (B = W^T from the
    column-wise quantization of W) and wgrad 3072x3072x37440 (both operands column-wise)."""
    from bit_kv_cache_24_b200 import synth
    timeit = standalone_timer(dev, reps)
    out = {}
    d = {k: v.to(dev) for k, v in synth.ffn().items()}
    out["gemm_ffn_up"] = time_gemm(nv, timeit, dev, nv.nvfp4_quantize(d["A_up"]), nv.nvfp4_quantize(d["W_up"]),
                                   fp4_peak, library=library)
    out["gemm_ffn_down"] = time_gemm(nv, timeit, dev, nv.nvfp4_quantize(d["A_down"]),
                                     nv.nvfp4_quantize(d["W_down"]), fp4_peak, resid=d["R"], library=library)
    del d
    d = {k: v.to(dev) for k, v in synth.train().items()}
    X, dY, W = nv.nvfp4_quantize(d["X"]), nv.nvfp4_quantize(d["dY"]), nv.nvfp4_quantize(d["W"])
    out["gemm_fprop"] = time_gemm(nv, timeit, dev, X, W, fp4_peak, library=library)
    out["gemm_dgrad"] = time_gemm(nv, timeit, dev, dY, nv.nvfp4_quantize(d["W"], nv.COLWISE), fp4_peak,
                                  library=library)
    del X, W
    out["gemm_wgrad"] = time_gemm(nv, timeit, dev, nv.nvfp4_quantize(d["dY"], nv.COLWISE),
                                  nv.nvfp4_quantize(d["X"], nv.COLWISE), fp4_peak, library=library)
    del d, dY
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------------- our arm

class QKVStep:
    """All buffers of the step, preallocated: no allocation inside the timed region."""

    def __init__(self, device, nsets=3):
        import bit_kv_cache_24_b200 as nv
        from bit_kv_cache_24_b200 import synth
        self.nv = nv
        self.sets = []
        for i in range(nsets):
            d = synth.qkv(seed=1 + 100 * i)
            self.sets.append({k: v.to(device) for k, v in d.items()})
        self.A_host = synth.qkv(seed=1)["A"].pin_memory()
        self.Wq = nv.QTensor(NQKV, HID, nv.SF_MMA, device)
        self.Aq = nv.QTensor(M_TOK, HID, nv.SF_MMA, device)
        self.Acq = nv.QTensor(HID, M_TOK, nv.SF_MMA, device)
        L = nv.lib()
        self.ws_w = torch.empty(L.nvfp4_quantize_workspace(NQKV, HID), dtype=torch.uint8, device=device)
        self.ws_a = torch.empty(L.nvfp4_quantize_workspace(M_TOK, HID), dtype=torch.uint8, device=device)
        self.Y = torch.empty(M_TOK, NQKV, dtype=torch.bfloat16, device=device)
        self.Y_host = torch.empty(M_TOK, NQKV, dtype=torch.bfloat16).pin_memory()
        self.cache = nv.KVCache(1, HEADS, HEAD_DIM, SLOTS, M_TOK, device)
        for s in range(SLOTS):                            # the window: 12 chunks already cached
            k, v = synth.kv_chunk(0, s)
            nv.kv_quant_append(self.cache, 0, s, k.to(device), v.to(device))
        tokens = SLOTS * M_TOK
        self.Kout = torch.empty(tokens, HEADS, HEAD_DIM, dtype=torch.bfloat16, device=device)
        self.Vout = torch.empty_like(self.Kout)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.amax_qkv = torch.empty(3, dtype=torch.float32, device=device)
        self.ws_cam = torch.empty(L.nvfp4_gemm_colamax_workspace(M_TOK, NQKV), dtype=torch.uint8, device=device)
        self.main = torch.cuda.Stream(device)
        self.side = torch.cuda.Stream(device)
        self.wq_free = torch.cuda.Event()                 # the previous step's GEMM has read Wq
        self.w_done = torch.cuda.Event()
        self.wq_free.record()

        self.slots = list(range(SLOTS))
        self.ops = ["w_quantize", "a_quantize_rowcol", "gemm", "kv_append", "kv_dequant"]
        self.side_ops = {"w_quantize"}                    # on the side stream, overlapping the others
        self.launches = 0                                 # kernels launched by step() so far
        # kernels per step: W amax + scale record + row pass; A amax + record + row + column pass;
        # GEMM + the column-group amax finish; the K/V row pass (both tensors per launch; their
        # amax comes from the GEMM epilogue and the pass builds its own scale record); dequant
        self.launches_per_step = 3 + 4 + 2 + 1 + 1

    def step(self, i, events=None, A=None, Y=None):
        """One step.  W's quantization is independent of the rest, so it runs on a side stream as
        soon as the previous step's GEMM has read Wq (overlapping that step's KV append and restore
        and this step's A quantization); the GEMM waits for it.  events: {op: (start, end)} recorded on the op's own stream."""
        nv = self.nv
        s = self.sets[i % len(self.sets)]
        A = s["A"] if A is None else A
        Y = self.Y if Y is None else Y
        main = torch.cuda.current_stream()

        def mark(op, k, stream):
            if events is not None and op in events:
                events[op][k].record(stream)
        self.launches += self.launches_per_step
        self.side.wait_event(self.wq_free)
        with torch.cuda.stream(self.side):
            mark("w_quantize", 0, self.side)
            nv.nvfp4_quantize(s["W"], nv.ROWWISE, out=self.Wq, ws=self.ws_w, status=self.status)
            mark("w_quantize", 1, self.side)
            self.w_done.record(self.side)
        mark("a_quantize_rowcol", 0, main)
        nv.nvfp4_quantize(A, nv.ROWCOL, out=(self.Aq, self.Acq), ws=self.ws_a, status=self.status)
        mark("a_quantize_rowcol", 1, main)
        main.wait_event(self.w_done)
        mark("gemm", 0, main)
        # the epilogue also reduces max |Y| of the Q, K and V column groups (for the KV append)
        nv.nvfp4_gemm_colamax(self.Aq, self.Wq, HID, bias=s["bias"], out=Y, amax_out=self.amax_qkv,
                              ws=self.ws_cam, status=self.status)
        mark("gemm", 1, main)
        self.wq_free.record(main)
        mark("kv_append", 0, main)
        nv.kv_quant_append(self.cache, 0, i % SLOTS, Y[:, HID:2 * HID], Y[:, 2 * HID:],
                           status=self.status, amax_kv=self.amax_qkv[1:])
        mark("kv_append", 1, main)
        mark("kv_dequant", 0, main)
        nv.kv_dequant(self.cache, 0, self.slots, k_out=self.Kout, v_out=self.Vout, status=self.status)
        mark("kv_dequant", 1, main)

    # algorithmic work per launch of each op (bytes or FLOPs)
    @staticmethod
    def work():
        mk, nk = M_TOK * HID, NQKV * HID
        q = 2 + 0.5 + 1 / 16                              # BF16 in, codes + scales out, per element
        win = SLOTS * M_TOK * HEADS * HEAD_DIM
        return {
            # bytes that must cross HBM at least once per op: BF16 in (read once), codes + scales
            # out; the second read of the two-pass quantizers is not counted
            "w_quantize": ("hbm", q * nk),
            "a_quantize_rowcol": ("hbm", (2 + 2 * (0.5 + 1 / 16)) * mk),   # both layouts from one read
            "gemm": ("tensor", GEMM_FLOP),
            "kv_append": ("hbm", 2 * q * mk),                # K and V
            "kv_dequant": ("hbm", 2 * win * (0.5 + 1 / 16 + 2)),
        }


def attention_on_step_window(st, bf16_peak, reps=10):
    """kv_attention of the step's queries (the Q third of its QKV output, row stride 9216) over
    the step's 12-slot NVFP4 window (56160 tokens x 24 heads x 128), timed outside the step:
    device time per launch, mean of `reps` launches after 3 warm-up launches."""
    nv = st.nv
    q = st.Y[:, :HID]
    o = torch.empty(M_TOK, HEADS * HEAD_DIM, dtype=torch.bfloat16, device=st.Y.device)
    slots, scale = list(range(SLOTS)), 1.0 / math.sqrt(HEAD_DIM)
    for _ in range(3):
        nv.kv_attention(st.cache, 0, slots, q, scale, out=o, status=st.status)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        nv.kv_attention(st.cache, 0, slots, q, scale, out=o, status=st.status)
    b.record()
    torch.cuda.synchronize()
    t = a.elapsed_time(b) / 1e3 / reps
    tf = ATTN_FLOP / t / 1e12
    return {"bound": "tensor", "us_per_launch": round(t * 1e6, 1), "achieved": round(tf, 1), "unit": "TFLOP/s",
            "peak": round(bf16_peak, 1), "frac": round(tf / bf16_peak, 4), "share": None,
            "stream": "outside the step: the step's Q over its 12-slot NVFP4 window (restore fused), mean of "
                      f"{reps} launches", "peak_source": "measured bf16 cuBLAS burst"}


def summarize_ops(per_op_ms, K, work, side_ops, hbm_peak, fp4_peak):
    """Per-op averages, throughputs and roofline fractions from the summed event times of K steps.
    `share` is an op's part of the summed main-stream (critical-path) op times; side-stream ops
    overlap them, so their share is None and they are never the dominant op."""
    main_ms = sum(t for op, t in per_op_ms.items() if op not in side_ops)
    kernels = {}
    for op, (bound, w) in work.items():
        avg_s = per_op_ms[op] / K / 1e3
        if bound == "tensor":
            ach, peak, unit = w / avg_s / 1e12, fp4_peak, "TFLOP/s"
        else:
            ach, peak, unit = w / avg_s / 1e9, hbm_peak, "GB/s"
        nominal = NOMINAL["fp4_tflops"] if bound == "tensor" else NOMINAL["hbm_gbs"]
        kernels[op] = {"bound": bound, "us_per_launch": round(avg_s * 1e6, 2), "achieved": round(ach, 1),
                       "unit": unit, "peak": round(peak, 1), "frac": round(ach / peak, 4),
                       ("frac_nominal_9pf" if bound == "tensor" else "frac_nominal_7700gbs"): round(ach / nominal, 4),
                       "share": None if op in side_ops else round(per_op_ms[op] / main_ms, 4)}
        if op in side_ops:
            kernels[op]["stream"] = "side (overlaps other ops; time includes sharing the GPU)"
    dominant = max((op for op in kernels if op not in side_ops), key=lambda op: kernels[op]["share"])
    return kernels, dominant


def workload_config(world):
    """The workload both arms report (the reference arm times a bounded row sample of it, stated in
    its cpu_baseline.sample)."""
    return {"workload": "qkv_chunk_step: A[4680x3072] x W[9216x3072]^T + bias, KV append 4680 tok, "
                        "KV window 12x4680 tok x 24 heads x 128",
            "global_batch": M_TOK * world, "seq_len": SLOTS * M_TOK, "parallelism": f"replicas x{world}",
            "l2": "inputs rotate over 3 sets (~300 MB) and each step streams ~1.1 GB (> 126 MB L2)",
            "value_def": "GEMM FLOPs per step / time per step (all 5 ops; W and A quantization concurrent), "
                         "summed over replicas; device time for the GPU arm, host time of the row "
                         "sample for the reference arm"}


def run_ours(args, rank, local_rank, world):
    dist = init_dist(world, "nccl")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    st = QKVStep(dev)
    torch.cuda.synchronize()
    torch.cuda.set_stream(st.main)                        # every op of the run on the step's streams
    nops = len(st.ops)
    for i in range(args.warmup):
        st.step(i)
    torch.cuda.synchronize()
    if int(st.status.item()) != 0:
        raise RuntimeError(f"device status {int(st.status.item())} after warm-up")

    K = args.steps
    # Per-op times and shares come from a separate pass with events around every op (events
    # between chained launches cost some of their overlap); the timed region below records events
    # only around the dominant op, for the roofline's live per-launch time.
    P = min(K, 300)
    pre = [{op: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for op in st.ops}
           for _ in range(P)]
    for i in range(P):
        st.step(args.warmup + i, pre[i])
    torch.cuda.synchronize()
    per_op_pre = {op: sum(ev[op][0].elapsed_time(ev[op][1]) for ev in pre) for op in st.ops}
    _, dominant = summarize_ops(per_op_pre, P, st.work(), st.side_ops, 1.0, 1.0)
    events = [{dominant: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))}
              for _ in range(K)]
    clocks = ClockSampler(local_rank)
    time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    st.wq_free.record()                                   # the side stream starts after t_start
    launches0 = st.launches
    for i in range(K):
        st.step(args.warmup + P + i, events[i])
    t_end.record()
    launches = st.launches - launches0
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    # every op at its separate-pass average, the dominant one at its timed-region average
    per_op = {op: per_op_pre[op] * K / P for op in st.ops}
    per_op[dominant] = sum(ev[dominant][0].elapsed_time(ev[dominant][1]) for ev in events)
    status = int(st.status.item())
    max_s = reduce_max(total_ms / 1e3, dist, dev)
    value = aggregate(GEMM_FLOP * K / 1e12, world, max_s)

    # end to end through the public API: every step copies its A from pinned host memory to the
    # device, runs the step and copies its Y back to pinned host memory.  The copies run on their
    # own streams and overlap neighbouring steps' compute (double-buffered A and Y on the device),
    # as a serving pipeline would; the timed region spans the first copy in to the last copy out.
    E = args.e2e_steps
    e2e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    A_dev = [torch.empty_like(st.sets[0]["A"]) for _ in range(2)]
    Y_dev = [st.Y, torch.empty_like(st.Y)]
    comp = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n, first=None, last=None):
        a_free = [None, None]                             # compute done with A_dev[b]
        y_free = [None, None]                             # copy-out done with Y_dev[b]
        if first is not None:
            first.record(comp)
            h2d.wait_event(first)
            d2h.wait_event(first)
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(h2d):
                if a_free[b] is not None:
                    h2d.wait_event(a_free[b])
                A_dev[b].copy_(st.A_host, non_blocking=True)
                a_in = torch.cuda.Event()
                a_in.record(h2d)
            comp.wait_event(a_in)
            if y_free[b] is not None:
                comp.wait_event(y_free[b])
            st.step(i, A=A_dev[b], Y=Y_dev[b])
            done = torch.cuda.Event()
            done.record(comp)
            a_free[b] = done
            with torch.cuda.stream(d2h):
                d2h.wait_event(done)
                st.Y_host.copy_(Y_dev[b], non_blocking=True)
                y_out = torch.cuda.Event()
                y_out.record(d2h)
            y_free[b] = y_out
        for ev in y_free:
            if ev is not None:
                comp.wait_event(ev)
        if last is not None:
            last.record(comp)

    e2e_run(3)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e2e_run(E, e2e_ev[0], e2e_ev[1])
    torch.cuda.synchronize()
    e2e_s = reduce_max(e2e_ev[0].elapsed_time(e2e_ev[1]) / 1e3, dist, dev)
    e2e = {"value": aggregate(GEMM_FLOP * E / 1e12, world, e2e_s), "unit": UNIT,
           "h2d_bytes_per_step": st.A_host.numel() * 2, "d2h_bytes_per_step": st.Y_host.numel() * 2,
           "steps": E}

    peaks, peak_src = load_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", PEAK_FALLBACK["hbm_gbs"]))
    # the timed region is a few hundred 0.3 ms steps (seconds at most, no sustained power-capped
    # loop): the burst cuBLAS figure applies, times the nominal dense FP4:BF16 ratio
    fp4_peak = float(peaks.get("bf16_tflops", PEAK_FALLBACK["bf16_tflops"])) * FP4_OVER_BF16
    kernels, _ = summarize_ops(per_op, K, st.work(), st.side_ops, hbm_peak, fp4_peak)
    for op, e in kernels.items():
        e["timing"] = ("events in the timed region" if op == dominant
                       else f"events around every op in a separate pass of {P} steps")
    if world == 1 and not args.no_large_gemms:
        for name, e in large_gemms(st.nv, dev, fp4_peak).items():
            e["share"] = None
            e["stream"] = "standalone, outside the step (L2 flushed before each launch, median of 20)"
            kernels[name] = e
        kernels["kv_attention_window"] = attention_on_step_window(st, float(peaks.get("bf16_tflops",
                                                                                    PEAK_FALLBACK["bf16_tflops"])))
    dk = kernels[dominant]
    # DRAM bytes per launch from the committed ncu summary of the dominant kernel (None when the
    # summary was taken on other kernel sources)
    digests = {"gemm": ["gemm.cu", "gemm2sm.cu", "common.cuh", "launch.h"],
               "kv_dequant": ["kv_cache.cu", "common.cuh", "launch.h"]}
    traffic = None
    if dominant in digests:
        traffic = profiled_traffic(f"{dominant}_qkv_step", kernel_source_digest(digests[dominant]))
    roofline = {"kernel": dominant, "bound": dk["bound"], "achieved": dk["achieved"], "peak": dk["peak"],
                "unit": dk["unit"], "frac": dk["frac"], "traffic": traffic,
                "peak_source": f"{peak_src} ({'HBM copy' if dk['bound'] == 'hbm' else 'bf16 cuBLAS burst x 4 (nominal FP4:BF16)'})"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_seconds)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(max_s * 1e3 / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e4m3/16) -> fp32 acc -> bf16",
        "data": "synthetic (seeded; QKV-projection shapes of a 5B video DiT, random-init weights)",
        "config": workload_config(world),
        "gpu_launches": launches,
        "kernels": kernels, "roofline": roofline, "clocks": clk, "e2e": e2e,
        "device_status": status,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------------- oracle arm

def oracle_sample_step(rows, wrows, data, orc, synth):
    """The step's ops on a row sample: W[wrows] quantize, A[rows] amax/row/col quantize, the fp64
    GEMM of those rows against W[wrows] (+bias), a `rows`-token KV append and the restore of a
    12-slot window of `rows` tokens each."""
    A = data["A"][:rows].contiguous()
    W = data["W"][:wrows].contiguous()
    _, qw = orc.quantize(W)
    st, am = orc.amax(A)
    _, qa = orc.quantize(A, amax_in=am)
    _, qc = orc.quantize(A, colwise=True, amax_in=am)
    orc.gemm_rows(qa, qw, bias=data["bias"][:wrows].contiguous(), threads=os.cpu_count())
    kv = orc.KVCacheModel(1, HEADS, HEAD_DIM, SLOTS, rows)
    for s in range(SLOTS):
        kv.append(0, s, data["K"][s], data["V"][s])
    kv.dequant(0, list(range(SLOTS)))
    return 2.0 * rows * wrows * HID


def oracle_data(rows):
    from bit_kv_cache_24_b200 import synth
    d = synth.qkv()
    k, v = synth.kv_chunk(0, 0)
    d["K"] = [k[:rows].contiguous()] * SLOTS
    d["V"] = [v[:rows].contiguous()] * SLOTS
    return d


def cpu_baseline(seconds, rows=16, wrows=256):
    from oracle import oracle as orc
    from bit_kv_cache_24_b200 import synth
    orc.build()
    data = oracle_data(rows)
    flop, t0, n = 0.0, time.perf_counter(), 0
    while True:
        flop += oracle_sample_step(rows, wrows, data, orc, synth)
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": flop / dt / 1e12, "unit": UNIT, "cores": min(os.cpu_count(), rows), "kind": "oracle",
            "sample": f"{n} oracle steps on A rows [:{rows}] x W rows [:{wrows}] (of 4680 x 9216), "
                      f"{rows}-token KV append, 12x{rows}-token KV restore; {dt:.1f} s; the fp64 GEMM "
                      f"runs on {min(os.cpu_count(), rows)} threads, the codecs on one"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    from oracle import oracle as orc
    from bit_kv_cache_24_b200 import synth
    orc.build()
    total = args.steps + args.warmup
    budget = min(1.0, 150.0 / max(1, total))              # seconds per sample step
    rows = max(1, min(16, int(budget / 0.025)))
    wrows = 16 * rows
    data = oracle_data(rows)
    for _ in range(args.warmup):
        oracle_sample_step(rows, wrows, data, orc, synth)
    flop, t0 = 0.0, time.perf_counter()
    for _ in range(args.steps):
        flop += oracle_sample_step(rows, wrows, data, orc, synth)
    dt = time.perf_counter() - t0
    value = flop / dt / 1e12
    sample = (f"each step: A rows [:{rows}] x W rows [:{wrows}] (of 4680 x 9216), {rows}-token KV append, "
              f"12x{rows}-token KV restore")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic (seeded; same generator as the GPU arm)",
            "config": workload_config(world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(os.cpu_count(), rows), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ attention op

ATTN_FLOP = 4.0 * M_TOK * SLOTS * M_TOK * HEADS * HEAD_DIM    # Q.K^T and P.V over the window


def run_attention(args, rank, local_rank, world):
    """kv_attention over the QKV step's 12-slot window (56160 tokens x 24 heads x 128, NVFP4)
    for the chunk's 4680 queries: one launch per step, restore fused into the K/V tile loads."""
    import bit_kv_cache_24_b200 as nv
    from bit_kv_cache_24_b200 import synth
    dist = init_dist(world, "nccl")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    nslots = args.attn_slots
    if not 1 <= nslots <= SLOTS:
        raise SystemExit(f"--attn-slots must be in [1, {SLOTS}]")
    attn_flop = ATTN_FLOP * nslots / SLOTS
    cache = nv.KVCache(1, HEADS, HEAD_DIM, nslots, M_TOK, dev)
    for s in range(nslots):
        k, v = synth.kv_chunk(0, s)
        nv.kv_quant_append(cache, 0, s, k.to(dev), v.to(dev))
    q_host = synth.normal(21, 0, (M_TOK, HEADS, HEAD_DIM)).pin_memory()
    q = q_host.to(dev)
    o = torch.empty_like(q)
    o_host = torch.empty_like(q_host).pin_memory()
    slots, scale = list(range(nslots)), 1.0 / math.sqrt(HEAD_DIM)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        nv.kv_attention(cache, 0, slots, q, scale, out=o)
    torch.cuda.synchronize()
    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    if dist:
        dist.barrier()
    clocks = ClockSampler(local_rank)
    ev[0].record(stream)
    for _ in range(K):
        nv.kv_attention(cache, 0, slots, q, scale, out=o)
    ev[1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    max_s = reduce_max(ev[0].elapsed_time(ev[1]) / 1e3, dist, dev)
    value = aggregate(attn_flop * K / 1e12, world, max_s)

    # end to end through the public call: q in from pinned host memory, O back out, every step
    E = max(3, min(K, 20))
    e2e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    e2e_ev[0].record(stream)
    for _ in range(E):
        q.copy_(q_host, non_blocking=True)
        nv.kv_attention(cache, 0, slots, q, scale, out=o)
        o_host.copy_(o, non_blocking=True)
    e2e_ev[1].record(stream)
    torch.cuda.synchronize()
    e2e_s = reduce_max(e2e_ev[0].elapsed_time(e2e_ev[1]) / 1e3, dist, dev)
    nbytes = q_host.numel() * 2

    peaks, src = load_peaks()
    peak = float(peaks.get("bf16_tflops", PEAK_FALLBACK["bf16_tflops"]))
    ach = attn_flop / (max_s / K) / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = attention_cpu_baseline(args.cpu_seconds)
    line = {
        "metric": "kv_attention TFLOP/s (NVFP4 KV window, restore fused; % of BF16 tensor peak)",
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(max_s * 1e3 / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4 K/V (e2m1 x e4m3/16) -> bf16 mma, fp32 acc -> bf16",
        "data": "synthetic (seeded; K/V of the KV workload, q ~ N(0,1))",
        "config": {"workload": f"kv_attention: 4680 queries x 24 heads x 128 over the {nslots}-slot NVFP4 window "
                               f"({nslots * M_TOK} tokens), no mask", "global_batch": M_TOK * world,
                   "seq_len": nslots * M_TOK,
                   "parallelism": f"replicas x{world}",
                   "l2": f"the window's NVFP4 K/V ({nslots * 16.2:.0f} MB) "
                         + ("exceeds the 126 MB L2" if nslots * 16.2 > 126 else "fits in the 126 MB L2")},
        "gpu_launches": K,
        "roofline": {"kernel": "kv_attention_kernel", "bound": "tensor", "achieved": round(ach, 1),
                     "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(ach / peak, 4), "traffic": None,
                     "peak_source": f"{src} (bf16 cuBLAS burst)"},
        "clocks": clk,
        "e2e": {"value": round(aggregate(attn_flop * E / 1e12, world, e2e_s), 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes, "steps": E},
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def attention_cpu_baseline(seconds, rows=4):
    """The oracle's fp64 attention on a row sample: `rows` query rows of one head at a time over
    the full 56160-token window, cycling over the 24 heads for about `seconds` (the window is
    restored once, before the timed loop)."""
    from oracle import oracle as orc
    from bit_kv_cache_24_b200 import synth
    model = orc.KVCacheModel(1, HEADS, HEAD_DIM, SLOTS, M_TOK)
    for s in range(SLOTS):
        k, v = synth.kv_chunk(0, s)
        model.append(0, s, k, v)
    kb, vb = model.dequant(0, list(range(SLOTS)))
    q = synth.normal(21, 0, (rows, HEADS, HEAD_DIM))
    t0, n = time.perf_counter(), 0
    while True:
        h = n % HEADS
        orc.attention(q[:, h:h + 1], kb[:, h:h + 1], vb[:, h:h + 1], 1.0 / math.sqrt(HEAD_DIM))
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    flop = 4.0 * rows * SLOTS * M_TOK * HEAD_DIM * n
    return {"value": flop / dt / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{n} calls of {rows} query rows x 1 head over the 56160-token window in {dt:.1f} s"}


# ------------------------------------------------------------------------------ appends op

LAYERS = 30
APPEND_BYTES = 2 * M_TOK * HEADS * HEAD_DIM * (2 + 0.5 + 1 / 16)   # K and V: BF16 in, codes + scales out


def run_appends(args, rank, local_rank, world):
    """One chunk's KV append into every layer of a 30-layer cache (kv_quant_append per layer,
    three kernels each), launched back to back and, separately, replayed as one CUDA graph.
    A step is all 30 appends. The K/V inputs rotate over 6 distinct layers' tensors (345 MB,
    more than the 126 MB L2)."""
    import bit_kv_cache_24_b200 as nv
    from bit_kv_cache_24_b200 import synth
    dist = init_dist(world, "nccl")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cache = nv.KVCache(LAYERS, HEADS, HEAD_DIM, 1, M_TOK, dev)
    kv = [tuple(t.to(dev) for t in synth.kv_chunk(layer, 0)) for layer in range(6)]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)

    def appends():
        for layer in range(LAYERS):
            k, v = kv[layer % len(kv)]
            nv.kv_quant_append(cache, layer, 0, k, v, status=status)

    for _ in range(max(args.warmup, 3)):                  # also sets every launch attribute once
        appends()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        appends()
    torch.cuda.synchronize()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} after warm-up")

    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    if dist:
        dist.barrier()
    clocks = ClockSampler(local_rank)
    ev[0].record(stream)
    for _ in range(K):
        graph.replay()
    ev[1].record(stream)
    for _ in range(K):
        appends()
    ev[2].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    graph_s = reduce_max(ev[0].elapsed_time(ev[1]) / 1e3, dist, dev)
    eager_s = reduce_max(ev[1].elapsed_time(ev[2]) / 1e3, dist, dev)
    peaks, src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", PEAK_FALLBACK["hbm_gbs"]))
    gbs = APPEND_BYTES * LAYERS * K / graph_s / 1e9
    line = {
        "metric": "KV append GB/s (30 layers per step, CUDA graph; % of HBM peak)",
        "value": round(aggregate(APPEND_BYTES * LAYERS * K / 1e9, world, graph_s), 1), "unit": "GB/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(graph_s * 1e3 / K, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 -> nvfp4 (e2m1 x e4m3/16)", "data": "synthetic (seeded; K/V of the KV workload)",
        "config": {"workload": "kv_quant_append of one 4680-token chunk (24 heads x 128, K and V) into each "
                               "of 30 layers", "global_batch": M_TOK * world, "seq_len": M_TOK,
                   "parallelism": f"replicas x{world}",
                   "l2": "inputs rotate over 6 layers' K/V (345 MB) > 126 MB L2"},
        "gpu_launches": 3 * LAYERS * 2 * K,                 # amax, record, row pass per layer; graph + eager
        "eager": {"ms_per_step": round(eager_s * 1e3 / K, 4),
                  "value": round(APPEND_BYTES * LAYERS * K / eager_s / 1e9, 1), "unit": "GB/s"},
        "roofline": {"kernel": "kv_quant_append (amax, scale record, row pass)", "bound": "hbm",
                     "achieved": round(gbs, 1), "peak": round(hbm, 1), "unit": "GB/s", "frac": round(gbs / hbm, 4),
                     "traffic": None, "peak_source": f"{src} (HBM copy)"},
        "clocks": clk,
        "device_status": int(status.item()),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    if dist:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------------------ kernels op

def run_kernels(args, rank, local_rank, world):
    """Every kernel standalone on the workload shapes: L2 flushed (a 256 MB read) before each
    launch, the host enqueue hidden behind a device sleep, median of `--steps` launches (20 by
    default). Beside each NVFP4 GEMM, cuBLASLt's NVFP4 GEMM (torch scaled_mm) on the same quantized
    operands, as library context; it is not part of the path."""
    import bit_kv_cache_24_b200 as nv
    from bit_kv_cache_24_b200 import synth
    if world > 1:
        raise SystemExit("--op kernels runs on one GPU")
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    reps = args.steps
    timeit = standalone_timer(dev, reps)
    peaks, src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", PEAK_FALLBACK["hbm_gbs"]))
    fp4 = float(peaks.get("bf16_tflops", PEAK_FALLBACK["bf16_tflops"])) * FP4_OVER_BF16
    out = {}

    def gemm(name, A, B, bias=None, resid=None):
        out[f"gemm_{name}"] = time_gemm(nv, timeit, dev, A, B, fp4, bias=bias, resid=resid)

    def quant(name, x):
        M, K = x.shape
        byt = M * K * (2 + 0.5 + 1 / 16)
        A = nv.nvfp4_quantize(x)
        amax = nv.nvfp4_amax(x)
        Ac = nv.nvfp4_quantize(x, nv.COLWISE)
        e = {"shape": [M, K]}
        for key, fn in (("two_pass", lambda: nv.nvfp4_quantize(x, out=A)),
                        ("row_amax_given", lambda: nv.nvfp4_quantize(x, amax_in=amax, out=A)),
                        ("col_amax_given", lambda: nv.nvfp4_quantize(x, nv.COLWISE, amax_in=amax, out=Ac))):
            t = timeit(fn)
            e[key] = {"us": round(t * 1e6, 1), "gbs": round(byt / t / 1e9, 1), "frac_hbm": round(byt / t / 1e9 / hbm, 4)}
        out[f"quantize_{name}"] = e

    d = {k: v.to(dev) for k, v in synth.qkv().items()}
    quant("qkv_A", d["A"])
    quant("qkv_W", d["W"])
    gemm("qkv", nv.nvfp4_quantize(d["A"]), nv.nvfp4_quantize(d["W"]), bias=d["bias"])
    d = {k: v.to(dev) for k, v in synth.ffn().items()}
    quant("ffn_down_A", d["A_down"])
    del d
    d = {k: v.to(dev) for k, v in synth.train().items()}
    quant("train_X", d["X"])
    del d
    out.update(large_gemms(nv, dev, fp4, reps))
    sq = synth.ragged(8192, 8192, 8192).to(dev)
    gemm("8192cubed", nv.nvfp4_quantize(sq), nv.nvfp4_quantize(sq))
    del sq

    cache = nv.KVCache(1, HEADS, HEAD_DIM, SLOTS, M_TOK, dev)
    chunks = [tuple(t.to(dev) for t in synth.kv_chunk(0, s)) for s in range(SLOTS)]
    for s, (k, v) in enumerate(chunks):
        nv.kv_quant_append(cache, 0, s, k, v)
    kout = torch.empty(SLOTS * M_TOK, HEADS, HEAD_DIM, dtype=torch.bfloat16, device=dev)
    vout = torch.empty_like(kout)
    t = timeit(lambda: nv.kv_dequant(cache, 0, list(range(SLOTS)), k_out=kout, v_out=vout))
    byt = 2 * SLOTS * M_TOK * HEADS * HEAD_DIM * (0.5 + 1 / 16 + 2)
    out["kv_dequant_window"] = {"us": round(t * 1e6, 1), "gbs": round(byt / t / 1e9, 1),
                                "frac_hbm": round(byt / t / 1e9 / hbm, 4)}
    k, v = chunks[0]
    t = timeit(lambda: nv.kv_quant_append(cache, 0, 0, k, v))
    byt = APPEND_BYTES
    out["kv_append_chunk"] = {"us": round(t * 1e6, 1), "gbs": round(byt / t / 1e9, 1),
                              "frac_hbm": round(byt / t / 1e9 / hbm, 4)}
    line = {"metric": "standalone kernel timings (L2 flushed, median)", "unit": "us", "reps": reps,
            "peaks": {"hbm_gbs": hbm, "fp4_ref_tflops_burst": fp4, "source": src},
            "data": "synthetic (seeded workload generators)", "kernels": out}
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    rank, local_rank, world = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.op == "attention":
        run_attention(args, rank, local_rank, world)
        return
    if args.op == "appends":
        run_appends(args, rank, local_rank, world)
        return
    if args.op == "kernels":
        run_kernels(args, rank, local_rank, world)
        return
    run_ours(args, rank, local_rank, world)


if __name__ == "__main__":
    main()
