#!/usr/bin/env python
"""Benchmark of the BitLinear hot path on B200.

One step = the input-projection prefill workload, both activation variants:
  X [2048 tokens x 2048] bf16, N(0,1) with 1% outlier channels x20;
  fused q|k|v W [2048 x 6144] (3 scale groups) and gate|up W [2048 x 11264]
  (2 groups), ternary, 2-bit packed.
  INT4: quant_act(X, INT4) -> gemm_w2a4(qkv) -> gemm_w2a4(gate_up)
  FP4 : quant_act(X, FP4)  -> gemm_w2fp4(qkv) -> gemm_w2fp4(gate_up)
value = 2*M*K*N summed over the four GEMMs / step time, in TOPS.

Inputs are already resident in HBM; R replicas of all buffers rotate so the
working set (>= 270 MB) exceeds the 126 MB L2 between consecutive steps.
Each replica's step is one CUDA graph (no event nodes inside). Per-kernel
durations come from CUDA graphs of 8 back-to-back launches of that kernel
alone over the replicas, timed the same way.

Also reported (same run, rank 0, unless --no-breakdown): the o_proj top-k
INT8 GEMM, the down_proj ReLU^2 INT8 GEMM, the decode layer at batch 1/8/64
(weight GB/s), the 3-bit KV quantiser (GB/s), the 3-bit KV attention, and
library references on the prefill shapes (cuBLAS int8 / fp8 / mxfp4 GEMMs on
plain operands, a read-only HBM stream).

--impl reference times the CPU oracle on host cores on a bounded sample of
the same workload (rows of X), in the same metric.

Multi-GPU (torchrun): each rank runs the same per-GPU workload (replicas,
weak scaling, no collective on the data path); value = all ranks' ops /
max-over-ranks time.
"""
from __future__ import annotations

import argparse
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
sys.path.insert(0, ROOT)

METRIC = "BitLinear prefill TOPS vs int8/fp4 peak; decode weight GB/s vs HBM (1×B200)"
WORKLOAD = ("Input-projection prefill W1.58A4: X [2048 tokens×2048] bf16 ~N(0,1) with 1% "
            "channels ×20 outliers; fused q/k/v W [2048×6144] and gate/up W "
            "[2048×2×5632] ternary; INT4 and FP4(e2m1) activation variants")
M_TOK, D, FFN = 2048, 2048, 5632
QKV = (D, (D, 2 * D, 3 * D))
GU = (D, (FFN, 2 * FFN))
OPS_PER_STEP = 2 * (2 * M_TOK * D * 3 * D + 2 * M_TOK * D * 2 * FFN)
# nominal dense ratios to bf16 (2.25 PF): int8 4.5 P, fp8 4.5 P, fp4 9 P
RATIO_INT8, RATIO_FP4 = 2.0, 4.0
# nominal B200 dense peaks (vendor figures) and ~8 TB/s HBM, reported beside the measured ones
NOMINAL = {"int8_tops": 4500.0, "fp8_tflops": 4500.0, "fp4_tflops": 9000.0, "hbm_gbs": 8000.0}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CSRC = os.path.join(ROOT, "bit_quantised_gemm_b200", "csrc")
# DRAM bytes per launch of a kernel from one ncu capture, with the sha256 of
# the kernel source it was taken on (the figure reads as null once it changes).
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-breakdown", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch without programmatic dependent launch (each kernel waits for "
                         "the previous one before it starts)")
    ap.add_argument("--section", default=None,
                    help="run only one breakdown section (o_proj, down_proj, decode, kv, kv_attn, library), e.g. "
                         "to profile its kernels; prints that section's JSON")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def read_traffic(kernel: str):
    """(DRAM bytes per launch, source) of `kernel` from profiles/traffic.json,
    or (None, why) when there is no capture or the source changed since."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, "no ncu capture committed"
    with open(TRAFFIC_FILE) as f:
        rec = json.load(f).get(kernel)
    if rec is None:
        return None, "no ncu capture of this kernel"
    src = os.path.join(CSRC, rec["source"])
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != rec["source_sha256"]:
        return None, "kernel changed since the ncu capture"
    return float(rec["dram_bytes_per_launch"]), "ncu"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples during the timed region (SM clock, throttle reasons)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.th.join(timeout=2)
        sm, smax, reasons, util = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                util.append(float(parts[4]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        loaded = [s for s, u in zip(sm, util) if u > 0] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ distributed
def dist_init():
    import torch
    import torch.distributed as dist
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1 and not dist.is_initialized():
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def max_over_ranks(v: float, ws: int) -> float:
    if ws == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------ our arm
class PrefillReplica:
    """Device buffers of one replica of the prefill workload."""

    def __init__(self, B, torch, x_bits, qkv, gu, dev):
        self.x = torch.from_numpy(x_bits.view(np.int16)).to(dev).view(torch.bfloat16)
        self.qkv = [torch.from_numpy(a).to(dev) for a in qkv]  # Wp, gamma
        self.gu = [torch.from_numpy(a).to(dev) for a in gu]
        M, K = self.x.shape
        self.q4 = torch.empty((M, K), dtype=torch.int8, device=dev)
        self.xs4 = torch.empty(M, dtype=torch.float32, device=dev)
        self.f4 = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        self.xsf = torch.empty(M, dtype=torch.float32, device=dev)
        self.y = {k: torch.empty((M, n), dtype=torch.bfloat16, device=dev)
                  for k, n in (("qkv4", 3 * D), ("gu4", 2 * FFN), ("qkvf", 3 * D), ("guf", 2 * FFN))}


def gemm_call(B, r: PrefillReplica, name):
    """Launch one of the step's four GEMMs on replica r."""
    if name == "w2a4_qkv":
        B.gemm_w2a4(r.q4, r.xs4, r.qkv[0], r.qkv[1], QKV[1], y=r.y["qkv4"])
    elif name == "w2a4_gu":
        B.gemm_w2a4(r.q4, r.xs4, r.gu[0], r.gu[1], GU[1], y=r.y["gu4"])
    elif name == "w2fp4_qkv":
        B.gemm_w2fp4(r.f4, r.xsf, r.qkv[0], r.qkv[1], QKV[1], y=r.y["qkvf"])
    else:
        B.gemm_w2fp4(r.f4, r.xsf, r.gu[0], r.gu[1], GU[1], y=r.y["guf"])


def run_step(B, r: PrefillReplica, ev=None):
    """One step: INT4 quantiser, its two GEMMs, FP4 quantiser, its two GEMMs
    (ev is unused: steps are timed whole)."""
    B.quant_act(r.x, B.MODE_INT4, out=r.q4, xs=r.xs4)
    gemm_call(B, r, "w2a4_qkv")
    gemm_call(B, r, "w2a4_gu")
    B.quant_act(r.x, B.MODE_FP4, out=r.f4, xs=r.xsf)
    gemm_call(B, r, "w2fp4_qkv")
    gemm_call(B, r, "w2fp4_gu")


LAUNCHES_PER_STEP = 6
GEMM_NAMES = ("w2a4_qkv", "w2a4_gu", "w2fp4_qkv", "w2fp4_gu")
GEMM_DESC = {"w2a4_qkv": "gemm_w2a4 q|k|v, tcgen05 kind::i8", "w2a4_gu": "gemm_w2a4 gate|up, tcgen05 kind::i8",
             "w2fp4_qkv": "gemm_w2fp4 q|k|v, tcgen05 kind::mxf4", "w2fp4_gu": "gemm_w2fp4 gate|up, tcgen05 kind::mxf4"}
# names in profiles/traffic.json
KERNEL_IDS = {n: f"gemm_{n}_prefill_2048x2048x{3 * D if 'qkv' in n else 2 * FFN}" for n in
              ("w2a4_qkv", "w2a4_gu", "w2fp4_qkv", "w2fp4_gu")}
# algorithmic bytes of one launch: codes (1 B or 1/2 B per element) + packed weights + bf16 output
GEMM_BYTES = {n: M_TOK * D // (2 if "fp4" in n else 1) + (3 * D if "qkv" in n else 2 * FFN) * D // 4
              + 2 * M_TOK * (3 * D if "qkv" in n else 2 * FFN) for n in ("w2a4_qkv", "w2a4_gu", "w2fp4_qkv", "w2fp4_gu")}
GEMM_OPS = {"w2a4_qkv": 2 * M_TOK * D * 3 * D, "w2a4_gu": 2 * M_TOK * D * 2 * FFN,
            "w2fp4_qkv": 2 * M_TOK * D * 3 * D, "w2fp4_gu": 2 * M_TOK * D * 2 * FFN}


def make_prefill(B, torch, dev, seed):
    import workloads as W
    d = W.input_projection_prefill(seed=seed)
    qkv_p, gu_p = d["projs"]
    qkv = B.ternarize_pack(qkv_p.W, qkv_p.group_ends)
    gu = B.ternarize_pack(gu_p.W, gu_p.group_ends)
    return d, qkv, gu


def graph_set(torch, stream, steps_fns, names, E, timed=True):
    """Capture E copies of each replica's step as CUDA graphs, each copy with
    its own external timing events around the named launches (timed=False:
    no event nodes, for whole-step timing; event nodes inside a graph
    serialise the work around them and add their own cost)."""
    graphs, events = [], []
    with torch.cuda.stream(stream):
        for fn in steps_fns:  # run once eagerly (first-call set-up outside capture)
            fn(None)
    torch.cuda.synchronize()
    for _ in range(E):
        for fn in steps_fns:
            ev = {n: (torch.cuda.Event(enable_timing=True, external=True),
                      torch.cuda.Event(enable_timing=True, external=True)) for n in names} if timed else None
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn(ev)
            graphs.append(g)
            events.append(ev)
    torch.cuda.synchronize()
    return graphs, events


def run_graphs(torch, stream, graphs, events, names, steps, warmup, ws=1, clocks=None):
    """Replay `steps` graphs (rotating) in one timed region; returns (max-over-
    ranks ms for all steps, {name: mean ms per launch over the last steps})."""
    NG = len(graphs)
    for i in range(warmup):
        graphs[i % NG].replay()
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.start()
        time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    off = (NG - steps % NG) % NG  # the last NG steps replay every graph once
    with torch.cuda.stream(stream):
        t0.record()
        for i in range(steps):
            graphs[(i + off) % NG].replay()
        t1.record()
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop() if clocks is not None else None
    ms = max_over_ranks(t0.elapsed_time(t1), ws)
    last = min(steps, NG)
    kms = {}
    for n in (names if events[0] is not None else ()):
        v = [events[j][n][0].elapsed_time(events[j][n][1]) for j in range(NG - last, NG)]
        kms[n] = statistics.mean(v)
    return ms, kms, clk


def time_calls(torch, stream, calls, steps, warm, per_graph=8):
    """Mean device time (ms) of one call: graphs of `per_graph` back-to-back
    calls cycling over `calls` (one closure per buffer replica), no event
    nodes inside, timed as a whole over `steps` graph replays."""
    n = len(calls)
    fns = [(lambda ev, i=i: [calls[(i + j) % n]() for j in range(per_graph)]) for i in range(n)]
    gs, es = graph_set(torch, stream, fns, (), max(1, 8 // n), timed=False)
    ms, _, _ = run_graphs(torch, stream, gs, es, (), steps, warm)
    del gs
    return ms / steps / per_graph


def measure_tensor_peaks(B, torch, stream, reps=3):
    """Dense tensor-pipe rates (TOPS) of this GPU in the GEMMs' MMA shapes,
    best of `reps` (bitlinear_tensor_peak; each run ~2 ms of MMAs)."""
    out = {}
    for kind, name, iters in ((0, "i8_pair", 8192), (1, "mxf4_pair", 8192), (2, "i8_cta", 8192)):
        out[name] = max(B.tensor_peak(kind, iters, stream=stream)["tops"] for _ in range(reps))
    torch.cuda.synchronize()
    return out


def bench_ours(args, ws, rank, local):
    import torch
    import bit_quantised_gemm_b200 as B
    dev = f"cuda:{local}"
    torch.cuda.set_device(local)
    B.lib()
    B.set_launch_overlap(not args.no_overlap)
    d, qkv, gu = make_prefill(B, torch, dev, args.seed)
    R = 3
    reps = [PrefillReplica(B, torch, d["x"], qkv, gu, dev) for _ in range(R)]
    stream = torch.cuda.Stream(device=dev)
    fns = [(lambda ev, r=r: run_step(B, r, ev)) for r in reps]
    # whole-step timing: graphs without event nodes
    graphs, events = graph_set(torch, stream, fns, GEMM_NAMES, E=8, timed=False)
    B.check_status(stream=stream)
    ms, _, clk = run_graphs(torch, stream, graphs, events, GEMM_NAMES, args.steps, args.warmup,
                            ws, ClockSampler(local))
    B.check_status(stream=stream)
    del graphs
    # per-kernel durations: each GEMM alone, back to back over the replicas
    ksteps, kwarm = min(args.steps, 240), max(3, args.warmup // 4)
    kms = {n: time_calls(torch, stream, [(lambda r=r, n=n: gemm_call(B, r, n)) for r in reps],
                         ksteps, kwarm) for n in GEMM_NAMES}
    B.check_status(stream=stream)

    peaks, peak_src = load_peaks()
    int8_peak = RATIO_INT8 * peaks["bf16_tflops"]
    fp4_peak = RATIO_FP4 * peaks["bf16_tflops"]
    pipe = measure_tensor_peaks(B, torch, stream)
    # the roofline is reported on the kernel that takes the largest share of the step
    dom = max(GEMM_NAMES, key=lambda n: kms[n])
    dom_int8 = "w2a4" in dom
    ach = GEMM_OPS[dom] / (kms[dom] * 1e-3) / 1e12
    traffic, tsrc = read_traffic(KERNEL_IDS[dom])
    dom_peak = int8_peak if dom_int8 else fp4_peak
    dom_pipe = pipe["i8_pair"] if dom_int8 else pipe["mxf4_pair"]
    roofline = {"bound": "tensor", "kernel": f"{dom} ({GEMM_DESC[dom]})",
                "achieved": round(ach, 1), "peak": round(dom_peak, 1), "unit": "TOPS",
                "frac": round(ach / dom_peak, 4), "traffic": traffic, "traffic_source": tsrc,
                "algorithmic_bytes": GEMM_BYTES[dom],
                "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} TF/s x "
                               f"{RATIO_INT8 if dom_int8 else RATIO_FP4} (nominal dense ratio to bf16)",
                "measured_pipe_peak": round(dom_pipe, 1),
                "frac_of_measured_pipe": round(ach / dom_pipe, 4),
                "pipe_peak_source": "bitlinear_tensor_peak in this run: back-to-back tcgen05 MMAs of the "
                                    "GEMM's own kind and shape on resident operands, every SM",
                "timing": "the GEMM alone: CUDA graphs of 8 back-to-back launches over the 3 replicas, "
                          "CUDA events on the launching stream"}
    kernels = {}
    for n in GEMM_NAMES:
        tops = GEMM_OPS[n] / (kms[n] * 1e-3) / 1e12
        i8 = "w2a4" in n
        pk = int8_peak if i8 else fp4_peak
        pp = pipe["i8_pair"] if i8 else pipe["mxf4_pair"]
        nom = NOMINAL["int8_tops"] if i8 else NOMINAL["fp4_tflops"]
        kernels[n] = {"us": round(kms[n] * 1e3, 2), "TOPS": round(tops, 1),
                      "frac_of_peak": round(tops / pk, 4), "frac_of_measured_pipe": round(tops / pp, 4),
                      "frac_of_nominal": round(tops / nom, 4),
                      "peak": "int8 (bf16 x 2)" if i8 else "fp4 (bf16 x 4; tcgen05 kind::mxf4, block scales 1.0)"}

    value = OPS_PER_STEP * args.steps * ws / (ms * 1e-3) / 1e12
    out = {"metric": METRIC, "value": round(value, 2), "unit": "TOPS", "n_gpus": ws,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "s8,e2m1 (x ternary)", "data": "synthetic",
           "config": {"workload": WORKLOAD, "tokens": M_TOK, "d_model": D, "qkv_out": 3 * D,
                      "gate_up_out": 2 * FFN, "variants": ["INT4 (s8 MMA)", "FP4 e2m1 (mxf4 MMA, unit block scales)"],
                      "parallelism": f"replicas x{ws}",
                      "l2": f"{R} rotating replicas of all inputs/weights/outputs (>270 MB > 126 MB L2)",
                      "graphs": "one CUDA graph per step",
                      "launch_overlap": not args.no_overlap},
           "roofline": roofline, "tensor_pipe_peaks_TOPS": {k: round(v, 1) for k, v in pipe.items()},
           "kernels": kernels, "clocks": clk,
           "gpu_launches": LAUNCHES_PER_STEP * args.steps}
    return out, (d, qkv, gu, reps, B, torch, dev, stream)


def bench_e2e(args, ctx, ws):
    """Same metric through the Python API with host buffers: per step the
    H2D copy of X from pinned memory, the six calls, and the D2H copies of
    the four outputs are inside the timed region."""
    d, qkv, gu, reps, B, torch, dev, stream = ctx
    r = reps[0]
    x_host = torch.from_numpy(d["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    outs = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in r.y.items()}
    steps = args.steps
    h2d = x_host.numel() * 2
    d2h = sum(v.numel() * 2 for v in outs.values())
    with torch.cuda.stream(stream):
        for _ in range(max(1, args.warmup // 4)):
            r.x.copy_(x_host, non_blocking=True)
            run_step(B, r)
            for k, v in outs.items():
                v.copy_(r.y[k], non_blocking=True)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        t0.record()
        for _ in range(steps):
            r.x.copy_(x_host, non_blocking=True)
            run_step(B, r)
            for k, v in outs.items():
                v.copy_(r.y[k], non_blocking=True)
        t1.record()
    torch.cuda.synchronize()
    barrier(ws)
    ms = max_over_ranks(t0.elapsed_time(t1), ws)
    B.check_status(stream=stream)
    return {"value": round(OPS_PER_STEP * steps * ws / (ms * 1e-3) / 1e12, 3), "unit": "TOPS",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms / steps, 4), "path": "python API (ctypes -> C ABI), pinned host buffers"}


# ------------------------------------------------------- CPU oracle timing
def _window(wt, c0, width):
    """Columns [c0, c0+width) of a ternarised projection: (W_t slice, gamma, group ends)."""
    Wt, gamma, ends = wt
    c1 = min(c0 + width, Wt.shape[1])
    g_sub, e_sub, start = [], [], 0
    for gm, end in zip(gamma, ends):
        lo, hi = max(start, c0), min(end, c1)
        if lo < hi:
            g_sub.append(gm)
            e_sub.append(hi - c0)
        start = end
    return Wt[:, c0:c1], np.array(g_sub, np.float32), tuple(e_sub)


def oracle_sample(d, qkv_wt, gu_wt, rows, col0=0, width=None):
    """Oracle on a sample of the workload: the given token rows through both
    variants, against a window of `width` output columns of each projection
    (all of them when width is None). Returns the sample's ops."""
    from oracle import bitlinear_oracle as O
    x = d["x"][rows]
    ops = 0
    q4, xs4 = O.quant_act(x, O.MODE_INT4)
    f4, xsf = O.quant_act(x, O.MODE_FP4)
    for wt in (qkv_wt, gu_wt):
        n_all = wt[0].shape[1]
        w = n_all if width is None else width
        Wt, g, e = _window(wt, (col0 * w) % n_all if width else 0, w)
        O.bitlinear_int(q4, xs4, Wt, g, e)
        O.bitlinear_fp4(f4, xsf, Wt, g, e)
        ops += 2 * 2 * len(rows) * Wt.shape[0] * Wt.shape[1]
    return ops


def oracle_weights(d):
    from oracle import bitlinear_oracle as O
    qkv_p, gu_p = d["projs"]
    return (O.ternarize(qkv_p.W, qkv_p.group_ends) + (qkv_p.group_ends,),
            O.ternarize(gu_p.W, gu_p.group_ends) + (gu_p.group_ends,))


def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i.get("num_threads") for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def _oracle_rate(d, qkv_wt, gu_wt, budget_s, block):
    ops, t, rows_done = 0.0, 0.0, 0
    while t < budget_s and rows_done < M_TOK:
        rows = np.arange(rows_done, min(M_TOK, rows_done + block))
        t0 = time.perf_counter()
        ops += oracle_sample(d, qkv_wt, gu_wt, rows)
        t += time.perf_counter() - t0
        rows_done += len(rows)
    return ops / t / 1e12, rows_done, t


def cpu_baseline(d, budget_s=8.0, block=32):
    """The oracle as it stands on the host cores, on the first token rows of
    the workload that fit the time budget: once with NumPy's BLAS on every
    core, once on one thread. A baseline, not a target."""
    from threadpoolctl import threadpool_limits
    qkv_wt, gu_wt = oracle_weights(d)
    v_all, rows_all, t_all = _oracle_rate(d, qkv_wt, gu_wt, budget_s, block)
    cores = blas_threads()
    with threadpool_limits(limits=1):
        v_one, rows_one, t_one = _oracle_rate(d, qkv_wt, gu_wt, budget_s, block)
    return {"value": round(v_all, 6), "unit": "TOPS", "cores": cores, "kind": "oracle",
            "sample": f"first {rows_all} of {M_TOK} token rows through both variants ({t_all:.1f} s of CPU "
                      f"time; weight ternarisation untimed)",
            "single_thread": {"value": round(v_one, 6), "unit": "TOPS", "cores": 1,
                              "sample": f"first {rows_one} token rows ({t_one:.1f} s)"}}


def bench_reference(args, ws, rank):
    """The oracle on host cores, as it stands, in the same metric."""
    if rank != 0:
        return None
    import workloads as W
    d = W.input_projection_prefill(seed=args.seed)
    qkv_wt, gu_wt = oracle_weights(d)
    block, width = 8, 512
    for i in range(args.warmup):
        s0 = (i * block) % M_TOK
        oracle_sample(d, qkv_wt, gu_wt, np.arange(s0, s0 + block), i, width)
    ops = 0.0
    t0 = time.perf_counter()
    for i in range(args.steps):
        s0 = (i * block) % M_TOK
        ops += oracle_sample(d, qkv_wt, gu_wt, np.arange(s0, s0 + block), i, width)
    t = time.perf_counter() - t0
    value = ops / t / 1e12
    sample = (f"each step: {block} of the {M_TOK} token rows through both variants against a "
              f"{width}-column window of each projection (rotating rows and windows)")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TOPS",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t * 1e3 / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens": M_TOK, "d_model": D},
            "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------ breakdown
def _dev_bf16(torch, bits, dev):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)


SECTIONS = ("o_proj", "down_proj", "decode", "kv", "kv_attn", "library")


def breakdown(ctx, args, sections=SECTIONS, pipe=None):
    """The other workloads of the path, each timed the same way (rotating
    replicas larger than L2, CUDA graphs without event nodes; a kernel's time
    is that of a graph of back-to-back launches of it alone). `pipe`: the
    tensor-pipe rates measured in this run (measured here when None)."""
    B, torch, dev, stream = ctx[4], ctx[5], ctx[6], ctx[7]
    peaks, src = load_peaks()
    peaks = dict(peaks, pipe=pipe if pipe is not None else measure_tensor_peaks(B, torch, stream))
    out = {"peaks": f"{src}: HBM {peaks['hbm_gbs']} GB/s, int8 {RATIO_INT8 * peaks['bf16_tflops']:.0f} "
                    "TOPS (2 x bf16 burst)"}
    steps, warm = max(24, min(args.steps, 200)), min(5, args.warmup)
    for name in sections:
        out.update(globals()["section_" + name](B, torch, dev, stream, peaks, steps, warm))
    B.check_status(stream=stream)
    return out


def section_o_proj(B, torch, dev, stream, peaks, steps, warm):
    """o_proj: top-k 50% + INT8, then the s8 GEMM 4096 x 4096 x 4096."""
    import workloads as W
    hbm, int8_peak = peaks["hbm_gbs"], RATIO_INT8 * peaks["bf16_tflops"]
    out = {}
    o = W.o_proj_sparse()
    Wp, g = B.ternarize_pack(o["proj"].W, (4096,))
    M, K, N = 4096, 4096, 4096
    bufs = []
    for _ in range(3):
        bufs.append(dict(x=_dev_bf16(torch, o["x"], dev), Wp=torch.from_numpy(Wp).to(dev),
                         g=torch.from_numpy(g).to(dev), q=torch.empty((M, K), dtype=torch.int8, device=dev),
                         xs=torch.empty(M, dtype=torch.float32, device=dev),
                         y=torch.empty((M, N), dtype=torch.bfloat16, device=dev)))

    def topk(b): B.topk_sparsify_i8(b["x"], out=b["q"], xs=b["xs"])
    def gemm(b): B.gemm_w2a8(b["q"], b["xs"], b["Wp"], b["g"], (N,), y=b["y"])

    def o_step(ev, b):
        topk(b)
        gemm(b)
    gs, es = graph_set(torch, stream, [(lambda ev, b=b: o_step(ev, b)) for b in bufs], (), 8, timed=False)
    ms, _, _ = run_graphs(torch, stream, gs, es, (), steps, warm)
    del gs
    k = {"topk": time_calls(torch, stream, [(lambda b=b: topk(b)) for b in bufs], steps, warm),
         "gemm": time_calls(torch, stream, [(lambda b=b: gemm(b)) for b in bufs], steps, warm)}
    ops = 2 * M * K * N
    tb = M * K * 2 + M * K + M * 4
    out["o_proj_topk_w2a8_4096x4096x4096"] = {
        "step_us": round(ms / steps * 1e3, 2),
        "gemm_us": round(k["gemm"] * 1e3, 2), "gemm_TOPS": round(ops / k["gemm"] / 1e9, 1),
        "gemm_frac_int8": round(ops / k["gemm"] / 1e9 / int8_peak, 4),
        "gemm_frac_of_pipe": round(ops / k["gemm"] / 1e9 / peaks["pipe"]["i8_pair"], 4),
        "topk_us": round(k["topk"] * 1e3, 2), "topk_GBps": round(tb / k["topk"] / 1e6, 1),
        "topk_frac_hbm": round(tb / k["topk"] / 1e6 / hbm, 4)}
    return out


def section_down_proj(B, torch, dev, stream, peaks, steps, warm):
    """down_proj: ReLU^2 gate + INT8, then the s8 GEMM 4096 x 11008 x 4096."""
    import workloads as W
    hbm, int8_peak = peaks["hbm_gbs"], RATIO_INT8 * peaks["bf16_tflops"]
    out = {}
    dn = W.down_proj_relu2()
    Wp, g = B.ternarize_pack(dn["proj"].W, (4096,))
    M, K, N = 4096, 11008, 4096
    b = dict(gate=_dev_bf16(torch, dn["gate"], dev), up=_dev_bf16(torch, dn["up"], dev),
             Wp=torch.from_numpy(Wp).to(dev), g=torch.from_numpy(g).to(dev),
             q=torch.empty((M, K), dtype=torch.int8, device=dev),
             xs=torch.empty(M, dtype=torch.float32, device=dev),
             y=torch.empty((M, N), dtype=torch.bfloat16, device=dev))
    del dn

    b2 = dict(b, q=torch.empty_like(b["q"]), y=torch.empty_like(b["y"]), Wp=b["Wp"].clone())

    def quant(b): B.quant_act(b["gate"], B.MODE_INT8, up=b["up"], out=b["q"], xs=b["xs"])
    def gemm(b): B.gemm_w2a8(b["q"], b["xs"], b["Wp"], b["g"], (N,), y=b["y"])

    def d_step(ev):
        quant(b)
        gemm(b)
    gs, es = graph_set(torch, stream, [d_step], (), 24, timed=False)
    ms, _, _ = run_graphs(torch, stream, gs, es, (), steps, warm)
    del gs
    quant(b2)
    # gate/up (180 MB) exceed L2 on their own; the GEMM alone alternates two
    # sets of codes/weights/outputs (2 x 88 MB)
    k = {"quant": time_calls(torch, stream, [lambda: quant(b)], steps, warm),
         "gemm": time_calls(torch, stream, [lambda: gemm(b), lambda: gemm(b2)], steps, warm)}
    ops = 2 * M * K * N
    qb = 2 * M * K * 2 + M * K + M * 4
    zero_codes = float((b["q"] == 0).float().mean().item())
    out["down_proj_relu2_w2a8_4096x11008x4096"] = {
        "step_us": round(ms / steps * 1e3, 2),
        "gemm_us": round(k["gemm"] * 1e3, 2), "gemm_TOPS": round(ops / k["gemm"] / 1e9, 1),
        "gemm_frac_int8": round(ops / k["gemm"] / 1e9 / int8_peak, 4),
        "gemm_frac_of_pipe": round(ops / k["gemm"] / 1e9 / peaks["pipe"]["i8_pair"], 4),
        "relu2_quant_us": round(k["quant"] * 1e3, 2), "relu2_quant_GBps": round(qb / k["quant"] / 1e6, 1),
        "relu2_quant_frac_hbm": round(qb / k["quant"] / 1e6 / hbm, 4),
        "zero_code_fraction": round(zero_codes, 4)}
    return out


def section_decode(B, torch, dev, stream, peaks, steps, warm):
    """Decode: one LLaMA-7B-shaped layer at batch 1 / 4 / 8 / 64 (weight GB/s).

    The projections that share an input run as one launch with per-group
    scales (q|k|v: N = 12288, 3 groups; gate|up: N = 22016, 2 groups), then
    o (4096) and down (11008 -> 4096): four GEMV launches per layer."""
    import workloads as W
    hbm = peaks["hbm_gbs"]
    out = {}
    lay = W.decode_layer(batch=64, make_kv=False)
    P = {p.name: p for p in lay["projs"]}
    D, F = P["q"].K, P["gate"].N
    fused = {
        "qkv": (np.concatenate([P["q"].W, P["k"].W, P["v"].W], axis=1), (D, 2 * D, 3 * D)),
        "o": (P["o"].W, (D,)),
        "gate_up": (np.concatenate([P["gate"].W, P["up"].W], axis=1), (F, 2 * F)),
        "down": (P["down"].W, (D,)),
    }
    packed = {k: B.ternarize_pack(w, ge) for k, (w, ge) in fused.items()}
    shapes = {k: (w.shape[0], w.shape[1], ge) for k, (w, ge) in fused.items()}
    del fused, lay["projs"]
    wbytes = sum(K * N // 4 for K, N, _ in shapes.values())
    R = 6  # weight replicas: 6 x 48 MB > 2 x L2
    wdev = [{k: (torch.from_numpy(wp).to(dev), torch.from_numpy(gm).to(dev)) for k, (wp, gm) in packed.items()}
            for _ in range(R)]
    names = tuple(shapes)
    # the six K = 4096 projections as one grouped launch (q|k|v|o|gate|up
    # concatenated, one scale group each, one shared input: a weight-streaming
    # measure, not the layer's data flow), plus down: 2 launches for all 7
    six = ("q", "k", "v", "o", "gate", "up")
    g_ends = tuple(int(e) for e in np.cumsum([P[n].N for n in six]))
    g_wp, g_gm = B.ternarize_pack(np.concatenate([P[n].W for n in six], axis=1), g_ends)
    g_dev = [(torch.from_numpy(g_wp).to(dev), torch.from_numpy(g_gm).to(dev)) for _ in range(R)]
    g_bytes = D * g_ends[-1] // 4
    del g_wp
    dec = {}
    for batch in (1, 4, 8, 64):
        x = _dev_bf16(torch, lay["x"][:batch], dev)
        xo = _dev_bf16(torch, lay["xo"][:batch], dev)
        ga = _dev_bf16(torch, lay["gate"][:batch], dev)
        up = _dev_bf16(torch, lay["up"][:batch], dev)
        ys = {k: torch.empty((batch, N), dtype=torch.bfloat16, device=dev) for k, (_, N, _) in shapes.items()}
        q4 = torch.empty((batch, D), dtype=torch.int8, device=dev)
        xs4 = torch.empty(batch, dtype=torch.float32, device=dev)
        qo = torch.empty((batch, D), dtype=torch.int8, device=dev)
        xso = torch.empty(batch, dtype=torch.float32, device=dev)
        qd = torch.empty((batch, F), dtype=torch.int8, device=dev)
        xsd = torch.empty(batch, dtype=torch.float32, device=dev)

        ins = {"qkv": (q4, xs4), "o": (qo, xso), "gate_up": (q4, xs4), "down": (qd, xsd)}

        def gemv(name, r):
            xq, xs = ins[name]
            B.gemv_w2(xq, xs, wdev[r][name][0], wdev[r][name][1], shapes[name][2], y=ys[name])

        def l_step(ev, r):
            B.quant_act(x, B.MODE_INT4, out=q4, xs=xs4)
            gemv("qkv", r)
            B.topk_sparsify_i8(xo, out=qo, xs=xso)
            gemv("o", r)
            gemv("gate_up", r)
            B.quant_act(ga, B.MODE_INT8, up=up, out=qd, xs=xsd)
            gemv("down", r)
        gs, es = graph_set(torch, stream, [(lambda ev, r=r: l_step(ev, r)) for r in range(R)], (), 4,
                           timed=False)
        ms, _, _ = run_graphs(torch, stream, gs, es, (), steps, warm)
        del gs
        k = {n: time_calls(torch, stream, [(lambda n=n, r=r: gemv(n, r)) for r in range(R)], steps, warm)
             for n in names}
        gemv_ms = sum(k.values())
        fused = {}
        if batch <= 8:
            # the quantisers inside the GEMVs (bitlinear_gemv_w2_quant): 5 launches per layer
            fq = {"qkv": (x, None, B.MODE_INT4), "gate_up": (x, None, B.MODE_INT4),
                  "down": (ga, up, B.MODE_INT8)}

            def gemv_q(name, r):
                xa, ua, mode = fq[name]
                B.gemv_w2_quant(xa, mode, wdev[r][name][0], wdev[r][name][1], shapes[name][2], up=ua,
                                y=ys[name])

            def l_step_fused(ev, r):
                gemv_q("qkv", r)
                B.topk_sparsify_i8(xo, out=qo, xs=xso)
                gemv("o", r)
                gemv_q("gate_up", r)
                gemv_q("down", r)
            gs, es = graph_set(torch, stream, [(lambda ev, r=r: l_step_fused(ev, r)) for r in range(R)],
                               (), 4, timed=False)
            fms, _, _ = run_graphs(torch, stream, gs, es, (), steps, warm)
            del gs
            fk = {n: time_calls(torch, stream, [(lambda n=n, r=r: gemv_q(n, r)) for r in range(R)], steps, warm)
                  for n in fq}
            fused = {"layer_step_us_quantisers_fused": round(fms / steps * 1e3, 2),
                     "fused_gemv_us": {n: round(v * 1e3, 2) for n, v in fk.items()},
                     "fused_note": "q|k|v, gate|up and down quantise their bf16 inputs inside the GEMV "
                                   "(bitlinear_gemv_w2_quant); o keeps the separate top-k launch"}
        per = {n: {"us": round(k[n] * 1e3, 2), "GBps": round(K_ * N_ // 4 / k[n] / 1e6, 1)}
               for n, (K_, N_, _) in shapes.items()}
        dec[f"batch{batch}"] = {
            "layer_step_us": round(ms / steps * 1e3, 2),
            "gemv_sum_us": round(gemv_ms * 1e3, 2),
            "gemv_sum_note": "each projection timed alone, back to back over 6 weight replicas",
            "weight_GBps": round(wbytes / gemv_ms / 1e6, 1),
            "weight_frac_hbm": round(wbytes / gemv_ms / 1e6 / hbm, 4),
            "layer_weight_GBps_incl_quantisers": round(wbytes / (ms / steps) / 1e6, 1),
            "per_projection": per, **fused}
        if batch in (1, 8):
            yg = torch.empty((batch, g_ends[-1]), dtype=torch.bfloat16, device=dev)
            tg = time_calls(torch, stream, [(lambda r=r: B.gemv_w2(q4, xs4, g_dev[r][0], g_dev[r][1], g_ends,
                                                                  y=yg)) for r in range(R)], steps, warm)
            tot = tg + k["down"]
            dec[f"batch{batch}"]["grouped_7_projections"] = {
                "launches": 2, "us": round(tot * 1e3, 2), "six_k4096_us": round(tg * 1e3, 2),
                "weight_GBps": round((g_bytes + shapes["down"][0] * shapes["down"][1] // 4) / tot / 1e6, 1),
                "weight_frac_hbm": round((g_bytes + shapes["down"][0] * shapes["down"][1] // 4) / tot / 1e6 / hbm, 4)}
    out["decode_llama7b_layer"] = dict(weight_bytes=wbytes, launches_per_layer=7,
                                       gemv_launches="qkv (fused, 3 groups), o, gate_up (fused, 2 groups), down",
                                       **dec)
    return out


def section_kv(B, torch, dev, stream, peaks, steps, warm):
    """KV cache: K and V [4096 x 32 x 128] -> 3-bit codes, bos at 4 bits; both
    tensors in one launch (kv_quant_3bit_kv), and as two kv_quant_3bit calls."""
    import workloads as W
    hbm = peaks["hbm_gbs"]
    out = {}
    kvd = W.decode_layer(batch=1, make_weights=False)
    keep = torch.tensor([0], dtype=torch.int32, device=dev)
    kvs = [(_dev_bf16(torch, kvd["k_cache"], dev), _dev_bf16(torch, kvd["v_cache"], dev)) for _ in range(4)]
    T, H, Dh = kvd["k_cache"].shape
    o3 = [torch.empty((T, H, 3 * Dh // 8), dtype=torch.uint8, device=dev) for _ in range(2)]
    o4 = [torch.empty((1, H, Dh // 2), dtype=torch.uint8, device=dev) for _ in range(2)]
    sc = [torch.empty((T, H), dtype=torch.float32, device=dev) for _ in range(2)]

    def kv_step(r):
        B.kv_quant_3bit_kv(kvs[r][0], kvs[r][1], keep, k_store=(o3[0], o4[0], sc[0]),
                           v_store=(o3[1], o4[1], sc[1]))

    def kv_step_two_calls(r):
        for j in range(2):
            B.kv_quant_3bit(kvs[r][j], keep, codes3=o3[j], codes4=o4[j], scale=sc[j])
    k = {"kv": time_calls(torch, stream, [(lambda r=r: kv_step(r)) for r in range(4)], steps, warm),
         "two": time_calls(torch, stream, [(lambda r=r: kv_step_two_calls(r)) for r in range(4)], steps, warm)}
    kb = 2 * (T * H * Dh * 2 + T * H * 3 * Dh // 8 + T * H * 4 + H * Dh // 2)
    out["kv_quant_3bit_2x4096x32x128"] = {"us": round(k["kv"] * 1e3, 2),
                                         "GBps": round(kb / k["kv"] / 1e6, 1),
                                         "frac_hbm": round(kb / k["kv"] / 1e6 / hbm, 4),
                                         "launches": 1, "us_two_launches": round(k["two"] * 1e3, 2)}
    return out


def section_kv_attn(B, torch, dev, stream, peaks, steps, warm):
    """Decode attention over the 3-bit cache of one layer (K and V [4096 x 32
    x 128], bos at 4 bits) for 1 and 8 queries per head."""
    import workloads as W
    hbm = peaks["hbm_gbs"]
    kvd = W.decode_layer(batch=1, make_weights=False)
    T, H, Dh = kvd["k_cache"].shape
    keep = torch.tensor([0], dtype=torch.int32, device=dev)
    k_src, v_src = _dev_bf16(torch, kvd["k_cache"], dev), _dev_bf16(torch, kvd["v_cache"], dev)
    R = 12  # cache replicas: 12 x 13.6 MB > L2
    stores = [(B.kv_quant_3bit(k_src, keep), B.kv_quant_3bit(v_src, keep)) for _ in range(R)]
    del k_src, v_src
    cache_bytes = 2 * (T * H * 3 * Dh // 8 + T * H * 4 + H * Dh // 2)
    out = {}
    for nq in (1, 8):
        q = _dev_bf16(torch, W.normal_bf16(np.random.default_rng(nq), (nq, H, Dh)), dev)
        o = torch.empty((nq, H, Dh), dtype=torch.bfloat16, device=dev)
        ms = time_calls(torch, stream, [(lambda r=r: B.kv_attention_3bit(q, stores[r][0], stores[r][1], keep,
                                                                             out=o)) for r in range(R)],
                        steps, warm)
        byt = cache_bytes + 2 * 2 * nq * H * Dh
        out[f"queries{nq}"] = {"us": round(ms * 1e3, 2), "GBps": round(byt / ms / 1e6, 1),
                               "frac_hbm": round(byt / ms / 1e6 / hbm, 4)}
    return {"kv_attention_3bit_4096x32x128": dict(cache_bytes=cache_bytes, **out)}


def section_library(B, torch, dev, stream, peaks, steps, warm):
    """Library references on the prefill shapes (not this library's kernels):
    cuBLAS int8 GEMM (torch._int_mm) and fp8 e4m3 GEMM (torch._scaled_mm, unit
    scales) on plain 8-bit operands with no unpack, an mxfp4 torch._scaled_mm
    where this torch offers it, and a read-only HBM stream (a torch sum over
    2 GiB). Each timed like the kernels above over 3 operand replicas."""
    out = {}
    int8_peak, hbm = RATIO_INT8 * peaks["bf16_tflops"], peaks["hbm_gbs"]
    shapes = {"qkv": (M_TOK, D, 3 * D), "gate_up": (M_TOK, D, 2 * FFN)}

    def rate(name, M, K, N, fn_make, peak, nominal):
        try:
            calls = [fn_make() for _ in range(3)]
            ms = time_calls(torch, stream, calls, steps, warm)
            tops = 2 * M * K * N / (ms * 1e-3) / 1e12
            out[name] = {"us": round(ms * 1e3, 2), "TOPS": round(tops, 1),
                         "frac_of_peak": round(tops / peak, 4), "frac_of_nominal": round(tops / nominal, 4)}
        except Exception as e:  # an unsupported dtype or shape in this torch / cuBLAS
            out[name] = {"unavailable": f"{type(e).__name__}: {str(e).splitlines()[0][:160]}"}
        torch.cuda.synchronize()

    for sh, (M, K, N) in shapes.items():
        def mk_i8(M=M, K=K, N=N):
            a = torch.randint(-8, 8, (M, K), dtype=torch.int8, device=dev)
            b = torch.randint(-1, 2, (N, K), dtype=torch.int8, device=dev).t()
            return lambda: torch._int_mm(a, b)
        rate(f"cublas_int8_{sh}", M, K, N, mk_i8, int8_peak, NOMINAL["int8_tops"])

        def mk_f8(M=M, K=K, N=N):
            a = torch.randn(M, K, device=dev).to(torch.float8_e4m3fn)
            b = torch.randn(N, K, device=dev).to(torch.float8_e4m3fn).t()
            one = torch.ones((), device=dev)
            return lambda: torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16)
        rate(f"cublaslt_fp8_{sh}", M, K, N, mk_f8, RATIO_INT8 * peaks["bf16_tflops"], NOMINAL["fp8_tflops"])

        def mk_f4(M=M, K=K, N=N):
            a = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev).view(torch.float4_e2m1fn_x2)
            b = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev).view(torch.float4_e2m1fn_x2).t()
            # every e8m0 block scale 1.0 (127): the same in any scale layout, so
            # the first layout this torch accepts is used
            import torch.nn.functional as F
            err = None
            for swz in ("SWIZZLE_32_4_4", "NO_SWIZZLE"):
                for flat in (True, False):
                    shp_a, shp_b = ((M * K // 32,), (N * K // 32,)) if flat else ((M, K // 32), (N, K // 32))
                    sa = torch.full(shp_a, 127, dtype=torch.uint8, device=dev).view(torch.float8_e8m0fnu)
                    sb = torch.full(shp_b, 127, dtype=torch.uint8, device=dev).view(torch.float8_e8m0fnu)
                    bw, sw = F.ScalingType.BlockWise1x32, getattr(F.SwizzleType, swz)
                    call = (lambda sa=sa, sb=sb, bw=bw, sw=sw: F.scaled_mm(
                        a, b, sa, bw, sb, bw, swizzle_a=sw, swizzle_b=sw, output_dtype=torch.bfloat16))
                    try:
                        call()
                        return call
                    except (RuntimeError, ValueError, TypeError) as e:
                        err = e
            raise err
        rate(f"cublaslt_mxfp4_{sh}", M, K, N, mk_f4, RATIO_FP4 * peaks["bf16_tflops"], NOMINAL["fp4_tflops"])

    try:
        buf = torch.ones(2 << 30 >> 2, dtype=torch.float32, device=dev)  # 2 GiB
        ms = time_calls(torch, stream, [lambda: buf.sum()], max(8, steps // 8), warm, per_graph=2)
        gbs = buf.numel() * 4 / (ms * 1e-3) / 1e9
        out["hbm_read_stream_2GiB"] = {"us": round(ms * 1e3, 1), "GBps": round(gbs, 1),
                                       "frac_of_measured_copy": round(gbs / hbm, 4),
                                       "frac_of_nominal": round(gbs / NOMINAL["hbm_gbs"], 4)}
        del buf
    except Exception as e:
        out["hbm_read_stream_2GiB"] = {"unavailable": f"{type(e).__name__}: {str(e)[:160]}"}
    torch.cuda.empty_cache()
    return {"library_reference": out}


def summary(out):
    """The headline fractions in a few hundred bytes: GEMMs against the tensor
    pipe measured in this run, decode GEMVs and the HBM-bound kernels against
    the measured copy bandwidth."""
    r = lambda v: round(v, 3) if isinstance(v, float) else v
    sm = {"prefill_TOPS": out["value"], "roofline_frac": out["roofline"]["frac"],
          "pipe_TOPS": out.get("tensor_pipe_peaks_TOPS"),
          "gemm_frac_of_pipe": {n: r(k["frac_of_measured_pipe"]) for n, k in out["kernels"].items()}}
    b = out.get("breakdown", {})
    o = b.get("o_proj_topk_w2a8_4096x4096x4096", {})
    dn = b.get("down_proj_relu2_w2a8_4096x11008x4096", {})
    if o:
        sm["gemm_frac_of_pipe"]["o_proj"] = r(o.get("gemm_frac_of_pipe"))
        sm["topk_frac_hbm"] = r(o.get("topk_frac_hbm"))
    if dn:
        sm["gemm_frac_of_pipe"]["down_proj"] = r(dn.get("gemm_frac_of_pipe"))
        sm["relu2_quant_frac_hbm"] = r(dn.get("relu2_quant_frac_hbm"))
    dec = b.get("decode_llama7b_layer", {})
    if dec:
        sm["decode_weight_frac_hbm"] = {k: r(v["weight_frac_hbm"]) for k, v in dec.items() if k.startswith("batch")}
        sm["decode_gemv_us"] = {k: r(v["gemv_sum_us"]) for k, v in dec.items() if k.startswith("batch")}
    kv = b.get("kv_quant_3bit_2x4096x32x128")
    if kv:
        sm["kv_quant_frac_hbm"] = r(kv["frac_hbm"])
    at = b.get("kv_attention_3bit_4096x32x128")
    if at:
        sm["kv_attn_frac_hbm"] = {q: r(at[q]["frac_hbm"]) for q in ("queries1", "queries8") if q in at}
    if "e2e" in out:
        sm["e2e_TOPS"] = out["e2e"]["value"]
    if "cpu_baseline" in out:
        sm["cpu_TOPS"] = {"all_cores": out["cpu_baseline"]["value"],
                          "one_core": out["cpu_baseline"]["single_thread"]["value"]}
    return sm


def main():
    args = parse()
    ws, rank, local = dist_init()
    if args.section:
        import torch
        import bit_quantised_gemm_b200 as B
        torch.cuda.set_device(local)
        B.lib()
        B.set_launch_overlap(not args.no_overlap)
        stream = torch.cuda.Stream(device=f"cuda:{local}")
        ctx = (None, None, None, None, B, torch, f"cuda:{local}", stream)
        print(json.dumps(breakdown(ctx, args, (args.section,))), flush=True)
        return
    if args.impl == "reference":
        out = bench_reference(args, ws, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    out, ctx = bench_ours(args, ws, rank, local)
    if not args.no_e2e:
        out["e2e"] = bench_e2e(args, ctx, ws)
    if rank == 0 and ws == 1 and not args.no_breakdown:
        pipe = {k: v for k, v in out["tensor_pipe_peaks_TOPS"].items()}
        out["breakdown"] = breakdown(ctx, args, pipe=pipe)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(ctx[0])
    if rank == 0:
        out["summary"] = summary(out)  # last: the end of the line is what a log tail keeps
        print(json.dumps(out), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
