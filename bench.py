#!/usr/bin/env python
"""Benchmark of the packed binary (+1/-1) matrix product on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--no-rows] [--no-cpu-baseline] [--no-e2e]

Headline (one JSON line on rank 0): the batch-1 LLM-decode binary GEMV,
packed +1/-1 weights [11008, 4096] (from N(0, 0.02)), activation x bf16 [4096]
binarised and packed inside the kernel, alpha-scaled fp32 output; metric =
algorithmic GB/s.  One step = one GEMV (x pack + XOR/popcount + alpha
epilogue) through the C ABI.  K steps are captured in CUDA graphs and timed
with CUDA events on the launching stream; steps rotate over 48 copies of the
packed weights (270 MB, more than the 126 MB L2), so every step streams its
weights from HBM.

Also on the line:
  roofline      the GEMV kernel against the measured HBM copy bandwidth.
  cpu_baseline  the CPU oracle on a bounded sample of the same workload.
  e2e           the same metric through the public API with host buffers: per
                step, pinned x -> device, GEMV, y -> pinned host.
  rows          the other hot-path rows, each timed the same way: weight pack
                + alpha (HBM GB/s), the square 8192^3 GEMM, the ResNet-class
                3x3 binary convolution and the 4-layer binary MLP (binary MAC/s
                against the integer-pipe roofline).
Under torchrun (N > 1) every rank runs its own replica of the workload (the
path has no data exchange), timing is the max over ranks, and value is the
whole job's bytes / that time ("weak" scaling).

--impl reference times the CPU oracle (the plain +1/-1 integer definition)
on the host cores on the same workload and metric; rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "binary GMAC/s (TOPS) for packed XNOR-popcount GEMM; GEMV GB/s vs HBM peak"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# Dense int8 tensor throughput is twice dense bf16 (4.5 vs 2.25 PFLOP/s nominal);
# the int8 peak used here is the measured bf16 peak times that ratio.
INT8_PER_BF16 = 2.0
# Dense fp4 (e2m1) over dense bf16 tensor throughput, nominal (9 / 2.25 PFLOP/s).
FP4_PER_BF16 = 4.0
# Whether AUTO runs the stride-1 convolution on the tensor cores (mirrors the
# library's dispatch, for labelling the conv row's roofline).
CONV_AUTO_TENSOR = True
SM_COUNT = 148
# Nominal integer-pipe rates per SM clock (CUDA arithmetic-instruction
# throughput table): 32-bit population count 16, logic ops 64.  Used only when
# the library's probe (bnn_probe_int_pipes) cannot run; the bench measures them.
POPC_PER_CLK_PER_SM = 16
LOP3_PER_CLK_PER_SM = 64
# The carry-save popcount GEMM's instruction mix per XOR word: 8 XOR + 8 LOP3
# (four full adders) + 1 IADD3 on the ALU pipe and 4 POPC per 8 words.
CSA_ALU_PER_WORD = 17 / 8
CSA_POPC_PER_WORD = 4 / 8


# ---------------------------------------------------------------------------
# process setup
# ---------------------------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(torch, dist, v: float, device) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    if dist is None:
        return float(v)
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world_size: int, steps: int, units_per_step: float, ms_max: float) -> float:
    """Whole-job units/s: every rank processes `steps` steps of its own replica,
    timed as the slowest rank (weak scaling)."""
    return world_size * steps * units_per_step / (ms_max * 1e-3)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)),
                "bf16_tflops": float(d.get("bf16_tflops", FALLBACK_BF16_TFLOPS)),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", 1400.0)),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": 1965.0, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def int_pipe_peaks(bnn, sm_mhz: float, sms: int = SM_COUNT) -> dict:
    """Integer rooflines in binary MAC/s (one 32-bit word = 32 binary MACs).
    `popc_only`: every SM retiring POPC at its measured rate (one word each).
    `combined`: the carry-save GEMM's mix -- a word needs CSA_ALU_PER_WORD ALU
    ops and CSA_POPC_PER_WORD POPC, so the slower of the two pipes at their
    measured rates bounds the word rate.  `csa_probe`: the same step measured
    end to end on registers, for comparison."""
    try:
        r = bnn.bnn_probe_int_pipes(4096)
        src = "measured (bnn_probe_int_pipes)"
    except Exception as e:            # no device: the nominal table rates, labelled as such
        r = {"popc": float(POPC_PER_CLK_PER_SM), "lop3": float(LOP3_PER_CLK_PER_SM), "csa_words": None}
        src = f"nominal table rates ({type(e).__name__})"
    hz = sms * 32 * sm_mhz * 1e6
    words = min(r["lop3"] / CSA_ALU_PER_WORD, r["popc"] / CSA_POPC_PER_WORD)
    return {"popc_per_clk_sm": r["popc"], "lop3_per_clk_sm": r["lop3"], "csa_words_per_clk_sm": r["csa_words"],
            "popc_only": r["popc"] * hz, "combined": words * hz,
            "csa_probe": r["csa_words"] * hz if r["csa_words"] else None, "source": src, "sm_mhz": sm_mhz}


def alu_roofline(mac_s: float, ip: dict) -> dict:
    """The popcount engine against the integer pipes (binary TMAC/s)."""
    out = {"bound": "alu", "achieved": round(mac_s / 1e12, 2), "peak": round(ip["combined"] / 1e12, 2),
           "unit": "binary TMAC/s", "frac": round(mac_s / ip["combined"], 4),
           "peak_derivation": (f"{SM_COUNT} SMs x min(LOP3 {ip['lop3_per_clk_sm']:.1f}/clk / {CSA_ALU_PER_WORD}, "
                               f"POPC {ip['popc_per_clk_sm']:.2f}/clk / {CSA_POPC_PER_WORD}) words/clk x 32 MAC x "
                               f"{ip['sm_mhz']:.0f} MHz; rates {ip['source']}"),
           "popc_only_peak": round(ip["popc_only"] / 1e12, 2), "popc_only_frac": round(mac_s / ip["popc_only"], 4)}
    if ip["csa_probe"]:
        out["csa_probe_peak"] = round(ip["csa_probe"] / 1e12, 2)
    return out


# Source files that determine each kernel's code (its own header + shared helpers).
KERNEL_SOURCES = {
    "xnor_gemv_row128_kernel": ("gemv.cuh", "common.cuh"),
    "xnor_gemm_tc_kernel": ("gemm_tc.cuh", "gemm_popc.cuh", "common.cuh"),
    "xnor_gemm_f4_kernel": ("gemm_f4.cuh", "gemm_tc.cuh", "gemm_popc.cuh", "common.cuh"),
    "xnor_gemm_popc_kernel": ("gemm_popc.cuh", "common.cuh"),
    "xnor_conv3x3_kernel": ("conv.cuh", "common.cuh"),
    "xnor_conv3x3_tcw_kernel": ("conv_tc.cuh", "conv.cuh", "gemm_f4.cuh", "gemm_tc.cuh", "gemm_popc.cuh",
                                "common.cuh"),
    "pack_sign_rows_kernel": ("pack.cuh", "common.cuh"),
    "pack_sign_nchw_kernel": ("pack.cuh", "common.cuh"),
    "pack_sign_nchw_tma_kernel": ("pack.cuh", "common.cuh"),
    "bw_gemv_kernel": ("bwgemv.cuh", "common.cuh"),
    "bw_gemv_i8_kernel": ("bwgemv_i8.cuh", "common.cuh"),
    "ternary_gemv_i8_kernel": ("ternary.cuh", "common.cuh"),
    "xnor_conv1x1_kernel": ("conv1x1.cuh", "conv.cuh", "gemm_popc.cuh", "common.cuh"),
    "pack_ternary_kernel": ("ternary.cuh", "common.cuh"),
    "pack_bit_planes_kernel": ("pack.cuh", "common.cuh"),
    "xnor_gemv_chain_kernel": ("chain.cuh", "common.cuh"),
}


def source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel.split("<")[0]]:
        h.update(open(os.path.join(ROOT, "xnor_popcount_gemm_bnn_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(row: str, kernel: str):
    """DRAM bytes per launch (read + write) of `kernel` on the workload of bench
    row `row`, from the committed ncu summary of that row's capture, if it was
    taken on the kernel's current sources; else None.  Entries are keyed by
    row, so a capture of one workload is never reported for another."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(f"{row}/{kernel}")
    if not e or e.get("source_hash") != source_hash(kernel):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """SM clock and throttle reasons, sampled with NVML during the timed region."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                r = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# device timing helpers
# ---------------------------------------------------------------------------

def _graph(torch, fn, n):
    """Capture n calls of fn(i) into one CUDA graph (launch-bound inner loop)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn(0)                                    # warm the stream and library once
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            fn(i)
    return g


# Largest number of timed steps captured in one graph.
MAX_GRAPH_STEPS = 960


def time_steps(torch, fn, steps, warmup, period, sync):
    """Run at least `warmup` untimed steps, then time exactly `steps` steps
    with CUDA events on the device.  fn(i) launches step i.

    The steps run from CUDA graphs.  The first graph holds `lead` untimed
    steps (max(period, warmup)), then the start event, then the first timed
    steps; further graphs hold up to MAX_GRAPH_STEPS timed steps each (a
    multiple of `period`, the rotation of the inputs), and the last one ends
    with the end event.  The events are graph nodes (external events): the
    start event sits on a forked branch that waits for the last lead step, so
    the first timed step keeps its place in the launch chain (a kernel that
    may start before its predecessor ends still does), and the timed window
    runs from the completion of the last lead step to the completion of the
    last timed step.  Every graph is replayed once before the host
    synchronize and the barrier, so no first-replay upload is timed; then the
    graphs are replayed back to back and the events read after a synchronize.
    Returns milliseconds for the timed steps."""
    lead = max(period, warmup)
    chunk = max(period, MAX_GRAPH_STEPS // period * period)
    sizes = []
    left = steps
    while left > 0:
        sizes.append(min(chunk, left))
        left -= sizes[-1]
    start = torch.cuda.Event(enable_timing=True, external=True)
    end = torch.cuda.Event(enable_timing=True, external=True)

    # warm the stream and the library once, outside any graph
    s0 = torch.cuda.Stream()
    s0.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s0):
        fn(0)
    torch.cuda.current_stream().wait_stream(s0)

    side = torch.cuda.Stream()                 # the start event's branch, created outside capture
    graphs = []
    i = 0
    for gi, n in enumerate(sizes):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            main = torch.cuda.current_stream()
            if gi == 0:
                for _ in range(lead):
                    fn(i)
                    i += 1
                side.wait_stream(main)
                with torch.cuda.stream(side):
                    start.record()
            for _ in range(n):
                fn(i)
                i += 1
            if gi == len(sizes) - 1:
                end.record()
            if gi == 0:
                main.wait_stream(side)
        graphs.append(g)
    for g in graphs:                           # warm-up: lead + every timed step once, every graph uploaded
        g.replay()
    torch.cuda.synchronize()
    sync()
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    sync()
    return ms


# ---------------------------------------------------------------------------
# the headline: LLM-decode binary GEMV
# ---------------------------------------------------------------------------

GEMV_N, GEMV_K = 11008, 4096


def gemv_bytes(N=GEMV_N, K=GEMV_K) -> int:
    kw = ((K + 31) // 32 + 3) // 4 * 4
    return N * kw * 4 + N * 4 + K * 2 + N * 4     # packed W + alpha + bf16 x + fp32 y


def gemv_setup(torch, bnn, workloads, dev, copies):
    g = workloads.gemv()
    W_p = bnn.empty_packed(g.N, g.K, dev)
    alpha = torch.empty(g.N, dtype=torch.float32, device=dev)
    bnn.bnn_pack_sign(g.W.to(dev), W_p, alpha)
    Ws = [W_p] + [W_p.clone() for _ in range(copies - 1)]
    x = g.x.to(dev)
    y = torch.empty(g.N, dtype=torch.float32, device=dev)
    return g, Ws, alpha, x, y


def run_ours(args, torch, dist):
    import workloads
    import xnor_popcount_gemm_bnn_b200 as bnn

    ws, rank, local = dist_env()
    dev = torch.device("cuda", local)
    pk = peaks()

    def sync():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(v):
        return reduce_max(torch, dist, v, dev)

    copies = max(2, math.ceil(2 * L2_BYTES / gemv_bytes()) + 1)
    copies = (copies + 7) // 8 * 8                       # 48
    g, Ws, alpha, x, y = gemv_setup(torch, bnn, workloads, dev, copies)

    # Every step's inputs (packed W, x, alpha) are resident before the timed
    # region, and each step writes its own output (the y buffers rotate with
    # the weights), so no step depends on another: each GEMV streams its
    # weights, packs x, forms the product and stores y while the previous one
    # may still run, and waits for it only before exiting.
    ys = [torch.empty(g.N, dtype=torch.float32, device=dev) for _ in range(copies)]
    all_flags = bnn.BNN_GEMV_WEIGHTS_STATIC | bnn.BNN_GEMV_INPUTS_STATIC | bnn.BNN_GEMV_OUTPUT_FREE

    def step(i):
        bnn.bnn_xnor_gemv_ex(Ws[i % copies], x, g.K, alpha, None, ys[i % copies], flags=all_flags)

    # The same steps with one shared y: the store waits for the previous kernel.
    def step_ordered(i):
        bnn.bnn_xnor_gemv_ex(Ws[i % copies], x, g.K, alpha, None, y,
                             flags=bnn.BNN_GEMV_WEIGHTS_STATIC | bnn.BNN_GEMV_INPUTS_STATIC)

    # A decode chain where x is the previous kernel's output: only the weight
    # stream may start before the previous kernel has finished.
    def step_dep(i):
        bnn.bnn_xnor_gemv_ex(Ws[i % copies], x, g.K, alpha, None, y, flags=bnn.BNN_GEMV_WEIGHTS_STATIC)

    def step_plain(i):
        bnn.bnn_xnor_gemv(Ws[i % copies], x, g.K, alpha, None, y)

    with ClockSampler(local) as clk:
        ms = time_steps(torch, step, args.steps, args.warmup, copies, sync)
    ms = max_over_ranks(ms)
    side_steps = min(args.steps, 48 * copies)
    ms_ord = max_over_ranks(time_steps(torch, step_ordered, side_steps, args.warmup, copies, sync))
    ms_dep = max_over_ranks(time_steps(torch, step_dep, side_steps, args.warmup, copies, sync))
    ms_plain = max_over_ranks(time_steps(torch, step_plain, side_steps, args.warmup, copies, sync))
    if bnn.bnn_device_error() != 0:
        raise RuntimeError("a kernel reported a device-side timeout")
    per_step_bytes = gemv_bytes()
    value = job_throughput(ws, args.steps, per_step_bytes, ms) / 1e9
    launch_s = ms * 1e-3 / args.steps
    achieved = per_step_bytes / launch_s / 1e9

    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u32",
        "data": "synthetic",
        "config": {
            "workload": "LLM-decode binary GEMV: packed +1/-1 W [11008, 4096] from N(0,0.02), "
                        "x bf16 [4096] N(0,1) sign-packed in-kernel, per-row alpha, fp32 y",
            "N": g.N, "K": g.K,
            "algorithmic_bytes_per_step": per_step_bytes,
            "l2": f"inputs larger than L2: {copies} rotating packed weight copies "
                  f"({copies * Ws[0].numel() * 4 / 1e6:.0f} MB > 126 MB L2)",
            "timing": f"CUDA graphs (first: {max(copies, args.warmup)} untimed lead steps, then the timed steps, up to "
                      f"{MAX_GRAPH_STEPS} per graph); start and end are CUDA events captured as graph nodes",
            "parallelism": "replicas" if ws == 1 else f"replicas x{ws}",
        },
        "roofline": {
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": pk["hbm_gbs"],
            "unit": "GB/s",
            "frac": round(achieved / pk["hbm_gbs"], 4),
            "traffic": recorded_traffic("gemv", "xnor_gemv_row128_kernel"),
            "peak_source": pk["source"],
            "kernel": "xnor_gemv_row128_kernel",
        },
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
        "flags": "BNN_GEMV_WEIGHTS_STATIC | BNN_GEMV_INPUTS_STATIC | BNN_GEMV_OUTPUT_FREE "
                 "(independent steps: resident inputs, one output buffer per step)",
        "store_ordered": {
            "value": round(ws * side_steps * per_step_bytes / (ms_ord * 1e-3) / 1e9, 2), "unit": "GB/s",
            "steps": side_steps, "ms_per_step": ms_ord / side_steps,
            "frac": round(side_steps * per_step_bytes / (ms_ord * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
            "note": "BNN_GEMV_WEIGHTS_STATIC | BNN_GEMV_INPUTS_STATIC with one shared y: each store waits for "
                    "the previous kernel"},
        "dependent_chain": {
            "value": round(ws * side_steps * per_step_bytes / (ms_dep * 1e-3) / 1e9, 2), "unit": "GB/s",
            "steps": side_steps, "ms_per_step": ms_dep / side_steps,
            "frac": round(side_steps * per_step_bytes / (ms_dep * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
            "note": "BNN_GEMV_WEIGHTS_STATIC only: W and alpha are read before, x after the wait for the "
                    "previous kernel, as when x is the previous layer's output"},
        "gemv_default_flags": {
            "value": round(ws * side_steps * per_step_bytes / (ms_plain * 1e-3) / 1e9, 2), "unit": "GB/s",
            "steps": side_steps, "ms_per_step": ms_plain / side_steps,
            "note": "bnn_xnor_gemv (no flags): W, x and alpha are read after the wait for the previous kernel"},
    }

    # e2e: the public API with host buffers
    if not args.no_e2e:
        # Host-driven steps: at least 200, so that the first call's host
        # latency after the start event is a small part of the window.
        result["e2e"] = e2e_gemv(torch, bnn, g, Ws, alpha, dev, min(max(args.steps, 200), 2000), sync,
                                 max_over_ranks, ws)

    if not args.no_rows:
        result["rows"] = bench_rows(torch, bnn, workloads, dev, pk, args, sync, max_over_ranks, ws)

    del Ws
    torch.cuda.empty_cache()
    if rank == 0 and not args.no_cpu_baseline and ws == 1:
        result["cpu_baseline"] = cpu_baseline_gemv(args.cpu_seconds)
        if "rows" in result:
            cpu_baseline_rows(result["rows"], args.cpu_row_seconds)
    return result


def run_only_rows(args, torch, dist):
    import workloads
    import xnor_popcount_gemm_bnn_b200 as bnn
    ws, rank, local = dist_env()
    dev = torch.device("cuda", local)

    def sync():
        if dist is not None:
            dist.barrier()

    names = [n for n in args.only_rows.split(",") if n]
    if args.square_shape:
        _row_square.shape = tuple(int(v) for v in args.square_shape.split(","))
    for n in names:
        if n not in ROW_NAMES:
            raise SystemExit(f"unknown row {n!r}; choose from {ROW_NAMES}")
    return {"rows": bench_rows(torch, bnn, workloads, dev, peaks(), args, sync, lambda v: v, ws, names)}


def e2e_gemv(torch, bnn, g, Ws, alpha, dev, steps, sync, max_over_ranks, ws):
    """The headline metric end to end through the C ABI with host buffers:
    every step is one bnn_xnor_gemv_host call, which takes that step's x from
    pinned host memory, runs the GEMV and puts y back into pinned host memory
    on the stream (pinned buffers: two small copy kernels across PCIe chained
    to the GEMV).  The steps call the C entry point with its arguments
    marshalled once per weight copy, so the timed loop pays the library's
    host work, not the Python binding's per-call conversions.  (The same
    steps as three eager torch calls -- two copy_ and bnn_xnor_gemv_ex --
    took about 22 us each.)"""
    import ctypes
    x_host = g.x.clone().pin_memory()
    y_host = torch.empty(g.N, dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(g.x, device=dev)
    y_dev = torch.empty(g.N, dtype=torch.float32, device=dev)
    copies = len(Ws)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    call = bnn._lib.bnn_xnor_gemv_host
    args = [(ctypes.c_void_p(W.data_ptr()), W.stride(0), ctypes.c_void_p(x_host.data_ptr()), bnn.BNN_BF16, g.N, g.K,
             ctypes.c_void_p(alpha.data_ptr()), ctypes.c_void_p(x_dev.data_ptr()), ctypes.c_void_p(y_dev.data_ptr()),
             ctypes.c_void_p(y_host.data_ptr()), bnn.BNN_GEMV_WEIGHTS_STATIC | bnn.BNN_GEMV_INPUTS_STATIC, stream)
            for W in Ws]
    assert g.x.dtype == torch.bfloat16

    def one(i):
        # x comes from the host buffer, which no device work writes (INPUTS_STATIC
        # lets the copy-in read it early); the GEMV's x is written by that copy.
        st = call(*args[i % copies])
        if st != bnn.BNN_OK:
            raise bnn.BnnError("bnn_xnor_gemv_host", st, bnn._lib.bnn_status_string(st).decode())

    # Host-driven steps: warm the call path well past first-use costs, so a
    # short timed window measures the steady per-step cost.
    for i in range(50):
        one(i)
    torch.cuda.synchronize()
    sync()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        one(i)
    end.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(end))
    return {"value": round(ws * steps * gemv_bytes() / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
            "d2h_bytes_per_step": y_host.numel() * y_host.element_size(),
            "steps": steps, "ms_per_step": ms / steps,
            "path": "one C-ABI bnn_xnor_gemv_host call per step: x read from pinned host memory, GEMV, y written "
                    "to pinned host memory (copy kernels across PCIe, chained to the GEMV by programmatic dependent launch)"}


# ---------------------------------------------------------------------------
# the other rows
# ---------------------------------------------------------------------------

ROW_NAMES = ("pack_sign_weights", "square_gemm", "conv3x3", "mlp4", "bw_gemv", "ternary", "conv1x1", "multibit",
             "decode_chain")


def bench_rows(torch, bnn, workloads, dev, pk, args, sync, max_over_ranks, ws, only=None):
    rows = {}
    want = set(only or ROW_NAMES)
    steps = max(3, args.row_steps)
    warm = max(3, args.warmup)
    clk_mhz = pk["sm_max_mhz"]
    alu_peak = int_pipe_peaks(bnn, clk_mhz) if want & {"square_gemm", "conv3x3", "mlp4"} else None
    if alu_peak is not None:
        rows["int_pipes"] = {k: (round(v, 3) if isinstance(v, float) else v) for k, v in alu_peak.items()}

    def timed(fn, n=steps, period=None):
        return max_over_ranks(time_steps(torch, fn, n, warm, period or n, sync))

    plan = (
        # a1: weight pack + alpha, fp32 [11008, 4096] (HBM)
        ("pack_sign_weights", lambda: _row_pack(torch, bnn, workloads, dev, pk, rows, timed, steps, ws)),
        ("square_gemm", lambda: _row_square(torch, bnn, workloads, dev, rows, timed, steps, ws, alu_peak, clk_mhz,
                                            pk)),
        ("conv3x3", lambda: _row_conv(torch, bnn, workloads, dev, rows, timed, steps, ws, alu_peak, pk)),
        ("mlp4", lambda: _row_mlp(torch, bnn, workloads, dev, rows, timed, steps, ws, alu_peak, pk)),
        ("bw_gemv", lambda: _row_bw_gemv(torch, bnn, workloads, dev, pk, rows, timed, ws, steps)),
        ("ternary", lambda: _row_ternary(torch, bnn, workloads, dev, pk, rows, timed, steps, ws)),
        ("conv1x1", lambda: _row_conv1x1(torch, bnn, workloads, dev, pk, rows, timed, steps, ws, alu_peak)),
        ("multibit", lambda: _row_multibit(torch, bnn, workloads, dev, pk, rows, timed, steps, ws)),
        ("decode_chain", lambda: _row_chain(torch, bnn, workloads, dev, pk, rows, timed, steps, ws)),
    )
    for name, run in plan:
        if name not in want:
            continue
        try:
            run()
        except Exception as e:      # a failing row is reported in the line; the others and the headline stand
            rows[name] = {"error": f"{type(e).__name__}: {e}"[:400]}
            torch.cuda.empty_cache()
    code = bnn.bnn_device_error()
    if code != 0:
        rows["device_error"] = {"code": int(code), "note": "a kernel gave up waiting (device-side timeout)"}
    return rows


def _row_pack(torch, bnn, workloads, dev, pk, rows, timed, steps, ws):
    g = workloads.gemv()
    Wd = g.W.to(dev)
    W_p = bnn.empty_packed(g.N, g.K, dev)
    alpha = torch.empty(g.N, dtype=torch.float32, device=dev)
    ms = timed(lambda i: bnn.bnn_pack_sign(Wd, W_p, alpha))
    b = g.N * g.K * 4 + W_p.numel() * 4 + g.N * 4
    ach = b * steps / (ms * 1e-3) / 1e9
    rows["pack_sign_weights"] = {"workload": "fp32 W [11008, 4096] -> packed bits + alpha",
                                 "value": round(ws * ach, 1), "unit": "GB/s", "ms_per_step": ms / steps,
                                 "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"],
                                              "frac": round(ach / pk["hbm_gbs"], 4),
                                              "traffic": recorded_traffic("pack_sign_weights", "pack_sign_rows_kernel")}}
    del Wd, W_p, alpha, g
    torch.cuda.empty_cache()


def _tensor_roofline(pk, macs_per_s, sustained, row=None, operand="int8", kernel="xnor_gemm_tc_kernel<TC_BINARY>"):
    """A tensor-core engine against the dense peak of its operand type (one
    binary MAC is one MAC there): measured bf16 dense TFLOP/s x 2 for int8
    operands, x 4 for e2m1 (fp4) operands, in TOPS of that type."""
    bf16 = pk["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    ratio = FP4_PER_BF16 if operand == "e2m1" else INT8_PER_BF16
    peak_tops = bf16 * ratio
    achieved = 2 * macs_per_s / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak_tops, 1),
            "unit": f"TOPS ({operand})", "frac": round(achieved / peak_tops, 4),
            "peak_derivation": f"measured bf16 {'sustained' if sustained else 'burst'} {bf16} TFLOP/s x {ratio} "
                               f"(dense {operand} / bf16, nominal)",
            "traffic": recorded_traffic(row, kernel) if row else None}


def _row_square(torch, bnn, workloads, dev, rows, timed, steps, ws, alu_peak, clk_mhz, pk=None):
    # --- a2+a3+a6: square GEMM 8192^3, int32 + alpha-scaled fp32 outputs, both engines ---
    shape = getattr(_row_square, "shape", None)
    sq = workloads.square(*shape) if shape else workloads.square()
    Ad = sq.A.to(dev)
    A_p = bnn.empty_packed(sq.M, sq.K, dev)
    Wsq = bnn.empty_packed(sq.N, sq.K, dev)
    al = torch.empty(sq.N, dtype=torch.float32, device=dev)
    bnn.bnn_pack_sign(sq.W.to(dev), Wsq, al)
    bnn.bnn_pack_sign(Ad, A_p)
    Ci = torch.empty(sq.M, sq.N, dtype=torch.int32, device=dev)
    Cf = torch.empty(sq.M, sq.N, dtype=torch.float32, device=dev)
    macs = sq.M * sq.N * sq.K
    engines = (("square_gemm", bnn.BNN_GEMM_ENGINE_TENSOR), ("square_gemm_i8", bnn.BNN_GEMM_ENGINE_TENSOR_I8),
               ("square_gemm_popcount", bnn.BNN_GEMM_ENGINE_POPCOUNT))
    for name, engine in engines:
        with bnn.gemm_engine(engine):
            ms_g = timed(lambda i: bnn.bnn_xnor_gemm(A_p, Wsq, sq.K, al, Ci, Cf))
            ms_s = timed(lambda i: (bnn.bnn_pack_sign(Ad, A_p), bnn.bnn_xnor_gemm(A_p, Wsq, sq.K, al, Ci, Cf)))
        mac_s = macs * steps / (ms_g * 1e-3)
        if engine == bnn.BNN_GEMM_ENGINE_TENSOR:
            kernel = "xnor_gemm_f4_kernel"
            roof = _tensor_roofline(pk, mac_s, sustained=False, row=name, operand="e2m1", kernel=kernel)
            label = "tensor (tcgen05 kind::mxf4, e2m1 +1/-1, unit scales)"
        elif engine == bnn.BNN_GEMM_ENGINE_TENSOR_I8:
            kernel = "xnor_gemm_tc_kernel"
            roof = _tensor_roofline(pk, mac_s, sustained=False, row="square_gemm")
            label = "tensor (tcgen05 kind::i8)"
        else:
            roof = alu_roofline(mac_s, alu_peak)
            roof["traffic"] = recorded_traffic("square_gemm_popcount", "xnor_gemm_popc_kernel")
            kernel = "xnor_gemm_popc_kernel"
            label = "popcount (XOR + POPC, carry-save)"
        rows[name] = {
            "workload": f"M={sq.M} N={sq.N} K={sq.K} packed A x packed W^T, int32 s + alpha*s fp32 out",
            "engine": label,
            "kernel": kernel,
            "value": round(ws * mac_s / 1e9, 1), "unit": "binary GMAC/s", "tops": round(ws * 2 * mac_s / 1e12, 2),
            "ms_per_step": ms_g / steps,
            "with_activation_pack": {"value": round(ws * macs * steps / (ms_s * 1e-3) / 1e9, 1),
                                     "unit": "binary GMAC/s", "ms_per_step": ms_s / steps},
            "roofline": roof}
    del sq, Ad, A_p, Wsq, al, Ci, Cf
    torch.cuda.empty_cache()


def _row_conv(torch, bnn, workloads, dev, rows, timed, steps, ws, alu_peak, pk):
    # --- a2 (NCHW) + a5 + a6: ResNet-class binary 3x3 conv with affine epilogue ---
    cv = workloads.conv()
    n, c, h, w = cv.X.shape
    # Three rotating sets of (bf16 input, packed input, fp32 output), 235 MB
    # in all, so that consecutive steps do not find their data in the 126 MB L2.
    R = 3
    Xd = [cv.X.to(dev) for _ in range(R)]
    Xb = [bnn.empty_packed_nhwc(n, c, h, w, dev) for _ in range(R)]
    out = [torch.empty(n, 64, h, w, dtype=torch.float32, device=dev) for _ in range(R)]
    Wc = bnn.empty_conv3x3_weights(64, c, dev)
    alc = torch.empty(64, dtype=torch.float32, device=dev)
    bnn.bnn_pack_conv3x3_weights(cv.W.to(dev), Wc, alc)
    gam, bet = cv.gamma.to(dev), cv.beta.to(dev)
    ep = bnn.make_epilogue(bnn.BNN_OUT_AFFINE_F32, alpha=alc, gamma=gam, beta=bet)
    rot_mb = R * (Xd[0].numel() * 2 + Xb[0].numel() * 4 + out[0].numel() * 4) / 1e6

    def conv_step(i):
        bnn.bnn_pack_sign_nchw(Xd[i % R], Xb[i % R])
        bnn.bnn_binary_conv3x3_fused(Xb[i % R], c, Wc, ep, out[i % R], 1, 1)

    cmacs = n * h * w * 64 * 9 * c
    # Algorithmic bytes of one conv launch: packed activations and filters in,
    # fp32 NCHW out (alpha/gamma/beta are 768 B).
    cbytes = Xb[0].numel() * 4 + Wc.numel() * 4 + out[0].numel() * 4
    for i in range(R):
        bnn.bnn_pack_sign_nchw(Xd[i], Xb[i])
    ms_pack = timed(lambda i: bnn.bnn_pack_sign_nchw(Xd[i % R], Xb[i % R]))
    pbytes = Xd[0].numel() * 2 + Xb[0].numel() * 4
    pack_gbs = pbytes * steps / (ms_pack * 1e-3) / 1e9
    rbeta = torch.linspace(-0.5, 0.5, c, device=dev)       # a per-channel threshold (RSign)
    ms_rs = timed(lambda i: bnn.bnn_pack_sign_nchw_rsign(Xd[i % R], rbeta, Xb[i % R]))
    rs_gbs = (pbytes + c * 4) * steps / (ms_rs * 1e-3) / 1e9
    for name, engine in (("conv3x3", bnn.BNN_GEMM_ENGINE_AUTO), ("conv3x3_tensor", bnn.BNN_GEMM_ENGINE_TENSOR),
                         ("conv3x3_popcount", bnn.BNN_GEMM_ENGINE_POPCOUNT)):
        with bnn.gemm_engine(engine):
            ms_c = timed(conv_step)
            ms_ck = timed(lambda i: bnn.bnn_binary_conv3x3_fused(Xb[i % R], c, Wc, ep, out[i % R], 1, 1))
        cmac_s = cmacs * steps / (ms_ck * 1e-3)
        tensor = engine == bnn.BNN_GEMM_ENGINE_TENSOR or (engine == bnn.BNN_GEMM_ENGINE_AUTO and CONV_AUTO_TENSOR)
        if tensor:
            # The fp32 output write bounds this kernel: 51 MB out against 7.4 G
            # binary MACs, 8 us of HBM time versus under 5 us of int8 tensor time.
            ach = cbytes * steps / (ms_ck * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": round(ach / pk["hbm_gbs"], 4), "algorithmic_bytes": cbytes,
                    "tensor": _tensor_roofline(pk, cmac_s, sustained=False),
                    "traffic": recorded_traffic("conv3x3", "xnor_conv3x3_tcw_kernel")}
            roof["tensor"].pop("traffic")
        else:
            roof = alu_roofline(cmac_s, alu_peak)
            roof["traffic"] = recorded_traffic(name, "xnor_conv3x3_kernel")
        rows[name] = {
            "workload": "bf16 [64,64,56,56] -> pack NCHW -> binary 3x3 conv (64 filters, stride 1, pad 1), "
                        "alpha + affine epilogue, fp32 NCHW out",
            "engine": {bnn.BNN_GEMM_ENGINE_AUTO: "auto", bnn.BNN_GEMM_ENGINE_TENSOR: "tensor",
                       bnn.BNN_GEMM_ENGINE_POPCOUNT: "popcount"}[engine] + (" (tensor cores)" if tensor else " (popcount)"),
            "value": round(ws * cmacs * steps / (ms_c * 1e-3) / 1e9, 1), "unit": "binary GMAC/s",
            "ms_per_step": ms_c / steps, "conv_kernel_ms": ms_ck / steps,
            "conv_kernel_binary_tmac_s": round(cmac_s / 1e12, 2), "roofline": roof,
            "pack_nchw": {"ms": ms_pack / steps, "achieved_gbs": round(pack_gbs, 1),
                          "frac": round(pack_gbs / pk["hbm_gbs"], 4), "bytes": pbytes,
                          "traffic": recorded_traffic("conv3x3", "pack_sign_nchw_tma_kernel"),
                          "kernel": "pack_sign_nchw_tma_kernel"},
            "pack_nchw_rsign": {"ms": ms_rs / steps, "achieved_gbs": round(rs_gbs, 1),
                                "frac": round(rs_gbs / pk["hbm_gbs"], 4), "bytes": pbytes + c * 4},
            "l2": f"{R} rotating input/output sets, {rot_mb:.0f} MB"}
    del cv, Xd, Xb, Wc, alc, gam, bet, out
    torch.cuda.empty_cache()


def _row_bw_gemv(torch, bnn, workloads, dev, pk, rows, timed, ws, row_steps):
    # --- next row: binary weights x real (bf16) activations, the decode shape ---
    g = workloads.gemv()
    copies = max(2, math.ceil(2 * L2_BYTES / gemv_bytes()) + 1)
    copies = (copies + 7) // 8 * 8
    W_p = bnn.empty_packed(g.N, g.K, dev)
    alpha = torch.empty(g.N, dtype=torch.float32, device=dev)
    bnn.bnn_pack_sign(g.W.to(dev), W_p, alpha)
    Ws = [W_p] + [W_p.clone() for _ in range(copies - 1)]
    ys = [torch.empty(g.N, dtype=torch.float32, device=dev) for _ in range(copies)]
    x = g.x.to(dev)
    steps = max(row_steps, 20) * copies            # 960 steps by default: each copy streamed 20 times
    all_flags = bnn.BNN_GEMV_WEIGHTS_STATIC | bnn.BNN_GEMV_INPUTS_STATIC | bnn.BNN_GEMV_OUTPUT_FREE
    ms = timed(lambda i: bnn.bnn_binary_weight_gemv(Ws[i % copies], x, g.K, alpha, ys[i % copies], flags=all_flags),
               n=steps, period=copies)
    ms_dep = timed(lambda i: bnn.bnn_binary_weight_gemv(Ws[i % copies], x, g.K, alpha, ys[0],
                                                        flags=bnn.BNN_GEMV_WEIGHTS_STATIC), n=steps, period=copies)
    b = gemv_bytes()
    ach = b * steps / (ms * 1e-3) / 1e9
    ach_dep = b * steps / (ms_dep * 1e-3) / 1e9
    rows["bw_gemv"] = {
        "workload": "binary weights x real activations (eq. (1)): packed W [11008, 4096], x bf16 [4096] "
                    "not binarised, alpha-scaled fp32 y; independent steps over 48 rotating weight copies",
        "value": round(ws * ach, 1), "unit": "GB/s", "ms_per_step": ms / steps,
        "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"],
                     "frac": round(ach / pk["hbm_gbs"], 4), "algorithmic_bytes": b,
                     "traffic": recorded_traffic("bw_gemv", "bw_gemv_kernel")},
        "dependent_chain": {"value": round(ws * ach_dep, 1), "unit": "GB/s", "ms_per_step": ms_dep / steps,
                            "frac": round(ach_dep / pk["hbm_gbs"], 4)}}
    # the same weights x INT8 activations (x of the ternary workload, scale 1/64)
    t = workloads.ternary()
    xq = t.x.to(dev)
    xsc = torch.full((1,), 1.0 / 64, dtype=torch.float32, device=dev)
    ms8 = timed(lambda i: bnn.bnn_binary_weight_gemv_i8(Ws[i % copies], xq, g.K, alpha, xsc, None, ys[i % copies],
                                                        flags=all_flags), n=steps, period=copies)
    ms8_dep = timed(lambda i: bnn.bnn_binary_weight_gemv_i8(Ws[i % copies], xq, g.K, alpha, xsc, None, ys[0],
                                                            flags=bnn.BNN_GEMV_WEIGHTS_STATIC), n=steps, period=copies)
    b8 = Ws[0].numel() * 4 + 4 * g.N + g.K + 4 * g.N + 4        # packed W + alpha + int8 x + fp32 y + x scale
    a8 = b8 * steps / (ms8 * 1e-3) / 1e9
    a8_dep = b8 * steps / (ms8_dep * 1e-3) / 1e9
    rows["bw_gemv_i8"] = {
        "workload": "binary weights x INT8 activations: packed W [11008, 4096], x int8 [4096] with its scale, "
                    "exact int32 sum of +-x, alpha * x_scale fp32 y; independent steps over 48 rotating weight copies",
        "value": round(ws * a8, 1), "unit": "GB/s", "ms_per_step": ms8 / steps,
        "roofline": {"bound": "hbm", "achieved": round(a8, 1), "peak": pk["hbm_gbs"],
                     "frac": round(a8 / pk["hbm_gbs"], 4), "algorithmic_bytes": b8,
                     "traffic": recorded_traffic("bw_gemv_i8", "bw_gemv_i8_kernel")},
        "dependent_chain": {"value": round(ws * a8_dep, 1), "unit": "GB/s", "ms_per_step": ms8_dep / steps,
                            "frac": round(a8_dep / pk["hbm_gbs"], 4)}}
    del Ws, ys, W_p, x, g, xq, t
    torch.cuda.empty_cache()



def _row_ternary(torch, bnn, workloads, dev, pk, rows, timed, steps, ws):
    # --- next row: ternary (b1.58) weights: eq. (9) quantise + pack, then the int8 GEMV ---
    g = workloads.ternary()
    Wd = g.W.to(dev)
    codes = bnn.empty_ternary(g.N, g.K, dev)
    gam = torch.empty(1, dtype=torch.float32, device=dev)
    wsp = torch.empty(bnn.bnn_ternary_workspace_bytes(g.N) // 8, dtype=torch.float64, device=dev)
    ms_p = timed(lambda i: bnn.bnn_ternary_pack(Wd, codes, gamma_out=gam, workspace=wsp))
    q_bytes = codes.numel() * 4
    pb = 2 * g.N * g.K * 4 + q_bytes          # W read twice (gamma first, then the codes) + codes
    ach_p = pb * steps / (ms_p * 1e-3) / 1e9
    del Wd
    torch.cuda.empty_cache()
    copies = max(2, math.ceil(2 * L2_BYTES / q_bytes) + 1)
    copies = (copies + 7) // 8 * 8
    Qs = [codes] + [codes.clone() for _ in range(copies - 1)]
    ys = [torch.empty(g.N, dtype=torch.float32, device=dev) for _ in range(copies)]
    x = g.x.to(dev)
    xsc = torch.full((1,), 1.0 / 64, dtype=torch.float32, device=dev)
    n = max(steps, 20) * copies
    all_flags = bnn.BNN_GEMV_WEIGHTS_STATIC | bnn.BNN_GEMV_INPUTS_STATIC | bnn.BNN_GEMV_OUTPUT_FREE
    ms = timed(lambda i: bnn.bnn_ternary_gemv_i8(Qs[i % copies], x, g.K, y_f32=ys[i % copies], w_scale=gam,
                                                 x_scale=xsc, flags=all_flags), n=n, period=copies)
    ms_dep = timed(lambda i: bnn.bnn_ternary_gemv_i8(Qs[i % copies], x, g.K, y_f32=ys[0], w_scale=gam, x_scale=xsc,
                                                     flags=bnn.BNN_GEMV_WEIGHTS_STATIC), n=n, period=copies)
    b = q_bytes + g.K + 4 * g.N + 8           # codes + int8 x + fp32 y + two scales
    ach = b * n / (ms * 1e-3) / 1e9
    ach_dep = b * n / (ms_dep * 1e-3) / 1e9
    rows["ternary_gemv"] = {
        "workload": f"ternary (b1.58) weights x int8 activations: codes [11008, 4096] at 2 bits, x int8 [4096], "
                    f"fp32 y = gamma * x_scale * acc; independent steps over {copies} rotating code copies",
        "value": round(ws * ach, 1), "unit": "GB/s", "ms_per_step": ms / n,
        "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"],
                     "frac": round(ach / pk["hbm_gbs"], 4), "algorithmic_bytes": b,
                     "traffic": recorded_traffic("ternary_gemv", "ternary_gemv_i8_kernel")},
        "dependent_chain": {"value": round(ws * ach_dep, 1), "unit": "GB/s", "ms_per_step": ms_dep / n,
                            "frac": round(ach_dep / pk["hbm_gbs"], 4)}}
    rows["ternary_pack"] = {
        "workload": "fp32 W [11008, 4096] -> eq. (9) gamma (fp64 row sums, fixed-order total) + 2-bit codes; "
                    "3 launches",
        "value": round(ws * ach_p, 1), "unit": "GB/s", "ms_per_step": ms_p / steps,
        "roofline": {"bound": "hbm", "achieved": round(ach_p, 1), "peak": pk["hbm_gbs"],
                     "frac": round(ach_p / pk["hbm_gbs"], 4), "algorithmic_bytes": pb,
                     "traffic": recorded_traffic("ternary_pack", "pack_ternary_kernel")}}
    del Qs, ys, codes, x, g, wsp
    torch.cuda.empty_cache()



def _row_conv1x1(torch, bnn, workloads, dev, pk, rows, timed, steps, ws, alu_peak):
    # --- next row: binary 1x1 stride-2 downsampling projection (ResNet block) ---
    cv = workloads.downsample()
    n, c, h, w = cv.X.shape
    cout = cv.W.shape[0]
    oh, ow = (h - 1) // 2 + 1, (w - 1) // 2 + 1
    # Four rotating (packed input, fp32 output) sets, 109 MB, larger than L2 together.
    R = 4
    Xd = cv.X.to(dev)
    Xb = [bnn.empty_packed_nhwc(n, c, h, w, dev) for _ in range(R)]
    for i in range(R):
        bnn.bnn_pack_sign_nchw(Xd, Xb[i])
    Wp = bnn.empty_packed(cout, c, dev)
    al = torch.empty(cout, dtype=torch.float32, device=dev)
    bnn.bnn_pack_sign(cv.W.reshape(cout, c).to(dev), Wp, al)
    gam, bet = cv.gamma.to(dev), cv.beta.to(dev)
    ep = bnn.make_epilogue(bnn.BNN_OUT_AFFINE_F32, alpha=al, gamma=gam, beta=bet)
    out = [torch.empty(n, cout, oh, ow, dtype=torch.float32, device=dev) for _ in range(R)]
    ms = timed(lambda i: bnn.bnn_binary_conv1x1_fused(Xb[i % R], c, Wp, ep, out[i % R], stride=2))
    cw = (c + 31) // 32
    # Algorithmic bytes: the strided input pixels, the filters and the fp32 output.
    b = n * oh * ow * cw * 4 + Wp.numel() * 4 + out[0].numel() * 4
    ach = b * steps / (ms * 1e-3) / 1e9
    macs = n * oh * ow * cout * c
    rows["conv1x1"] = {
        "workload": "binary 1x1 stride-2 projection: packed [64,56,56,2 words] x 128 filters -> "
                    "alpha + affine fp32 NCHW [64,128,28,28]",
        "value": round(ws * ach, 1), "unit": "GB/s", "ms_per_step": ms / steps,
        "binary_tmac_s": round(macs * steps / (ms * 1e-3) / 1e12, 2),
        "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"],
                     "frac": round(ach / pk["hbm_gbs"], 4), "algorithmic_bytes": b,
                     "traffic": recorded_traffic("conv1x1", "xnor_conv1x1_kernel")},
        "l2": f"{R} rotating packed-input/output sets"}
    del cv, Xd, Xb, Wp, al, gam, bet, out
    torch.cuda.empty_cache()


def _row_multibit(torch, bnn, workloads, dev, pk, rows, timed, steps, ws):
    # --- next row: multi-bit products on bit planes (DoReFa codes, ABC-Net bases) ---
    bs = workloads.bitserial()
    M, K = bs.a.shape
    N = bs.w.shape[0]
    ld = bnn.bnn_packed_ld_words(K)
    ad, wd = bs.a.to(dev), bs.w.to(dev)
    A = torch.empty(M * bs.a_bits, ld, dtype=torch.int32, device=dev)
    W = torch.empty(N * bs.w_bits, ld, dtype=torch.int32, device=dev)
    bnn.bnn_pack_bit_planes(wd, bs.w_bits, W, K)
    alpha = torch.full((N,), 0.25, dtype=torch.float32, device=dev)
    # Two rotating (codes, planes, int32 out) sets, 2 x 100 MB, larger than L2 together.
    R = 2
    As = [A] + [A.clone() for _ in range(R - 1)]
    Cs = [torch.empty(M, N, dtype=torch.int32, device=dev) for _ in range(R)]
    ms_g = timed(lambda i: bnn.bnn_bitserial_gemm(As[i % R], bs.a_bits, W, bs.w_bits, K, None, Cs[i % R], None))
    ms_p = timed(lambda i: bnn.bnn_pack_bit_planes(ad, bs.a_bits, As[i % R], K))
    macs = M * N * K
    mac_s = macs * steps / (ms_g * 1e-3)
    pbytes = M * K + A.numel() * 4
    pack_gbs = pbytes * steps / (ms_p * 1e-3) / 1e9
    # Codes of up to two bits run on the e2m1 kernel (exact e2m1 values 0..3), wider ones on int8.
    f4 = max(bs.a_bits, bs.w_bits) <= 2
    kname = "xnor_gemm_f4_kernel" if f4 else "xnor_gemm_tc_kernel"
    roof = _tensor_roofline(pk, mac_s, sustained=False, operand="e2m1" if f4 else "int8")
    roof["traffic"] = recorded_traffic("bitserial_gemm", kname + ("<TC_PLANE_CODES>" if not f4 else ""))
    rows["bitserial_gemm"] = {
        "workload": f"DoReFa-style unsigned codes: a [{M}, {K}] {bs.a_bits}-bit x w [{N}, {K}] {bs.w_bits}-bit as bit "
                    f"planes -> exact int32 sum_k a*w (planes folded to "
                    + ("e2m1 code values, tcgen05 kind::mxf4, CTA pairs)" if f4 else "u8 codes, tcgen05 kind::i8)"),
        "kernel": kname,
        "value": round(ws * mac_s / 1e9, 1), "unit": "code GMAC/s",
        "plane_pair_gmac_s": round(ws * mac_s * bs.a_bits * bs.w_bits / 1e9, 1),
        "ms_per_step": ms_g / steps, "roofline": roof,
        "pack_bit_planes": {"ms": ms_p / steps, "achieved_gbs": round(pack_gbs, 1),
                            "frac": round(pack_gbs / pk["hbm_gbs"], 4), "bytes": pbytes},
        "l2": f"{R} rotating activation-plane / output sets"}
    del bs, ad, wd, A, W, As, Cs, alpha
    torch.cuda.empty_cache()

    bb = workloads.bases()
    J, M, K = bb.h_real.shape
    I, N, _ = bb.b_real.shape
    ld = bnn.bnn_packed_ld_words(K)
    H = torch.empty(M * J, ld, dtype=torch.int32, device=dev)
    B = torch.empty(N * I, ld, dtype=torch.int32, device=dev)
    for j in range(J):
        bnn.bnn_pack_sign(bb.h_real[j].to(dev), H[j::J])
    for i in range(I):
        bnn.bnn_pack_sign(bb.b_real[i].to(dev), B[i::I])
    al, be = bb.alpha.to(dev), bb.beta.to(dev)
    Ys = [torch.empty(M, N, dtype=torch.float32, device=dev) for _ in range(R)]
    Hs = [H] + [H.clone() for _ in range(R - 1)]
    ms_b = timed(lambda i: bnn.bnn_binary_bases_gemm(Hs[i % R], J, B, I, K, be, al, Ys[i % R]))
    jp, ip = 1 << (J - 1).bit_length(), 1 << (I - 1).bit_length()
    bmacs = M * N * K * J * I
    bmac_s = bmacs * steps / (ms_b * 1e-3)
    roof_b = _tensor_roofline(pk, bmac_s, sustained=False, operand="e2m1")
    roof_b["traffic"] = recorded_traffic("binary_bases_gemm", "xnor_gemm_f4_kernel")
    roof_b["note"] = (f"{J} x {I} bases run as {jp} x {ip} (zero bases fill the power-of-two tile): "
                      f"the tensor pipe does {jp * ip / (J * I):.2f}x the algorithmic MACs")
    rows["binary_bases_gemm"] = {
        "workload": f"ABC-Net-style bases: {J} activation bases [{M}, {K}] x {I} weight bases [{N}, {K}], "
                    f"Y = sum_j sum_i beta_j alpha_i[n] (H_j B_i^T) fp32",
        "kernel": "xnor_gemm_f4_kernel (bases mode, CTA pairs)",
        "value": round(ws * bmac_s / 1e9, 1), "unit": "binary GMAC/s (all base pairs)",
        "ms_per_step": ms_b / steps, "roofline": roof_b,
        "l2": f"{R} rotating activation-base / output sets"}
    del bb, H, B, Hs, Ys, al, be
    torch.cuda.empty_cache()


def chain_bytes(c) -> int:
    """Algorithmic bytes of one decode step through a binary layer chain: every
    layer's packed W once, thresholds and modes of the hidden layers, alpha of
    the last, the real input and the fp32 output."""
    total, L = 0, len(c.Ws)
    for l, W in enumerate(c.Ws):
        N, K = W.shape
        total += N * (((K + 31) // 32 + 3) // 4 * 4) * 4
        total += N * 5 if l < L - 1 else N * 4
    return total + c.x0.numel() * c.x0.element_size() + c.Ws[-1].shape[0] * 4


def _row_chain(torch, bnn, workloads, dev, pk, rows, timed, steps, ws):
    # --- next row: one decode step through a fully binary MLP, all layers in one launch ---
    c = workloads.chain()
    L = len(c.Ws)
    packed, layers = [], []
    for l, W in enumerate(c.Ws):
        N, K = W.shape
        Wp = bnn.empty_packed(N, K, dev)
        alpha = torch.empty(N, dtype=torch.float32, device=dev)
        bnn.bnn_pack_sign(W.to(dev), Wp, alpha)
        if l < L - 1:
            bn = c.bns[l]
            thr, mode = bnn.bnn_fold_bn_threshold(alpha.cpu(), bn.gamma, bn.beta, bn.mean, bn.var, bn.eps, K)
            layers.append({"popc_thresh": thr.to(dev), "thresh_mode": mode.to(dev)})
        else:
            layers.append({"alpha": alpha})
        packed.append(Wp)
    b = chain_bytes(c)
    copies = max(2, math.ceil(2 * L2_BYTES / b) + 1)
    sets = []
    for i in range(copies):
        sets.append(bnn.chain_layers([dict(ly, W=(Wp if i == 0 else Wp.clone())) for ly, Wp in zip(layers, packed)]))
    x = c.x0.to(dev)
    y = torch.empty(c.Ws[-1].shape[0], dtype=torch.float32, device=dev)
    wsp = bnn.gemv_chain_workspace(dev)
    n = max(steps, 20) * copies
    ms = timed(lambda i: bnn.bnn_xnor_gemv_chain(sets[i % copies], x, wsp, y_f32=y), n=n, period=copies)
    ach = b * n / (ms * 1e-3) / 1e9
    rows["decode_chain"] = {
        "workload": "batch-1 decode step through a fully binary MLP in one launch: x bf16 [4096] signed, 8 layers "
                    "alternating [11008, 4096] / [4096, 11008] packed W, BatchNorm folded into popcount thresholds "
                    f"between layers, alpha-scaled fp32 out; independent steps over {copies} rotating weight sets",
        "value": round(ws * ach, 1), "unit": "GB/s", "ms_per_step": ms / n, "layers": L,
        "us_per_layer": round(ms / n * 1e3 / L, 3),
        "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"],
                     "frac": round(ach / pk["hbm_gbs"], 4), "algorithmic_bytes": b,
                     "traffic": recorded_traffic("decode_chain", "xnor_gemv_chain_kernel")}}
    del sets, packed, layers, x, y
    torch.cuda.empty_cache()


def _row_mlp(torch, bnn, workloads, dev, rows, timed, steps, ws, alu_peak, pk=None):
    # --- MLP: pack input, 3 x (GEMM + folded-BN re-pack), GEMM + alpha ---
    m = workloads.mlp()
    B, D = m.X0.shape
    # Two rotating sets of (fp32 input, packed activations, fp32 logits), 270 MB
    # in all, so that consecutive steps do not find their data in the 126 MB L2.
    R = 2
    X0 = [m.X0.to(dev) for _ in range(R)]
    A0 = [bnn.empty_packed(B, D, dev) for _ in range(R)]
    acts = [[bnn.empty_packed(B, D, dev) for _ in range(3)] for _ in range(R)]
    eps_ = []
    Wps = []
    for l, W in enumerate(m.Ws):
        Wp = bnn.empty_packed(D, D, dev)
        a = torch.empty(D, dtype=torch.float32, device=dev)
        bnn.bnn_pack_sign(W.to(dev), Wp, a)
        Wps.append(Wp)
        if l < 3:
            bn = m.bns[l]
            thr, mode = bnn.bnn_fold_bn_threshold(a.cpu(), bn.gamma, bn.beta, bn.mean, bn.var, bn.eps, D)
            thr, mode = thr.to(dev), mode.to(dev)
            eps_.append((bnn.make_epilogue(bnn.BNN_OUT_THRESHOLD_PACK, popc_thresh=thr, thresh_mode=mode), thr, mode))
        else:
            eps_.append((bnn.make_epilogue(bnn.BNN_OUT_SCALED_F32, alpha=a), a))
    logits = [torch.empty(B, D, dtype=torch.float32, device=dev) for _ in range(R)]
    rot_mb = R * (X0[0].numel() * 4 + 4 * A0[0].numel() * 4 + logits[0].numel() * 4) / 1e6

    def mlp_step(i):
        r = i % R
        bnn.bnn_pack_sign(X0[r], A0[r])
        A = A0[r]
        for l in range(4):
            o = acts[r][l] if l < 3 else logits[r]
            bnn.bnn_binary_linear_fused(A, Wps[l], D, eps_[l][0], o)
            A = o

    mmacs = 4 * B * D * D
    for name, engine in (("mlp4", bnn.BNN_GEMM_ENGINE_TENSOR), ("mlp4_i8", bnn.BNN_GEMM_ENGINE_TENSOR_I8),
                         ("mlp4_popcount", bnn.BNN_GEMM_ENGINE_POPCOUNT)):
        with bnn.gemm_engine(engine):
            ms_m = timed(mlp_step)
        mac_s = mmacs * steps / (ms_m * 1e-3)
        if engine == bnn.BNN_GEMM_ENGINE_TENSOR:
            roof = _tensor_roofline(pk, mac_s, sustained=False, row=name, operand="e2m1", kernel="xnor_gemm_f4_kernel")
        elif engine == bnn.BNN_GEMM_ENGINE_TENSOR_I8:
            roof = _tensor_roofline(pk, mac_s, sustained=False, row="mlp4")
        else:
            roof = alu_roofline(mac_s, alu_peak)
        rows[name] = {
            "workload": "fully binary MLP, batch 4096, width 4096, 4 layers: pack fp32 input, "
                        "3 x (GEMM + folded BatchNorm sign re-pack), GEMM + alpha fp32 logits",
            "engine": {bnn.BNN_GEMM_ENGINE_TENSOR: "tensor (e2m1)", bnn.BNN_GEMM_ENGINE_TENSOR_I8: "tensor (int8)",
                       bnn.BNN_GEMM_ENGINE_POPCOUNT: "popcount"}[engine],
            "value": round(ws * mac_s / 1e9, 1), "unit": "binary GMAC/s",
            "ms_per_step": ms_m / steps, "roofline": roof,
            "l2": f"{R} rotating input/activation/logit sets, {rot_mb:.0f} MB"}
    del m, X0, A0, acts, eps_, Wps, logits
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# CPU oracle timing (the baseline, never the product path)
# ---------------------------------------------------------------------------

def rows_summary(result: dict) -> dict:
    """One compact entry per figure, placed last on the line so that a reader
    of the line's end sees every row: [value, unit, roofline fraction,
    microseconds per step]."""
    out = {}
    if "value" in result:
        rf = result.get("roofline", {})
        out["headline"] = [result["value"], result["unit"], rf.get("frac"), round(result["ms_per_step"] * 1e3, 3)]
        for k in ("store_ordered", "dependent_chain", "gemv_default_flags", "e2e"):
            v = result.get(k)
            if isinstance(v, dict) and "value" in v:
                out[k] = [v["value"], v["unit"], v.get("frac"), round(v["ms_per_step"] * 1e3, 3)]
    for name, row in result.get("rows", {}).items():
        if not isinstance(row, dict) or "value" not in row:
            continue
        rf = row.get("roofline", {})
        ms = row.get("ms_per_step")
        out[name] = [row["value"], row["unit"], rf.get("frac"), round(ms * 1e3, 3) if ms is not None else None]
        dep = row.get("dependent_chain")
        if isinstance(dep, dict) and "value" in dep:
            out[name + ".dependent_chain"] = [dep["value"], dep["unit"], dep.get("frac"),
                                              round(dep["ms_per_step"] * 1e3, 3)]
    return out


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _time_oracle(step, seconds: float, min_steps: int = 1):
    """Run step() until `seconds` have passed (at least `min_steps` times);
    returns (steps, elapsed seconds)."""
    done = 0
    t0 = time.perf_counter()
    while True:
        step()
        done += 1
        el = time.perf_counter() - t0
        if done >= min_steps and el >= seconds:
            return done, el


def cpu_oracle_gemv_steps(seconds: float, threads: int | None = None):
    """Time the oracle on the decode GEMV: sign(x), the int8 +1/-1 product
    with the pre-binarised W (the oracle's analogue of pre-packed weights),
    and alpha*s in float64.  Whole steps until `seconds` have passed.
    Returns (steps, elapsed_s, threads used)."""
    import oracle
    import workloads

    g = workloads.gemv()
    wb = oracle.sign_pm1(g.W)
    al = oracle.alpha(g.W)
    full = os.cpu_count() or 1
    oracle.set_num_threads(threads or full)
    try:
        n, el = _time_oracle(lambda: oracle.scaled(oracle.gemv_pm1(wb, oracle.sign_pm1(g.x)), al), seconds)
        used = oracle.num_threads()
    finally:
        oracle.set_num_threads(full)
    return n, el, used


def cpu_baseline_gemv(seconds: float):
    """The oracle on all host cores (the outputs split over OpenMP threads),
    and the same on one core beside it."""
    n, el, threads = cpu_oracle_gemv_steps(seconds)
    n1, el1, _ = cpu_oracle_gemv_steps(max(2.0, seconds / 3), threads=1)
    return {"value": round(n * gemv_bytes() / el / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{n} whole GEMV steps of the same workload ({el:.1f} s): sign(x), int8 +1/-1 "
                      f"product with the pre-binarised W, alpha*s in float64",
            "one_core": {"value": round(n1 * gemv_bytes() / el1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                         "sample": f"{n1} steps ({el1:.1f} s)"},
            "host_cpus": os.cpu_count(), "cpu_model": cpu_model()}


def cpu_baseline_rows(rows: dict, seconds: float) -> None:
    """Time the oracle on a bounded sample of each measured row's workload, on
    all host cores, and attach it as rows[name]["cpu_baseline"] in that row's
    unit.  The samples are stated; each is the oracle's own computation of the
    same outputs (sign, the plain +1/-1 integer product, the float64 epilogue)."""
    import numpy as np

    import oracle
    import workloads

    full = os.cpu_count() or 1
    oracle.set_num_threads(full)
    model = cpu_model()

    def put(name, value, unit, sample, one_core=None, numpy_only=False):
        # The C loops (products, convolutions) run on the OpenMP threads; the
        # add/sub GEMVs and the code product are numpy expressions on one core.
        if name in rows and isinstance(rows[name], dict) and "error" not in rows[name]:
            d = {"value": value, "unit": unit, "cores": 1 if numpy_only else oracle.num_threads(), "kind": "oracle",
                 "sample": sample, "host_cpus": os.cpu_count(), "cpu_model": model}
            if one_core is not None:
                d["one_core"] = one_core
            rows[name]["cpu_baseline"] = d

    if "square_gemm" in rows or "square_gemm_popcount" in rows:
        sq = workloads.square()
        ab, wb = oracle.sign_pm1(sq.A[:8]), oracle.sign_pm1(sq.W)
        al = oracle.alpha(sq.W)
        R = 2
        n, el = _time_oracle(lambda: oracle.scaled(oracle.matmul_pm1(ab[:R], wb), al), seconds)
        v = n * R * sq.N * sq.K / el / 1e9
        oracle.set_num_threads(1)
        n1, el1 = _time_oracle(lambda: oracle.scaled(oracle.matmul_pm1(ab[:1], wb), al), seconds / 2)
        oracle.set_num_threads(full)
        one = {"value": round(n1 * sq.N * sq.K / el1 / 1e9, 4), "unit": "binary GMAC/s", "cores": 1,
               "sample": f"{n1} x 1 row ({el1:.1f} s)"}
        for name in ("square_gemm", "square_gemm_popcount"):
            put(name, round(v, 4), "binary GMAC/s",
                f"{n} x {R} rows of A (of 8192) against all 8192 rows of W, K = 8192, pre-binarised operands, "
                f"int32 s and alpha*s in float64 ({el:.1f} s)", one)
        del sq, ab, wb
    if "conv3x3" in rows:
        cv = workloads.conv()
        x1 = cv.X[:1]
        n, el = _time_oracle(lambda: oracle.conv3x3_affine(x1, cv.W, cv.gamma.numpy(), cv.beta.numpy()), seconds)
        macs = 56 * 56 * 64 * 9 * 64
        for name in ("conv3x3", "conv3x3_tensor", "conv3x3_popcount"):
            put(name, round(n * macs / el / 1e9, 4), "binary GMAC/s",
                f"{n} x 1 image (of 64): sign, 7-loop +1/-1 convolution, alpha and affine in float64 ({el:.1f} s)")
        del cv
    if "mlp4" in rows:
        m = workloads.mlp()
        bns = [(b.gamma.numpy(), b.beta.numpy(), b.mean.numpy(), b.var.numpy(), b.eps) for b in m.bns]
        R = 4
        x = m.X0[:R]
        n, el = _time_oracle(lambda: oracle.mlp_forward(x, m.Ws, bns), seconds)
        macs = R * 4 * 4096 * 4096
        for name in ("mlp4", "mlp4_popcount"):
            put(name, round(n * macs / el / 1e9, 4), "binary GMAC/s",
                f"{n} x {R} rows (of 4096) through all 4 layers: sign of the input and of every W, +1/-1 "
                f"products, BatchNorm sign in float64, alpha*s logits ({el:.1f} s)")
        del m
    if "bw_gemv" in rows:
        g = workloads.gemv()
        wb, al, xf = oracle.sign_pm1(g.W), oracle.alpha(g.W), oracle._f32(g.x)
        n, el = _time_oracle(lambda: oracle.scaled(oracle.binary_weight_product(wb, xf), al), seconds)
        put("bw_gemv", round(n * gemv_bytes() / el / 1e9, 4), "GB/s",
            f"{n} whole steps, pre-binarised W: +x / -x sums in float64, alpha ({el:.1f} s)", numpy_only=True)
        del g, wb
    if "bw_gemv_i8" in rows:
        g, t = workloads.gemv(), workloads.ternary()
        wb, al, xq = oracle.sign_pm1(g.W), oracle.alpha(g.W), t.x.numpy().astype(np.float64)
        n, el = _time_oracle(lambda: al * (1.0 / 64) * oracle.binary_weight_product(wb, xq), seconds)
        b8 = 11008 * 128 * 4 + 4 * 11008 + 4096 + 4 * 11008 + 4
        put("bw_gemv_i8", round(n * b8 / el / 1e9, 4), "GB/s",
            f"{n} whole steps, pre-binarised W: +x / -x sums of the int8 x, alpha * x_scale ({el:.1f} s)",
            numpy_only=True)
        del g, t, wb
    if "ternary_gemv" in rows:
        t = workloads.ternary()
        tq, gam = oracle.ternary_quantize(t.W)
        xq = t.x.numpy()
        n, el = _time_oracle(lambda: oracle.ternary_gemv_i8(tq, xq, gam, 1.0 / 64), seconds)
        b = 11008 * bnn_ternary_ld(4096) * 4 + 4096 + 4 * 11008 + 8
        put("ternary_gemv", round(n * b / el / 1e9, 4), "GB/s",
            f"{n} whole steps with the pre-quantised ternary W: exact int64 sum of t*x, scaled ({el:.1f} s)",
            numpy_only=True)
        del t, tq
    if "conv1x1" in rows:
        cv = workloads.downsample()
        x1 = cv.X[:1]
        n, el = _time_oracle(lambda: oracle.conv_affine(x1, cv.W, cv.gamma.numpy(), cv.beta.numpy(), stride=2,
                                                        pad=0), seconds)
        b1 = 28 * 28 * 2 * 4 + 128 * 4 * 4 + 128 * 28 * 28 * 4
        put("conv1x1", round(n * b1 / el / 1e9, 4), "GB/s",
            f"{n} x 1 image (of 64): sign, 1x1 stride-2 +1/-1 convolution, alpha and affine ({el:.1f} s)")
        del cv
    if "bitserial_gemm" in rows:
        bs = workloads.bitserial()
        a, w = bs.a[:4].numpy(), bs.w.numpy()
        n, el = _time_oracle(lambda: [oracle.bitserial_product(a[i:i + 1], w) for i in range(4)], seconds)
        put("bitserial_gemm", round(n * 4 * 4096 * 4096 / el / 1e9, 4), "code GMAC/s",
            f"{n} x 4 rows (of 4096) of the 2-bit x 2-bit code product, int64 sums of products ({el:.1f} s)",
            numpy_only=True)
        del bs
    if "binary_bases_gemm" in rows:
        bb = workloads.bases()
        h = oracle.sign_pm1(bb.h_real[:, :2].numpy())
        bw = oracle.sign_pm1(bb.b_real.numpy())
        al, be = bb.alpha.numpy(), bb.beta.numpy()
        n, el = _time_oracle(lambda: oracle.binary_bases_product(h, bw, al, be), seconds)
        put("binary_bases_gemm", round(n * 2 * 4096 * 4096 * 9 / el / 1e9, 4), "binary GMAC/s (all base pairs)",
            f"{n} x 2 rows (of 4096), 3 x 3 base pairs of +1/-1 products, weighted sum in float64 ({el:.1f} s)")
        del bb


    if "decode_chain" in rows:
        c = workloads.chain()
        bns = [(b.gamma.numpy(), b.beta.numpy(), b.mean.numpy(), b.var.numpy(), b.eps) for b in c.bns]
        wb = [oracle.sign_pm1(W) for W in c.Ws]
        als = [oracle.alpha(W) for W in c.Ws]

        def forward():
            # the oracle's MLP forward at batch 1, with every W binarised once up front
            a = oracle.sign_pm1(c.x0)[None, :]
            for l in range(len(wb)):
                s_ = oracle.matmul_pm1(a, wb[l])
                if l < len(wb) - 1:
                    g_, be, mu, var, eps = bns[l]
                    a = oracle.bn_sign(s_, als[l].astype(np.float32), g_, be, mu, var, eps)
                else:
                    oracle.scaled(s_, als[l])
        n, el = _time_oracle(forward, seconds)
        put("decode_chain", round(n * chain_bytes(c) / el / 1e9, 4), "GB/s",
            f"{n} whole steps through all 8 layers with pre-binarised W: +1/-1 products, BatchNorm sign in "
            f"float64, alpha*s logits ({el:.1f} s)")
        del c, wb


def bnn_ternary_ld(K: int) -> int:
    return ((K + 15) // 16 + 3) // 4 * 4


def run_reference(args):
    """The CPU oracle on the headline workload.  Each step is a bounded sample:
    the GEMV over the first `rows` output rows, with `rows` chosen so that the
    whole --warmup + --steps run takes about two minutes of host time."""
    import oracle
    import workloads

    g = workloads.gemv()
    wb = oracle.sign_pm1(g.W)
    al = oracle.alpha(g.W)
    t0 = time.perf_counter()
    oracle.scaled(oracle.gemv_pm1(wb, oracle.sign_pm1(g.x)), al)
    t_full = time.perf_counter() - t0
    total = max(1, args.steps + args.warmup)
    rows = int(max(1, min(GEMV_N, GEMV_N * 120.0 / (total * t_full))))
    wbs, als = wb[:rows], al[:rows]

    def step():
        oracle.scaled(oracle.gemv_pm1(wbs, oracle.sign_pm1(g.x)), als)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    kw = ((GEMV_K + 31) // 32 + 3) // 4 * 4
    step_bytes = rows * kw * 4 + rows * 4 + GEMV_K * 2 + rows * 4
    value = args.steps * step_bytes / el / 1e9
    sample = (f"each step the GEMV over the first {rows} of {GEMV_N} output rows "
              f"(sign(x), int8 +1/-1 product with the pre-binarised W, alpha*s in float64); "
              f"{args.steps} timed steps, {el:.1f} s")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": el * 1e3 / max(1, args.steps),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int32",
        "data": "synthetic",
        "config": {"workload": "LLM-decode binary GEMV: packed +1/-1 W [11008, 4096] from N(0,0.02), "
                               "x bf16 [4096] N(0,1), per-row alpha, fp32 y",
                   "N": GEMV_N, "K": GEMV_K, "algorithmic_bytes_per_step": gemv_bytes()},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample, "host_cpus": os.cpu_count()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=192000)
    ap.add_argument("--warmup", type=int, default=480)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--row-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--cpu-row-seconds", type=float, default=3.0)
    ap.add_argument("--no-rows", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only-rows", default=None,
                    help="comma-separated rows to time alone (no headline line); for profiling: "
                         + ",".join(ROW_NAMES))
    ap.add_argument("--square-shape", default=None,
                    help="M,N,K of the square_gemm row in an --only-rows run (a smaller case of the same "
                         "kernel for profiling; default 8192,8192,8192)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.square_shape is not None and args.only_rows is None:
        ap.error("--square-shape only applies to --only-rows runs")

    ws, rank, local = dist_env()
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    import torch
    dist = None
    if ws > 1:
        import datetime
        import torch.distributed as dist_mod
        torch.cuda.set_device(local)
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        dist = dist_mod
    else:
        torch.cuda.set_device(local)
    try:
        if args.only_rows:
            result = run_only_rows(args, torch, dist)
        else:
            result = run_ours(args, torch, dist)
        if rank == 0:
            if "rows" in result:
                result["summary"] = rows_summary(result)
            print(json.dumps(result), flush=True)
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
