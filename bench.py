#!/usr/bin/env python
"""Benchmark of the B200 BitLinear forward (ternary weights x int8 activations).

Headline (one JSON line on rank 0): decode weight GB/s of the BitNet b1.58
2B4T feed-forward BitLinears at M = 1 token -- per step one token passes the
gate (2560 -> 6912), up (2560 -> 6912) and down (6912 -> 2560) projections of
every one of the 30 layers of a 2B4T-shaped stack (398 MB of 2-bit weights,
larger than the 126 MB L2, so every step streams its weights from HBM).  gate
and up share their input and run as one grouped GEMV launch, down as another:
60 launches per step.  Weights are drawn directly in ternary form (P(0) = 0.42,
P(+-1) = 0.29, alpha ~ U(0.01, 0.05)); x ~ N(0, 1) in bf16.  The step is
captured once in a CUDA graph with programmatic dependent launch between the
GEMVs.  Bytes per step = sum over matrices of N*K/4 packed codes + 4 (alpha)
+ 2N (y), plus 2K per distinct input row (x once for gate and up, h for down).

A second object, "prefill", reports int8 TOPS of the tensor-core GEMM on the
2B4T prefill shapes (M = 2048 tokens; 2560 -> 6912, 6912 -> 2560,
2560 -> 2560, 2560 -> 640; latent W ~ N(0, 0.02), x with 1% x10 outliers),
inputs larger than L2, counted as 2*M*N*K ops: the GEMM kernel alone (codes
in, bitlinear_forward_q8) as the value, the whole forward call (quantisation
launch + GEMM) beside it.

Further objects on the same line (skipped with --no-sweep, except the
last): "sweep" (the 7 BitLinears of a 2B4T layer at M = 1, 16, 256, 4096),
"nm" (Sparse-BitNet 2:4 and 6:8 on the Qwen2.5-3B MLP shapes at M = 1 and
4096), "norm" (RMSNorm fused into the activation quantisation), "decode_lut"
(the lookup-table decode GEMV against the dp4a one) and "isolated" (one
eager forward call at M = 1 on a cold L2, launch latency included).

--impl reference times the oracle (plain C, one host core) on the same
workload and metric.  Multi-GPU (torchrun) runs independent replicas: the
path has no exchange step, per-GPU work is fixed, the time is the max over
ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode weight GB/s (% HBM peak); prefill int8 TOPS (% tensor peak)"
LAYERS = 30
FFN = (("gate", 2560, 6912), ("up", 2560, 6912), ("down", 6912, 2560))  # (name, K, N)
PREFILL_SHAPES = ((2560, 6912), (6912, 2560), (2560, 2560), (2560, 640))  # (K, N)
PREFILL_M = 2048
DISTINCT_LAYERS = 2  # distinct weight draws, replicated to 30 layers at distinct addresses
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "gemv_dense__decode_2b4t_ffn.json")
GEMV_SOURCES = ("gemv.cuh", "quant_pack.cuh", "ptx.cuh")


def decode_bytes_per_gemv(K: int, N: int) -> int:
    return N * K // 4 + 4 + 2 * K + 2 * N


def decode_step_bytes(layers: int = LAYERS) -> int:
    mats = sum(N * K // 4 + 4 + 2 * N for _, K, N in FFN)
    inputs = 2 * 2560 + 2 * 6912  # x (read once by the grouped gate/up launch) and h
    return layers * (mats + inputs)


# ------------------------------------------------------------------ multi-rank plumbing

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank_step: float, steps: int, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return units_per_rank_step * steps * world / max_seconds


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Polls SM clock, max clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.002, pci_bus_id: str = None):
        self.index, self.period, self.bus = index, period_s, pci_bus_id
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            if self.bus:
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(self.bus.encode())
            else:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        except Exception:
            self.ok = False
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr:
            self._thr.join()
        return False

    def summary(self):
        if not self.ok or not self.samples:
            return None
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ------------------------------------------------------------------ peaks, profile

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# Definitions the dense decode GEMV is compiled from (kernel, device helpers, PTX wrappers).
GEMV_DEFS = ("gemv_dense_kernel", "quantise_row_smem", "quantise_row_smem_norm", "gemv_wchunk",
             "dot_word", "gemv_store", "gemv_stripes", "gemv_stripe_bytes", "gemv_smem_bytes", "codes8", "codes8f",
             "load8_raw", "sumsq8", "mbar_init", "mbar_arrive_expect_tx", "mbar_try_wait", "mbar_wait",
             "fence_mbar_init", "tma_prefetch_desc", "tma_load_2d_hint", "l2_policy_evict_first", "dp4a_us",
             "pdl_wait_primary", "pdl_launch_dependents", "smem_u32", "globaltimer_ns", "struct GemvDense",
             "struct GemvMat", "row_code_sum", "gemv_gave_up", "wait_limit_ns", "test_extra_tx",
             "gemv_row_totals")


# Lines of the test build's phase stamps: compiled out of the product library, so not part of the
# fingerprint of the code the measured kernel runs.
TIMELINE_MARKS = ("tl_now", "tl_commit", "kTimeline")


def gemv_source_hash() -> str:
    """Fingerprint of the text of the definitions in GEMV_DEFS: a top-level definition runs from
    its first line to the next line that is a lone closing brace (lines of the test build's phase
    stamps left out)."""
    import re
    h = hashlib.sha256()
    for n in GEMV_SOURCES:
        with open(os.path.join(ROOT, "ternary_weight_linear_fwd_b200", "csrc", n)) as f:
            lines = [ln for ln in f.read().split("\n") if not any(m in ln for m in TIMELINE_MARKS)]
        i = 0
        while i < len(lines):
            line = lines[i]
            hit = any(re.search(r"(^|\W)" + re.escape(d) + r"\s*(\(|\{|$)", line) for d in GEMV_DEFS)
            if hit and not line.startswith((" ", "/", "#")):
                j = i
                while j < len(lines) and lines[j] not in ("}", "};"):
                    j += 1
                h.update("\n".join(lines[i:j + 1]).encode())
                i = j + 1
            else:
                i += 1
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per GEMV launch from the committed ncu figures (profiles/*.json), if they were taken on
    today's kernel source (same fingerprint of the definitions in GEMV_DEFS)."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    with open(PROFILE_TRAFFIC) as f:
        d = json.load(f)
    if d.get("source_sha256_16") != gemv_source_hash():
        return None
    try:
        return float(d["dram_bytes_per_launch"])
    except (KeyError, TypeError, ValueError):
        return None


# ------------------------------------------------------------------ workloads (ours)

def build_decode(dev, layers: int, seed: int = 1):
    """Packed weights of `layers` FFN layers (distinct addresses), inputs and outputs."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth

    distinct = []
    for d in range(DISTINCT_LAYERS):
        mats = {}
        for j, (name, K, N) in enumerate(FFN):
            s = seed + 100 * d + j
            T = torch.from_numpy(synth.ternary_weights(N, K, seed=s)).to(dev)
            mats[name] = bl.pack_ternary(T, float(synth.alpha_uniform(s)))
            del T
        distinct.append(mats)
    layers_w = []
    for l in range(layers):
        src = distinct[l % DISTINCT_LAYERS]
        cp = {}
        for name, K, N in FFN:
            w = src[name]
            cp[name] = bl.PackedWeights(w.N, w.K, 0, 0, w.codes.clone(), None, w.alpha.clone())
        layers_w.append(cp)
    del distinct
    x_in = torch.from_numpy(synth.activations(layers, 2560, seed=seed, outlier_p=0.0).view(np.int16)).to(dev)
    h_in = torch.from_numpy(synth.activations(layers, 6912, seed=seed + 1, outlier_p=0.0).view(np.int16)).to(dev)
    x_in = x_in.view(torch.bfloat16)
    h_in = h_in.view(torch.bfloat16)
    y_gate = torch.empty((layers, 6912), dtype=torch.bfloat16, device=dev)
    y_up = torch.empty_like(y_gate)
    y_down = torch.empty((layers, 2560), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize(dev)
    return layers_w, x_in, h_in, y_gate, y_up, y_down


def decode_step_fn(layers_w, x_in, h_in, y_gate, y_up, y_down, flags):
    import ternary_weight_linear_fwd_b200 as bl

    def step():
        for l, w in enumerate(layers_w):
            bl.forward_group([w["gate"], w["up"]], x_in[l:l + 1], outs=[y_gate[l:l + 1], y_up[l:l + 1]], flags=flags)
            bl.forward(w["down"], h_in[l:l + 1], out=y_down[l:l + 1], flags=flags)
    return step


def time_graph(graph, steps: int, warmup: int, dev, clock_index: int):
    import torch
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize(dev)
    barrier(dev)
    s = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p = torch.cuda.get_device_properties(dev)
    bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
    with ClockSampler(clock_index, pci_bus_id=bus) as clk:
        torch.cuda.synchronize(dev)
        e0.record(s)
        for _ in range(steps):
            graph.replay()
        e1.record(s)
        e1.synchronize()
    torch.cuda.synchronize(dev)
    barrier(dev)
    return e0.elapsed_time(e1) / 1e3, clk.summary()


def run_decode(dev, steps, warmup, layers, clock_index):
    import torch

    import ternary_weight_linear_fwd_b200 as bl

    buf = build_decode(dev, layers)
    layers_w, x_in, h_in, y_gate, y_up, y_down = buf
    step = decode_step_fn(*buf, flags=bl.FLAG_PDL)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        step()  # warm the library (attributes, module load) outside capture
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    launches_per_step = 2 * layers
    secs, clocks = time_graph(g, steps, warmup, dev, clock_index)
    assert bl.device_status() == 0

    # end to end: pinned host inputs -> device, the captured public-API step, outputs -> host
    h_x = torch.empty(x_in.shape, dtype=x_in.dtype, pin_memory=True).copy_(x_in.cpu())
    h_h = torch.empty(h_in.shape, dtype=h_in.dtype, pin_memory=True).copy_(h_in.cpu())
    o_g = torch.empty(y_gate.shape, dtype=y_gate.dtype, pin_memory=True)
    o_u = torch.empty_like(o_g, pin_memory=True)
    o_d = torch.empty(y_down.shape, dtype=y_down.dtype, pin_memory=True)
    s = torch.cuda.current_stream(dev)

    def e2e_step():
        x_in.copy_(h_x, non_blocking=True)
        h_in.copy_(h_h, non_blocking=True)
        g.replay()
        o_g.copy_(y_gate, non_blocking=True)
        o_u.copy_(y_up, non_blocking=True)
        o_d.copy_(y_down, non_blocking=True)

    for _ in range(max(3, warmup)):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(1, min(steps, 2000))
    e0.record(s)
    for _ in range(e_steps):
        e2e_step()
    e1.record(s)
    e1.synchronize()
    e2e_secs = e0.elapsed_time(e1) / 1e3
    barrier(dev)
    h2d = (x_in.numel() + h_in.numel()) * 2
    d2h = (y_gate.numel() + y_up.numel() + y_down.numel()) * 2
    del g

    # the same, issued call by call (no graph): the per-call host path of the binding and the C ABI
    def e2e_eager_step():
        x_in.copy_(h_x, non_blocking=True)
        h_in.copy_(h_h, non_blocking=True)
        step()
        o_g.copy_(y_gate, non_blocking=True)
        o_u.copy_(y_up, non_blocking=True)
        o_d.copy_(y_down, non_blocking=True)

    for _ in range(max(3, warmup)):
        e2e_eager_step()
    torch.cuda.synchronize(dev)
    barrier(dev)
    eager_steps = max(1, min(steps, 200))
    e0.record(s)
    for _ in range(eager_steps):
        e2e_eager_step()
    e1.record(s)
    e1.synchronize()
    eager_secs = e0.elapsed_time(e1) / 1e3
    barrier(dev)
    return {"secs": secs, "clocks": clocks, "launches_per_step": launches_per_step, "e2e_secs": e2e_secs,
            "e2e_steps": e_steps, "h2d": h2d, "d2h": d2h, "e2e_eager_steps": eager_steps,
            "e2e_eager_ms": eager_secs / eager_steps * 1e3,
            "e2e_eager_gbps": decode_step_bytes(layers) * eager_steps / eager_secs / 1e9}


def run_ffn_glu(dev, layers: int, steps: int = 200, warmup: int = 5):
    """The decode FFN stack with its own dataflow: per layer h = ReLU(gate x)^2 * (up x) in one launch
    (bitlinear_forward_relu2_glu at M = 1), then down(h) reading that h; one CUDA graph with PDL edges.
    Same weight bytes per step as the headline decode step."""
    import torch

    import ternary_weight_linear_fwd_b200 as bl

    layers_w, x_in, h_in, y_gate, y_up, y_down = build_decode(dev, layers)
    h = torch.empty((layers, 6912), dtype=torch.bfloat16, device=dev)

    def step():
        for l, w in enumerate(layers_w):
            bl.forward_relu2_glu(w["gate"], w["up"], x_in[l:l + 1], out=h[l:l + 1], flags=bl.FLAG_PDL)
            bl.forward(w["down"], h[l:l + 1], out=y_down[l:l + 1], flags=bl.FLAG_PDL)

    secs = time_chain_graph(dev, [step], warmup, steps)
    kern = bl.last_kernel()
    step_bytes = decode_step_bytes(layers) - layers * 6912 * 2  # one FFN intermediate instead of two outputs
    return {"us_per_step": secs * 1e6, "GBps": step_bytes / secs / 1e9, "launches_per_step": 2 * layers,
            "kernels": ["gemv_m1_relu2_glu", kern]}


def run_prefill(dev, iters: int, warmup: int):
    """Per shape: forward at M = 2048, timed on the device two ways: over rotating copies of x and of
    the weights (working set > 2 x L2; the reported figure), and with an L2 flush (256 MB write)
    before each call, as CUDA-graph replays of (flush, forward) minus replays of the flush alone."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    x = torch.from_numpy(synth.activations(PREFILL_M, 6912, seed=3).view(np.int16)).to(dev).view(torch.bfloat16)
    out = {}
    tot_ops, tot_sec, tot_sec_fl, tot_gemm = 0.0, 0.0, 0.0, 0.0
    s = torch.cuda.current_stream(dev)
    kernel = None
    for K, N in PREFILL_SHAPES:
        W = torch.from_numpy(synth.latent_weights(N, K, seed=3)).to(dev)
        w = bl.pack_weights(W)
        del W
        xk = x[:, :K].contiguous()
        y = torch.empty((PREFILL_M, N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(bl.forward_workspace_bytes(PREFILL_M, N, K), dtype=torch.uint8, device=dev)
        for _ in range(warmup):
            bl.forward(w, xk, out=y, workspace=ws)
        kernel = bl.last_kernel()
        # Device time only: one graph replays (L2 flush, forward) pairs, another the flushes
        # alone; the difference per pair is the forward on a cold L2 (no host gaps).
        pair = [lambda: flush.fill_(1), lambda: bl.forward(w, xk, out=y, workspace=ws)]
        times = []
        for _ in range(max(1, iters // 10)):
            t_both = time_chain_graph(dev, pair * 10, 1, 3)
            t_flush = time_chain_graph(dev, [lambda: flush.fill_(1)] * 10, 1, 3)
            times.append((t_both - t_flush) / 10)
        med = statistics.median(times)
        # the activation quantisation alone (public bitlinear_quant_act: same kernel, natural k order), cold L2
        q = torch.empty((PREFILL_M, K), dtype=torch.int8, device=dev)
        gq = torch.empty(PREFILL_M, dtype=torch.float32, device=dev)
        lib = bl.lib()
        qcall = (lambda: lib.bitlinear_quant_act(xk.data_ptr(), PREFILL_M, K, q.data_ptr(), gq.data_ptr(), None,
                                                 torch.cuda.current_stream(dev).cuda_stream))
        t_qb = time_chain_graph(dev, [lambda: flush.fill_(1), qcall] * 10, 1, 3)
        t_qf = time_chain_graph(dev, [lambda: flush.fill_(1)] * 10, 1, 3)
        quant_us = (t_qb - t_qf) / 10 * 1e6
        ops = 2.0 * PREFILL_M * N * K
        # The same call over rotating copies of x and of the packed weights (working set > 2 x L2, so
        # every call reads both from HBM) in a PDL-chained graph: cold inputs without the write-back
        # of a dirty flush buffer competing with the call's reads.
        n_cp = max(2, -(-L2_DEFEAT_BYTES // (xk.numel() * 2 + w.nbytes)))
        xs = [xk] + [xk.clone() for _ in range(n_cp - 1)]
        wcs = [w] + [bl.PackedWeights(w.N, w.K, 0, 0, w.codes.clone(), None, w.alpha.clone()) for _ in range(n_cp - 1)]
        calls = [(lambda i=i: bl.forward(wcs[i], xs[i], out=y, workspace=ws, flags=bl.FLAG_PDL)) for i in range(n_cp)]
        rot = statistics.median([time_chain_graph(dev, calls, 2, 3) / n_cp for _ in range(3)])
        # The GEMM kernel alone: bitlinear_forward_q8 on each copy's codes (quantised once, before the
        # timed region), the same rotation of weight and code copies.
        qs = [bl.quant_act(xi) for xi in xs]
        gcalls = [(lambda i=i: bl.forward_q8(wcs[i], qs[i][0], qs[i][1], qs[i][2], out=y, flags=bl.FLAG_PDL))
                  for i in range(n_cp)]
        gem = statistics.median([time_chain_graph(dev, gcalls, 2, 3) / n_cp for _ in range(3)])
        gemm_kernel = bl.last_kernel()
        del xs, wcs, calls, qs, gcalls
        out[f"{K}x{N}"] = {"ms": rot * 1e3, "tops": ops / rot / 1e12, "copies": n_cp,
                           "gemm_us": gem * 1e6, "gemm_tops": ops / gem / 1e12, "gemm_kernel": gemm_kernel,
                           "flushed_ms": med * 1e3, "flushed_tops": ops / med / 1e12, "quant_alone_us": quant_us,
                           "quant_alone_GBps": (3 * PREFILL_M * K + 8 * PREFILL_M) / (quant_us * 1e-6) / 1e9}
        del q, gq
        tot_ops += ops
        tot_sec += rot
        tot_sec_fl += med
        tot_gemm += gem
    assert bl.device_status() == 0
    return {"shapes": out, "tops": tot_ops / tot_sec / 1e12, "kernel": kernel, "ops": tot_ops, "secs": tot_sec,
            "flushed_tops": tot_ops / tot_sec_fl / 1e12, "gemm_tops": tot_ops / tot_gemm / 1e12}


def time_chain_graph(dev, calls, warmup: int, reps: int) -> float:
    """Seconds per replay of a CUDA graph holding `calls` (callables that enqueue
    library calls on the current stream), after `warmup` replays."""
    import torch
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for c in calls:
            c()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c in calls:
            c()
    for _ in range(warmup):
        g.replay()
    s = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(s)
    for _ in range(reps):
        g.replay()
    e1.record(s)
    e1.synchronize()
    del g
    return e0.elapsed_time(e1) / 1e3 / reps


L2_DEFEAT_BYTES = 2 * 126 * 1024 * 1024  # weights rotated over copies until the working set is twice L2
SWEEP_M = (1, 16, 256, 4096)
NM_PATTERNS = ((2, 4), (6, 8))
NM_M = (1, 4096)


def _copies(w, nbytes: int):
    """Distinct device copies of packed weights so that a chain of calls streams > 2 x L2."""
    import ternary_weight_linear_fwd_b200 as bl
    n = max(1, min(1024, -(-L2_DEFEAT_BYTES // max(1, nbytes))))
    return [w] + [bl.PackedWeights(w.N, w.K, w.nm_n, w.nm_m, w.codes.clone(),
                                   None if w.meta is None else w.meta.clone(), w.alpha.clone()) for _ in range(n - 1)]


def run_sweep(dev, min_calls: int = 16, warmup: int = 3, reps: int = 5):
    """Layer sweep: the seven 2B4T BitLinears at M in SWEEP_M; per matrix a PDL-chained graph that
    calls each of its weight copies once (> 2 x L2 of weights per replay)."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth

    packed = {}
    for i, (name, (K, N)) in enumerate(synth.B2B4T_LAYER.items()):
        T = torch.from_numpy(synth.ternary_weights(N, K, seed=4 + 10 * i)).to(dev)
        packed[name] = bl.pack_ternary(T, float(synth.alpha_uniform(4 + 10 * i)))
        del T
    out = {}
    for M in SWEEP_M:
        x = torch.from_numpy(synth.activations(M, 6912, seed=4).view(np.int16)).to(dev).view(torch.bfloat16)
        ws = torch.empty(max(1, max(bl.forward_workspace_bytes(M, N, K) for K, N in synth.B2B4T_LAYER.values())),
                         dtype=torch.uint8, device=dev)
        row, tot_b, tot_ops, tot_s = {}, 0, 0.0, 0.0
        for name, (K, N) in synth.B2B4T_LAYER.items():
            xk = x[:, :K].contiguous()
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            wbytes = packed[name].nbytes
            cps = _copies(packed[name], wbytes)
            ncall = max(min_calls, len(cps))
            calls = [(lambda w=cps[i % len(cps)]: bl.forward(w, xk, out=y, workspace=ws, flags=bl.FLAG_PDL))
                     for i in range(ncall)]
            sec = time_chain_graph(dev, calls, warmup, reps) / ncall
            nbytes = N * K // 4 + 4 + 2 * M * K + 2 * M * N
            ops = 2.0 * M * N * K
            row[name] = {"us": sec * 1e6, "GBps": nbytes / sec / 1e9, "TOPS": ops / sec / 1e12,
                         "kernel": bl.last_kernel(), "weight_copies": len(cps)}
            tot_b, tot_ops, tot_s = tot_b + nbytes, tot_ops + ops, tot_s + sec
            del cps, calls, y, xk
        row["layer"] = {"us": tot_s * 1e6, "GBps": tot_b / tot_s / 1e9, "TOPS": tot_ops / tot_s / 1e12}
        peaks, _ = measured_peaks()
        row["layer"]["hbm_frac"] = row["layer"]["GBps"] / peaks["hbm_gbs"]
        row["layer"]["int8_frac"] = row["layer"]["TOPS"] / (2.0 * peaks["bf16_tflops"])
        out[f"M={M}"] = row
        del x, ws
    assert bl.device_status() == 0
    return out


def run_nm(dev, min_calls: int = 16, warmup: int = 3, reps: int = 5):
    """Sparse-BitNet N:M on the Qwen2.5-3B MLP shapes at M in NM_M (same chained-graph timing)."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth

    out = {}
    for n, m in NM_PATTERNS:
        for name, (K, N) in synth.QWEN25_3B_MLP.items():
            W = torch.from_numpy(synth.latent_weights(N, K, seed=5)).to(dev)
            w = bl.pack_weights(W, n, m)
            del W
            for M in NM_M:
                x = torch.from_numpy(synth.activations(M, K, seed=5).view(np.int16)).to(dev).view(torch.bfloat16)
                ws = torch.empty(max(1, bl.forward_workspace_bytes(M, N, K)), dtype=torch.uint8, device=dev)
                y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
                cps = _copies(w, w.nbytes) if M == 1 else [w]
                ncall = max(min_calls, len(cps))
                calls = [(lambda ww=cps[i % len(cps)]: bl.forward_nm(ww, x, out=y, workspace=ws, flags=bl.FLAG_PDL))
                         for i in range(ncall)]
                sec = time_chain_graph(dev, calls, warmup, reps) / ncall
                nbytes = w.nbytes + 4 + 2 * M * K + 2 * M * N
                key = f"{n}:{m} {name} {K}->{N} M={M}"
                out[key] = {"us": sec * 1e6, "GBps": nbytes / sec / 1e9, "TOPS_dense_equiv": 2.0 * M * N * K / sec / 1e12,
                            "packed_bytes": w.nbytes, "kernel": bl.last_kernel(), "weight_copies": len(cps)}
                if (n, m) == (2, 4) and M > 1:
                    # the same call with the kept values expanded for the dense MMA, and the dense (unpruned)
                    # matrix of the same shape: what the structured-sparse MMA is measured against
                    ce = [(lambda: bl.forward_nm(w, x, out=y, workspace=ws, flags=bl.FLAG_PDL | bl.FLAG_NM24_EXPAND))]
                    se = time_chain_graph(dev, ce * ncall, warmup, reps) / ncall
                    out[key]["expanded_dense_mma"] = {"us": se * 1e6, "TOPS_dense_equiv": 2.0 * M * N * K / se / 1e12,
                                                      "kernel": bl.last_kernel()}
                    Wd = torch.from_numpy(synth.latent_weights(N, K, seed=5)).to(dev)
                    wd = bl.pack_weights(Wd)
                    del Wd
                    cd = [(lambda: bl.forward(wd, x, out=y, workspace=ws, flags=bl.FLAG_PDL))]
                    sd = time_chain_graph(dev, cd * ncall, warmup, reps) / ncall
                    out[key]["dense_same_shape"] = {"us": sd * 1e6, "TOPS": 2.0 * M * N * K / sd / 1e12,
                                                    "kernel": bl.last_kernel()}
                    out[key]["speedup_vs_dense"] = sd / sec
                    del wd, ce, cd
                del cps, calls, x, ws, y
    assert bl.device_status() == 0
    return out


def run_lut(dev, warmup: int = 3, reps: int = 5):
    """Decode GEMV with dp4a against the TL2-style lookup-table variant, gate and down at M = 1
    (PDL-chained graphs calling each of > 2 x L2 of weight copies once)."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth

    out = {}
    for name, K, N in (("gate", 2560, 6912), ("down", 6912, 2560)):
        T = torch.from_numpy(synth.ternary_weights(N, K, seed=8)).to(dev)
        w = bl.pack_ternary(T, float(synth.alpha_uniform(8)))
        del T
        cps = _copies(w, w.nbytes)
        x = torch.from_numpy(synth.activations(1, K, seed=8).view(np.int16)).to(dev).view(torch.bfloat16)
        y = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
        nbytes = N * K // 4 + 4 + 2 * K + 2 * N
        row = {}
        for label, fl in (("dp4a", bl.FLAG_PDL), ("lut", bl.FLAG_PDL | bl.FLAG_DECODE_LUT)):
            calls = [(lambda ww=c, f=fl: bl.forward(ww, x, out=y, flags=f)) for c in cps]
            sec = time_chain_graph(dev, calls, warmup, reps) / len(calls)
            row[label] = {"us": sec * 1e6, "GBps": nbytes / sec / 1e9}
        out[f"{name} {K}->{N}"] = row
        del cps
    assert bl.device_status() == 0
    return out


def run_isolated(dev, iters: int = 30, warmup: int = 3):
    """Latency of one isolated forward call at M = 1 (gate 2560 -> 6912, down 6912 -> 2560): per
    iteration a 256 MB L2-flushing write, then one eager call without PDL between two CUDA events
    on the launching stream; median over `iters` (launch latency included, no graph)."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    s = torch.cuda.current_stream(dev)
    out = {}
    for name, K, N in (("gate", 2560, 6912), ("down", 6912, 2560)):
        T = torch.from_numpy(synth.ternary_weights(N, K, seed=9)).to(dev)
        w = bl.pack_ternary(T, float(synth.alpha_uniform(9)))
        del T
        x = torch.from_numpy(synth.activations(1, K, seed=9).view(np.int16)).to(dev).view(torch.bfloat16)
        y = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
        for _ in range(warmup):
            bl.forward(w, x, out=y, flags=0)
        ts = []
        for _ in range(iters):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            bl.forward(w, x, out=y, flags=0)
            e1.record(s)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1) / 1e3)
        sec = statistics.median(ts)
        nbytes = N * K // 4 + 4 + 2 * K + 2 * N
        out[f"{name} {K}->{N}"] = {"us": sec * 1e6, "GBps": nbytes / sec / 1e9, "kernel": bl.last_kernel()}
    assert bl.device_status() == 0
    return out


def run_hbit(dev, warmup: int = 3, reps: int = 5, calls: int = 16):
    """H-BitLinear (Hadamard transform + 4-bit codes + the tensor-core GEMM) on the 2B4T FFN shapes at
    M = 1 (chained over > 2 x L2 of weight copies) and M = 2048, against the 8-bit forward of the same
    call; and the transform-and-quantise kernel alone (GB/s on 2MK read + MK written + 8M)."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth

    out = {}
    for name, K, N in (("gate", 2560, 6912), ("down", 6912, 2560)):
        T = torch.from_numpy(synth.ternary_weights(N, K, seed=14)).to(dev)
        w = bl.pack_ternary(T, float(synth.alpha_uniform(14)))
        del T
        for M in (1, 2048):
            x = torch.from_numpy(synth.activations(M, K, seed=14).view(np.int16)).to(dev).view(torch.bfloat16)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(bl.forward_workspace_bytes(M, N, K, bl.FLAG_PATH_TC), dtype=torch.uint8, device=dev)
            cps = _copies(w, w.nbytes) if M == 1 else [w]
            n = max(calls, len(cps))
            t_h = time_chain_graph(dev, [(lambda ww=cps[i % len(cps)]: bl.forward_hbit(ww, x, out=y, workspace=ws,
                                                                                        flags=bl.FLAG_PDL))
                                         for i in range(n)], warmup, reps) / n
            kern = bl.last_kernel()
            t_8 = time_chain_graph(dev, [(lambda ww=cps[i % len(cps)]: bl.forward(ww, x, out=y, workspace=ws,
                                                                                   flags=bl.FLAG_PDL))
                                         for i in range(n)], warmup, reps) / n
            lib = bl.lib()
            q = torch.empty((M, K), dtype=torch.int8, device=dev)
            gm = torch.empty(M, dtype=torch.float32, device=dev)
            qcall = (lambda: lib.bitlinear_hadamard_quant_act4(x.data_ptr(), M, K, q.data_ptr(), gm.data_ptr(), None,
                                                               torch.cuda.current_stream(dev).cuda_stream))
            t_q = time_chain_graph(dev, [qcall] * calls, warmup, reps) / calls
            out[f"{name} {K}->{N} M={M}"] = {
                "forward_hbit_us": t_h * 1e6, "forward_hbit_TOPS": 2.0 * M * N * K / t_h / 1e12,
                "forward_hbit_GBps": (w.nbytes + 4 + 2 * M * K + 2 * M * N) / t_h / 1e9, "kernel": kern,
                "forward_8bit_us": t_8 * 1e6, "hadamard_quant_act4_us": t_q * 1e6,
                "hadamard_quant_act4_GBps": (3 * M * K + 8 * M) / t_q / 1e9, "weight_copies": len(cps)}
            del cps, x, y, ws, q, gm
    assert bl.device_status() == 0
    return out


def run_norm(dev, warmup: int = 3, reps: int = 5, calls: int = 16):
    """RMSNorm fused into the activation quantisation: the fused kernel alone (GB/s) and
    forward_norm against forward on the 2B4T gate shape (2560 -> 6912), PDL-chained graphs."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth

    K, N = 2560, 6912
    T = torch.from_numpy(synth.ternary_weights(N, K, seed=6)).to(dev)
    w = bl.pack_ternary(T, float(synth.alpha_uniform(6)))
    del T
    g = torch.from_numpy((0.5 + synth.uniform(6, 11, K)).astype(np.float32)).to(dev)
    out = {}
    for M in (1, 16, 2048):
        x = torch.from_numpy(synth.activations(M, K, seed=6).view(np.int16)).to(dev).view(torch.bfloat16)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(bl.forward_workspace_bytes(M, N, K, bl.FLAG_PATH_TC), dtype=torch.uint8, device=dev)
        q = torch.empty((M, K), dtype=torch.int8, device=dev)
        gm = torch.empty(M, dtype=torch.float32, device=dev)
        lib = bl.lib()
        qcall = (lambda: lib.bitlinear_rmsnorm_quant_act(x.data_ptr(), M, K, g.data_ptr(), 1e-5, q.data_ptr(),
                                                         gm.data_ptr(), None, torch.cuda.current_stream(dev).cuda_stream))
        t_q = time_chain_graph(dev, [qcall] * calls, warmup, reps) / calls
        t_fn = time_chain_graph(dev, [lambda: bl.forward_norm(w, x, g, 1e-5, out=y, workspace=ws,
                                                              flags=bl.FLAG_PDL)] * calls, warmup, reps) / calls
        t_f = time_chain_graph(dev, [lambda: bl.forward(w, x, out=y, workspace=ws, flags=bl.FLAG_PDL)]
                               * calls, warmup, reps) / calls
        out[f"M={M}"] = {"rmsnorm_quant_act_us": t_q * 1e6,
                         "rmsnorm_quant_act_GBps": (2 * M * K + M * K + 4 * K + 8 * M) / t_q / 1e9,
                         "forward_norm_us": t_fn * 1e6, "forward_us": t_f * 1e6,
                         "forward_norm_TOPS": 2.0 * M * N * K / t_fn / 1e12}
    assert bl.device_status() == 0
    return out


# ------------------------------------------------------------------ oracle (CPU) legs

def host_cpu():
    """CPU model, threads the system reports online, and threads this process may run on."""
    import oracle
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count() or 1
    return {"model": model, "online_cpus": oracle.online_cpus(), "usable_threads": usable}


def oracle_decode_setup(seed: int = 1):
    from ternary_weight_linear_fwd_b200 import synth
    mats = []
    for j, (name, K, N) in enumerate(FFN):
        mats.append((synth.ternary_weights(N, K, seed=seed + j), synth.alpha_uniform(seed + j), K, N))
    x = synth.activations(1, 2560, seed=seed, outlier_p=0.0)
    h = synth.activations(1, 6912, seed=seed + 1, outlier_p=0.0)
    return mats, x, h


def oracle_decode_pass(setup, frac: float = 1.0, threads: int = 1):
    """Oracle forward (quantise, contract, dequantise) of one FFN layer at M = 1, on the first
    `frac` of each matrix's output rows.  Returns (algorithmic bytes, seconds)."""
    import oracle
    mats, x, h = setup
    nbytes, t0 = 0, time.perf_counter()
    for T, a, K, N in mats:
        rows = max(1, int(round(N * frac)))
        oracle.forward(x if K == 2560 else h, T[:rows], a, threads=threads)
        nbytes += decode_bytes_per_gemv(K, rows)
    return nbytes, time.perf_counter() - t0


def oracle_decode_sample(seconds: float, threads: int, setup=None, seed: int = 1):
    """Repeats full-layer oracle passes until `seconds` pass; returns (GB/s, passes, seconds)."""
    setup = setup or oracle_decode_setup(seed)
    n, tot_b, tot_s = 0, 0, 0.0
    while tot_s < seconds:
        b, sec = oracle_decode_pass(setup, threads=threads)
        n, tot_b, tot_s = n + 1, tot_b + b, tot_s + sec
    return tot_b / tot_s / 1e9, n, tot_s


ORACLE_SLICE = 64  # tokens the oracle runs for the many-token workloads (time scaled linearly in M)


def _oracle_tokens(x_bits, Wt, alpha, threads):
    """Seconds of one oracle forward (quantise, contract, dequantise) of the given tokens."""
    import oracle
    t0 = time.perf_counter()
    oracle.forward(x_bits, Wt, alpha, threads=threads)
    return time.perf_counter() - t0


def run_cpu_baselines(decode_seconds: float, threads: int, with_sweep: bool):
    """The oracle, as it stands, on the host: the decode workload on one core and on `threads` cores, the
    prefill shapes, and (with_sweep) the layer sweep and the N:M shapes.  Many-token workloads run a
    slice of ORACLE_SLICE tokens and scale the time linearly to the full M (stated in each object)."""
    import numpy as np

    import oracle
    from ternary_weight_linear_fwd_b200 import synth
    cpu = host_cpu()
    setup = oracle_decode_setup()
    v1, n1, s1 = oracle_decode_sample(decode_seconds / 2, 1, setup)
    vt, nt, st = oracle_decode_sample(decode_seconds / 2, threads, setup)
    out = {"host": cpu, "decode": {
        "single_core": {"value": v1, "unit": "GB/s", "cores": 1, "passes": n1, "seconds": s1},
        "all_cores": {"value": vt, "unit": "GB/s", "cores": threads, "passes": nt, "seconds": st}}}

    def many_tokens(mats, M, seed):
        """mats: (key, K, N, Wt, alpha).  Per matrix the scaled oracle time of M tokens."""
        res, ops_tot, sec_tot = {}, 0.0, 0.0
        for key, K, N, Wt, alpha in mats:
            rows = min(M, ORACLE_SLICE)
            x = synth.activations(rows, K, seed=seed)
            sec = _oracle_tokens(x, Wt, alpha, threads) * M / rows
            ops = 2.0 * M * N * K
            res[key] = {"ms_scaled": sec * 1e3, "TOPS": ops / sec / 1e12,
                        "GBps": (N * K // 4 + 4 + 2 * M * K + 2 * M * N) / sec / 1e9}
            ops_tot, sec_tot = ops_tot + ops, sec_tot + sec
        return res, ops_tot, sec_tot

    mats = []
    for K, N in PREFILL_SHAPES:
        r = oracle.pack_weights(synth.latent_weights(N, K, seed=3))
        mats.append((f"{K}x{N}", K, N, r["Wt"], r["alpha"]))
    res, ops, sec = many_tokens(mats, PREFILL_M, 3)
    del mats
    out["prefill"] = {"value": ops / sec / 1e12, "unit": "TOPS", "cores": threads, "kind": "oracle",
                      "shapes": res,
                      "sample": f"oracle forward of {ORACLE_SLICE} of the {PREFILL_M} tokens per shape on "
                                f"{threads} threads, time scaled linearly to {PREFILL_M} tokens"}
    if with_sweep:
        layer = []
        for i, (name, (K, N)) in enumerate(synth.B2B4T_LAYER.items()):
            layer.append((name, K, N, synth.ternary_weights(N, K, seed=4 + 10 * i),
                          np.float32(synth.alpha_uniform(4 + 10 * i))))
        sweep = {}
        for M in SWEEP_M:
            res, ops, sec = many_tokens(layer, M, 4)
            nbytes = sum(N * K // 4 + 4 + 2 * M * K + 2 * M * N for _, K, N, _, _ in layer)
            sweep[f"M={M}"] = {"layer_us_scaled": sec * 1e6, "GBps": nbytes / sec / 1e9, "TOPS": ops / sec / 1e12,
                               "tokens_run": min(M, ORACLE_SLICE), "matrices": res}
        del layer
        out["sweep"] = {"cores": threads, "kind": "oracle", "by_M": sweep,
                        "sample": f"oracle forward of min(M, {ORACLE_SLICE}) tokens through the 7 matrices on "
                                  f"{threads} threads, time scaled linearly to M"}
        nm = {}
        for n, m in NM_PATTERNS:
            for name, (K, N) in synth.QWEN25_3B_MLP.items():
                r = oracle.pack_weights(synth.latent_weights(N, K, seed=5), n, m)
                nbytes_w = r["values"].size + r["meta"].size
                for M in NM_M:
                    rows = min(M, ORACLE_SLICE)
                    x = synth.activations(rows, K, seed=5)
                    sec = _oracle_tokens(x, r["Wt"], r["alpha"], threads) * M / rows
                    nm[f"{n}:{m} {name} {K}->{N} M={M}"] = {
                        "us_scaled": sec * 1e6, "GBps": (nbytes_w + 4 + 2 * M * K + 2 * M * N) / sec / 1e9,
                        "TOPS_dense_equiv": 2.0 * M * N * K / sec / 1e12, "tokens_run": rows}
        out["nm"] = {"cores": threads, "kind": "oracle", "cases": nm,
                     "sample": f"oracle forward (the masked ternary matrix, dense loop) of min(M, {ORACLE_SLICE}) "
                               f"tokens on {threads} threads, time scaled linearly to M"}
    return out


# ------------------------------------------------------------------ profiling cases

def _case_few_token(dev):
    """bitlinear_forward at M = 16 on a 2560 x 2560 ternary matrix: the fused few-token kernel."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth
    w = bl.pack_ternary(torch.from_numpy(synth.ternary_weights(2560, 2560, seed=1)).to(dev), 0.03)
    x = torch.from_numpy(synth.activations(16, 2560, seed=2).view(np.int16)).to(dev).view(torch.bfloat16)
    for _ in range(3):
        bl.forward(w, x)


def _case_hbit_m1(dev):
    """bitlinear_hadamard_quant_act4 on one 2560-wide token."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth
    x = torch.from_numpy(synth.activations(1, 2560, seed=4).view(np.int16)).to(dev).view(torch.bfloat16)
    for _ in range(3):
        bl.hadamard_quant_act4(x)


def _case_sparse24_m2048(dev):
    """bitlinear_forward_nm at M = 2048 on the Qwen2.5-3B up projection (2048 -> 11008) pruned 2:4:
    quantisation in natural K order, then the structured-sparse tensor-core GEMM."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth
    W = torch.from_numpy(synth.latent_weights(11008, 2048, seed=5)).to(dev)
    w = bl.pack_weights(W, 2, 4)
    del W
    x = torch.from_numpy(synth.activations(2048, 2048, seed=5).view(np.int16)).to(dev).view(torch.bfloat16)
    for _ in range(3):
        bl.forward_nm(w, x)


def _case_pair_gemm_m2048(dev):
    """bitlinear_forward_q8 (the GEMM alone, codes quantised first) at M = 2048 on the 2B4T gate projection
    2560 -> 6912: the pair GEMM (tcgen05 cta_group::2)."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth
    W = torch.from_numpy(synth.latent_weights(6912, 2560, seed=3)).to(dev)
    w = bl.pack_weights(W)
    del W
    x = torch.from_numpy(synth.activations(2048, 2560, seed=3).view(np.int16)).to(dev).view(torch.bfloat16)
    q, g, rs = bl.quant_act(x)
    for _ in range(3):
        bl.forward_q8(w, q, g, rs)


def _case_pair_gemm_wide_m2048(dev):
    """bitlinear_forward_q8 at M = 2048 on the 2B4T down projection 6912 -> 2560: the pair GEMM with a
    160-token tile (expanded codes in shared memory, A of the MMA from shared memory)."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth
    W = torch.from_numpy(synth.latent_weights(2560, 6912, seed=3)).to(dev)
    w = bl.pack_weights(W)
    del W
    x = torch.from_numpy(synth.activations(2048, 6912, seed=3).view(np.int16)).to(dev).view(torch.bfloat16)
    q, g, rs = bl.quant_act(x)
    for _ in range(3):
        bl.forward_q8(w, q, g, rs)


def _case_n8_gemm_m2048(dev):
    """bitlinear_forward_q8 at M = 2048 on the 2B4T gate projection 2560 -> 6912 pruned 6:8: the pair GEMM
    expanding kept codes and masks to dense codes (224-token tiles)."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth
    W = torch.from_numpy(synth.latent_weights(6912, 2560, seed=3)).to(dev)
    w = bl.pack_weights(W, 6, 8)
    del W
    x = torch.from_numpy(synth.activations(2048, 2560, seed=3).view(np.int16)).to(dev).view(torch.bfloat16)
    q, g, rs = bl.quant_act(x)
    for _ in range(3):
        bl.forward_q8(w, q, g, rs)


def _case_prefill_forward_m2048(dev):
    """bitlinear_forward (quantisation launch + GEMM) at M = 2048 on the 2B4T gate projection 2560 -> 6912."""
    import numpy as np
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import synth
    W = torch.from_numpy(synth.latent_weights(6912, 2560, seed=3)).to(dev)
    w = bl.pack_weights(W)
    del W
    x = torch.from_numpy(synth.activations(2048, 2560, seed=3).view(np.int16)).to(dev).view(torch.bfloat16)
    for _ in range(3):
        bl.forward(w, x)


PROFILE_CASES = {"few_token_m16": _case_few_token, "hbit_m1": _case_hbit_m1, "sparse24_m2048": _case_sparse24_m2048,
                 "pair_gemm_m2048": _case_pair_gemm_m2048, "pair_gemm_wide_m2048": _case_pair_gemm_wide_m2048,
                 "n8_gemm_m2048": _case_n8_gemm_m2048,
                 "prefill_forward_m2048": _case_prefill_forward_m2048}


def run_profile_case(name: str):
    import torch

    import ternary_weight_linear_fwd_b200 as bl
    from ternary_weight_linear_fwd_b200 import build as blbuild
    blbuild.build()
    dev = torch.device("cuda", 0)
    PROFILE_CASES[name](dev)
    torch.cuda.synchronize(dev)
    if bl.device_status() != 0:
        raise SystemExit(f"{name}: device status word set")
    print(f"{name}: ok, last kernel {bl.last_kernel()}")


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--prefill-iters", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the layer sweep and the N:M objects")
    ap.add_argument("--case", choices=sorted(PROFILE_CASES),
                    help="run one small profiling case (three calls of one kernel) and exit: the target of the "
                         "ncu captures summarised under profiles/")
    args = ap.parse_args()
    if args.case:
        run_profile_case(args.case)
        return
    if args.warmup < 3:
        raise SystemExit("at least 3 warm-up steps")

    world, rank, local = dist_env()
    config = {"workload": f"decode GEMV, BitNet-2B4T FFN (gate/up 2560->6912, down 6912->2560) x {args.layers} "
                          f"layers, M=1, ternary P(0)=0.42",
              "M": 1, "layers": args.layers, "matrices_per_step": 3 * args.layers,
              "gemv_launches_per_step": 2 * args.layers,
              "bytes_per_step": decode_step_bytes(args.layers), "l2": "weights per step exceed L2 (no reuse)",
              "parallelism": f"replicas x{world}"}

    if args.impl == "reference":
        if rank != 0:
            return
        threads = host_cpu()["usable_threads"]
        setup = oracle_decode_setup()
        full_b, full_s = oracle_decode_pass(setup, threads=threads)
        # a bounded sample per step: the whole run stays near two minutes of host time
        frac = min(1.0, (120.0 / (args.steps + args.warmup)) / full_s)
        for _ in range(args.warmup):
            oracle_decode_pass(setup, frac, threads)
        tot_b, tot_s, vals = 0, 0.0, []
        for _ in range(args.steps):
            b, sec = oracle_decode_pass(setup, frac, threads)
            tot_b, tot_s = tot_b + b, tot_s + sec
            vals.append(b / sec / 1e9)
        v = tot_b / tot_s / 1e9
        cpu = host_cpu()
        sample = (f"oracle forward (plain C; contraction over {threads} threads): per step one FFN layer (gate, "
                  f"up, down at M=1) restricted to the first {frac:.4f} of each matrix's output rows; GB/s on "
                  f"the same algorithmic bytes (packed codes + alpha + x + y); host {cpu['model']}, "
                  f"{cpu['online_cpus']} threads online")
        line = {"metric": METRIC, "impl": "reference", "value": v, "unit": "GB/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "int8 x ternary -> int32 (bf16 in/out)", "data": "synthetic", "config": config,
                "cpu_baseline": {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample,
                                 "host": cpu},
                "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist

    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    from ternary_weight_linear_fwd_b200 import build as blbuild
    blbuild.build()
    import ternary_weight_linear_fwd_b200 as bl
    bl.lib()

    dec = run_decode(dev, args.steps, args.warmup, args.layers, clock_index=local)
    max_secs = reduce_max(dec["secs"], dev)
    max_e2e = reduce_max(dec["e2e_secs"], dev)
    step_bytes = decode_step_bytes(args.layers)
    value = aggregate(step_bytes, args.steps, world, max_secs) / 1e9
    e2e_value = aggregate(step_bytes, dec["e2e_steps"], world, max_e2e) / 1e9

    pre = run_prefill(dev, args.prefill_iters, 3)
    iso = run_isolated(dev)
    sweep = nm = norm = lut = hbit = ffn = None
    if not args.no_sweep:
        ffn = run_ffn_glu(dev, args.layers)
        sweep = run_sweep(dev)
        nm = run_nm(dev)
        norm = run_norm(dev)
        lut = run_lut(dev)
        hbit = run_hbit(dev)

    if world > 1:
        barrier(dev)
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_kind = measured_peaks()
    # the step holds nothing but GEMV launches: average launch = step time / launches
    per_launch = dec["secs"] / (args.steps * dec["launches_per_step"])
    launch_bytes = step_bytes / dec["launches_per_step"]
    achieved = launch_bytes / per_launch / 1e9
    traffic = profiled_traffic()
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "kernel": "gemv_m1_dense",
                "peak_source": f"{peak_kind} hbm_gbs"}
    int8_peak = 2.0 * peaks["bf16_tflops"]
    prefill = {"metric": "prefill int8 TOPS (GEMM kernel)", "value": pre["gemm_tops"], "unit": "TOPS",
               "forward_tops": pre["tops"],
               "how": "value / roofline: the tensor-core GEMM kernel alone, bitlinear_forward_q8 on codes quantised "
                      "before the timed region; forward_tops: the whole bitlinear_forward call (activation "
                      "quantisation launch + GEMM), the same rotation of copies",
               "workload": f"2B4T prefill M={PREFILL_M}: " + ", ".join(f"{k}->{n}" for k, n in PREFILL_SHAPES),
               "shapes": pre["shapes"], "kernel": pre["kernel"],
               "l2": "inputs larger than L2: each call reads its own copy of x and of the packed weights "
                     "(copies > 2 x L2 per shape), PDL-chained graph; flushed_tops: a 256 MB write before each "
                     "call instead, device time of (flush, forward) graph replays minus flush-only replays",
               "flushed_tops": pre["flushed_tops"],
               "roofline": {"bound": "tensor", "achieved": pre["gemm_tops"], "peak": int8_peak, "unit": "TOPS",
                            "frac": pre["gemm_tops"] / int8_peak,
                            "kernel": " / ".join(sorted({v["gemm_kernel"] for v in pre["shapes"].values()})),
                            "forward_frac": pre["tops"] / int8_peak,
                            "peak_source": f"{peak_kind} bf16_tflops x 2 (int8/bf16 nominal ratio)"}}
    cpu = cpu_all = None
    if not args.no_cpu_baseline:
        threads = host_cpu()["usable_threads"]
        cpu_all = run_cpu_baselines(args.cpu_seconds, threads, sweep is not None)
        d = cpu_all["decode"]
        h = cpu_all["host"]
        cpu = {"value": d["all_cores"]["value"], "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"oracle forward (plain C; contraction over {threads} threads, quantisation and rescale "
                         f"on one) on one FFN layer (gate, up, down at M=1), {d['all_cores']['passes']} passes "
                         f"in {d['all_cores']['seconds']:.1f} s; host {h['model']}, {h['online_cpus']} threads "
                         f"online",
               "single_core": d["single_core"], "host": h}
        prefill["cpu_baseline"] = cpu_all["prefill"]
    e2e = {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": dec["h2d"],
           "d2h_bytes_per_step": dec["d2h"], "steps": dec["e2e_steps"],
           "how": "each step: pinned-host copies of every layer's inputs, the captured decode step (CUDA graph "
                  "of the public-API calls), copies of every output back",
           "eager": {"value": dec["e2e_eager_gbps"], "unit": "GB/s", "steps": dec["e2e_eager_steps"],
                     "ms_per_step": dec["e2e_eager_ms"],
                     "how": "the same step issued call by call through the Python binding and the C ABI "
                            "(argument checks, cached tensor maps, 60 launches), no graph"}}
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_secs / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8 x ternary -> int32 (bf16 in/out)",
            "data": "synthetic", "config": config, "roofline": roofline, "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps * dec["launches_per_step"], "clocks": dec["clocks"],
            "hbm_frac": value / world / peaks["hbm_gbs"], "prefill": prefill,
            "isolated": {"workload": "one forward call at M=1 on a cold L2 (256 MB write before it), eager, "
                                     "no PDL, CUDA events around the call (launch latency included); median of "
                                     "30; bytes = N*K/4 + 4 + 2K + 2N", "cases": iso}}
    if sweep is not None:
        line["sweep"] = {"workload": "2B4T layer's 7 BitLinears (q,k,v,o 2560->2560/640, gate/up 2560->6912, "
                                     "down 6912->2560), ternary P(0)=0.42; per matrix a PDL-chained graph "
                                     "calling each of its weight copies once (> 2 x L2 of weights); bytes = "
                                     "N*K/4 + 4 + 2MK + 2MN, ops = 2MNK", "by_M": sweep}
        line["nm"] = {"workload": "Sparse-BitNet N:M on Qwen2.5-3B MLP (2048->11008, 11008->2048), latent "
                                  "W ~ N(0,0.02); PDL-chained graph (M=1: each of > 2 x L2 of weight copies once; "
                                  "M=4096: 16 calls); "
                                  "bytes = packed values + metadata + 4 + 2MK + 2MN; TOPS counts dense-equivalent "
                                  "2MNK", "cases": nm}
        line["ffn_glu"] = {"workload": f"decode FFN stack with its dataflow, {args.layers} layers at M=1: "
                                       "h = ReLU(gate x)^2 * (up x) in one launch (bitlinear_forward_relu2_glu), "
                                       "then down(h); one CUDA graph with PDL edges; bytes = the decode step's "
                                       "weights + x + h + y", **ffn}
        line["norm"] = {"workload": "RMSNorm (fp32 weight, eps 1e-5) fused into the activation quantisation, "
                                    "2B4T gate 2560->6912, ternary P(0)=0.42; PDL-chained graphs of 16 calls; "
                                    "rmsnorm_quant_act bytes = 2MK (x) + MK (q) + 4K (g) + 8M; forward_norm vs "
                                    "forward (M=1: normalising quantisation + GEMV on the codes vs the GEMV "
                                    "quantising in-kernel; M>1: tensor-core path)", "by_M": norm}
        line["decode_lut"] = {"workload": "decode GEMV at M=1, dp4a against per-pair lookup tables (TL2 idea), "
                                          "ternary P(0)=0.42; PDL-chained graphs over > 2 x L2 of weight copies",
                              "cases": lut}
        line["hbit"] = {"workload": "H-BitLinear (Hadamard transform of each token row, 4-bit codes, tcgen05 "
                                    "GEMM, rescale by alpha*gamma/7) on 2B4T gate/down, ternary P(0)=0.42; "
                                    "PDL-chained graphs (M=1: > 2 x L2 of weight copies); the 8-bit forward of "
                                    "the same call beside it", "cases": hbit}
        if cpu_all is not None:
            line["sweep"]["cpu_baseline"] = cpu_all["sweep"]
            line["nm"]["cpu_baseline"] = cpu_all["nm"]
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
