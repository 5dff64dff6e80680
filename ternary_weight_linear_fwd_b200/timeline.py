"""Phase timeline of two launch chains, from the stamps of the test build.

    python -m ternary_weight_linear_fwd_b200.timeline

Builds ``libbitlinear_testhooks.so`` (the product sources with
-DBITLINEAR_TEST_HOOKS; see include/bitlinear_test_hooks.h), runs

* the decode step of a 30-layer BitNet-2B4T FFN stack at one token (per layer
  the grouped gate/up GEMV, then the down GEMV; one CUDA graph with
  programmatic-dependent-launch edges), and
* a chain of 40 calls of the pair GEMM alone (bitlinear_forward_q8) at
  M = 256 on the 2B4T gate projection 2560 -> 6912, one graph,

reads every CTA's record and prints one JSON object: per launch kind, the
median over launches of each phase (ns).  The stamps, the ring writes and
the extra registers make the test build a little slower than the product one; the
phase split, not the absolute time, is what it is for.
"""
from __future__ import annotations

import ctypes
import json
import statistics

import numpy as np

LAYERS = 30
GEMV_PHASES = ["dependency_wait_returned", "x_quantised", "weights_landed", "contracted", "stored"]
PAIR_PHASES = ["set_up", "producer_past_wait", "first_stage_landed", "first_tile_mmas_issued",
               "first_accumulator_ready", "last_epilogue_done", "end"]


def _clear(L):
    if L.bitlinear_test_timeline(None, 0) < 0:
        raise RuntimeError("bitlinear_test_timeline failed")


def _read(L):
    buf = (ctypes.c_uint64 * (10 * (1 << 17)))()
    n = L.bitlinear_test_timeline(buf, 1 << 17)
    if n < 0:
        raise RuntimeError("bitlinear_test_timeline failed")
    if n > (1 << 17):
        raise RuntimeError("timeline ring overflowed; time fewer launches")
    return np.frombuffer(buf, dtype=np.uint64).reshape(-1, 10)[:n].astype(np.int64)


def _launches(rec, end_col):
    """Records grouped into launches: sorted by their end stamp, a launch is gridDim consecutive
    records with the same first launch fact (K or M).  A launch ends before the next one's CTAs do,
    since each waits for its predecessor to complete."""
    rec = rec[np.argsort(rec[:, end_col], kind="stable")]
    grid, key = rec[:, 1] & 0xFFFF, rec[:, 1] >> 32
    out, cur = [], []
    for i in range(len(rec)):
        if cur and (key[i] != key[cur[0]] or len(cur) >= grid[cur[0]]):
            out.append(rec[cur])
            cur = []
        cur.append(i)
    if cur:
        out.append(rec[cur])
    return out


def _gemv_summary(rec):
    """Per K (the two launch shapes of the step): medians over launches of each phase of thread 0
    (median over the launch's CTAs), of the time from the previous launch's last store to this
    launch's first return from the dependency wait, and of the launch period."""
    rows = {}
    prev_end = None
    for L in _launches(rec, end_col=7):
        s = L[:, 2:8]  # entry, wait returned, x quantised, weights landed, contracted, stored
        row = {p: float(np.median(s[:, i + 1] - s[:, i])) for i, p in enumerate(GEMV_PHASES)}
        if prev_end is not None:
            row["previous_store_to_wait_return"] = float(s[:, 1].min() - prev_end)
            row["period"] = float(s[:, 5].max() - prev_end)
            rows.setdefault(int(L[0, 1] >> 32), []).append(row)
        prev_end = s[:, 5].max()
    return {f"K={k}": {p: statistics.median(r[p] for r in v) for p in v[0]} for k, v in rows.items()}


def _pair_summary(rec):
    """Medians over launches (first and last dropped) of each stamp's median over CTAs, relative to the
    CTA's entry, and of the spread of the CTAs' entries within a launch."""
    rows = []
    for L in _launches(rec, end_col=9)[1:-1]:
        s = L[:, 2:10]
        row = {}
        for i, p in enumerate(PAIR_PHASES):
            ok = s[:, i + 1] > 0
            if ok.any():
                row[p] = float(np.median(s[ok, i + 1] - s[ok, 0]))
        row["entry_spread"] = float(s[:, 0].max() - s[:, 0].min())
        rows.append(row)
    return {k: statistics.median(r[k] for r in rows if k in r) for k in rows[0]}


def main():
    import torch

    from . import build as blbuild
    from . import synth
    import ternary_weight_linear_fwd_b200 as bl

    bl._LIB_PATH = blbuild.build_test_hooks()
    bl._lib = None
    L = bl.lib()
    L.bitlinear_test_timeline.restype = ctypes.c_int32
    L.bitlinear_test_timeline.argtypes = [ctypes.c_void_p, ctypes.c_int32]
    dev = torch.device("cuda", 0)

    def graph_of(step):
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize(dev)
        return g

    # decode step: per layer the grouped gate/up GEMV on x, then the down GEMV on h
    ffn = [("gate", 2560, 6912), ("up", 2560, 6912), ("down", 6912, 2560)]
    layers = []
    for l in range(LAYERS):
        mats = {}
        for j, (name, K, N) in enumerate(ffn):
            T = torch.from_numpy(synth.ternary_weights(N, K, seed=1 + 100 * (l % 4) + j)).to(dev)
            mats[name] = bl.pack_ternary(T, float(synth.alpha_uniform(1 + j)))
            del T
        layers.append(mats)
    x = torch.from_numpy(synth.activations(LAYERS, 2560, seed=1).view(np.int16)).to(dev).view(torch.bfloat16)
    h = torch.from_numpy(synth.activations(LAYERS, 6912, seed=2).view(np.int16)).to(dev).view(torch.bfloat16)
    yg = torch.empty((LAYERS, 6912), dtype=torch.bfloat16, device=dev)
    yu = torch.empty_like(yg)
    yd = torch.empty((LAYERS, 2560), dtype=torch.bfloat16, device=dev)

    def decode_step():
        for l, w in enumerate(layers):
            bl.forward_group([w["gate"], w["up"]], x[l:l + 1], outs=[yg[l:l + 1], yu[l:l + 1]], flags=bl.FLAG_PDL)
            bl.forward(w["down"], h[l:l + 1], out=yd[l:l + 1], flags=bl.FLAG_PDL)

    g = graph_of(decode_step)
    _clear(L)
    for _ in range(2):
        g.replay()
    rec = _read(L)
    decode = _gemv_summary(rec[rec[:, 0] == 1])
    del g, layers

    # the pair GEMM alone at M = 256 on 40 copies of the gate projection
    M, K, N = 256, 2560, 6912
    T = torch.from_numpy(synth.ternary_weights(N, K, seed=3)).to(dev)
    w = bl.pack_ternary(T, 0.03)
    del T
    cps = [bl.PackedWeights(w.N, w.K, 0, 0, w.codes.clone(), None, w.alpha.clone()) for _ in range(40)]
    xq = torch.from_numpy(synth.activations(M, K, seed=3).view(np.int16)).to(dev).view(torch.bfloat16)
    q, gm, rs = bl.quant_act(xq)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

    def pair_chain():
        for c in cps:
            bl.forward_q8(c, q, gm, rs, out=y, flags=bl.FLAG_PDL)

    g = graph_of(pair_chain)
    _clear(L)
    g.replay()
    rec = _read(L)
    pair = _pair_summary(rec[rec[:, 0] == 2])
    kernel = bl.last_kernel()
    del g
    if bl.device_status() != 0:
        raise SystemExit("device status word set")
    print(json.dumps({"build": "test hooks (phase stamps)", "decode_step_gemv_ns_median": decode,
                      "pair_gemm_m256_ns_median_from_cta_entry": pair, "pair_kernel": kernel}, indent=1))


if __name__ == "__main__":
    main()
