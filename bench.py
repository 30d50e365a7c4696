#!/usr/bin/env python
"""Benchmark: ternary-g128 decode-step weight stream on B200.

One step = one synthetic decode token: 64 layers, each with the projections
q 5120->6144, k/v 5120->1024, o 6144->5120, gate/up 5120->17408,
down 17408->5120, plus a 5120->151936 output head; M = 1; all weights
ternary-g128 in 2-bit slots (6,000,015,360 bytes resident, far larger than
the 126 MB L2, so every step streams cold weights from HBM).  Every projection
gets its own fresh N(0,1) fp16 input, so all 449 products of a step are
independent and run as one tern_gemv_step call (five launches of at most 96
products, overlapped), captured in one CUDA graph.

The GPU idles REST_S seconds before each timed region: held back to back, the
step's HBM stream trips the power cap after ~60 ms and the SM clock drops to
~1.55 GHz.  The timed K steps therefore measure the burst rate, as the copy
that gives the roofline peak does, and "sustained" reports the same step
back to back once the cap has engaged.

Prints ONE JSON line (rank 0).  `--impl reference` times the fp64 CPU oracle
on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from ternary_weight_only_b200 import synth  # noqa: E402

GROUP = 128
METRIC = "ternary-g128 GEMV HBM GB/s (% of B200 peak); decode-step weight-stream ms"
BYTES_PER_WEIGHT = 0.25 + 2.0 / GROUP  # 2-bit slot + fp16 scale per 128
STEP_PER_LAUNCH = 96  # matrices one launch of the step kernel takes (tern_gemv_step splits longer lists)
REST_S = 1.0  # idle seconds before each timed region (see the device-timed steps)
SUSTAIN_LEAD, SUSTAIN_STEPS = 100, 200  # back-to-back steps before and inside the sustained timing


def wbytes(K, N):
    return N * K // 4 + N * (K // GROUP) * 2


def step_bytes():
    """Algorithmic bytes of one decode step: weights + activations in + outputs."""
    w = synth.N_LAYERS * sum(wbytes(K, N) for _, K, N in synth.LAYER_PROJ)
    w += wbytes(synth.HEAD[1], synth.HEAD[2])
    xin = synth.N_LAYERS * 2 * (5120 + 6144 + 17408) + 2 * synth.HEAD[1]
    yout = synth.N_LAYERS * 2 * sum(N for _, _, N in synth.LAYER_PROJ) + 2 * synth.HEAD[2]
    return w, xin, yout


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0) or 0), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """NVML SM clock + throttle reasons, polled in a thread while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.002):
        self.samples, self.reasons = [], 0
        self.period = period_s
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "tern" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif args.impl == "tern":
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, ws):
    if ws == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ model --
class DecodeModel:
    """The synthetic 64-layer decode weight set, packed on the GPU."""

    def __init__(self, T, device="cuda", n_layers=synth.N_LAYERS):
        self.T = T
        self.n_layers = n_layers
        self.layers = []  # per layer: list of (name, K, N, slots, scales)
        self.x_all = None
        for l in range(n_layers):
            g = synth.gen(4000 + l, device)
            mats = []
            for name, K, N in synth.LAYER_PROJ:
                codes = synth.codes_sparse(N, K, g, device=device)
                scales = synth.scales_uniform(N, K, g, device=device)
                slots, sc = T.tern_pack_g128(codes, scales)
                del codes
                mats.append((name, K, N, slots, sc))
            self.layers.append(mats)
        g = synth.gen(4000 + synth.N_LAYERS, device)  # head seed independent of n_layers
        _, K, N = synth.HEAD
        codes = synth.codes_sparse(N, K, g, device=device)
        scales = synth.scales_uniform(N, K, g, device=device)
        self.head = (synth.HEAD[0], K, N, *T.tern_pack_g128(codes, scales))
        del codes
        torch.cuda.synchronize()
        # Inputs: per layer x_h (q,k,v,gate,up), x_o (o), x_d (down); head input.
        per_layer = 5120 + 6144 + 17408
        self.x_all = torch.empty(n_layers * per_layer + 5120, dtype=torch.float16, device=device)
        g = synth.gen(5000, device)
        self.x_all.copy_(torch.randn(self.x_all.numel(), generator=g, device=device).half())
        yn = sum(N for _, _, N in synth.LAYER_PROJ)
        self.y_all = torch.empty(n_layers * yn + synth.HEAD[2], dtype=torch.float16, device=device)
        self.groups = []
        xo = yo = 0
        for l in range(n_layers):
            xh = self.x_all[xo:xo + 5120]
            xop = self.x_all[xo + 5120:xo + 5120 + 6144]
            xd = self.x_all[xo + 5120 + 6144:xo + per_layer]
            xo += per_layer
            grp = []
            for name, K, N, slots, sc in self.layers[l]:
                x = {"o": xop, "down": xd}.get(name, xh)
                y = self.y_all[yo:yo + N]
                yo += N
                grp.append((x, slots, sc, y))
            self.groups.append(grp)
        self.head_io = (self.x_all[xo:xo + 5120], self.y_all[yo:yo + synth.HEAD[2]])

    def all_mats(self):
        _, K, N, slots, sc = self.head
        return [m for grp in self.groups for m in grp] + [(self.head_io[0], slots, sc, self.head_io[1])]

    def step(self):
        """One decode step: every projection of every layer and the head in
        one tern_gemv_step call (the inputs are independent)."""
        self.T.tern_gemv_step(self.all_mats())

    def e2e_chunks(self, frac=(8 / 64, 60 / 64)):
        """The step's products in chunks of consecutive layers cut at the
        given fractions of the layer count, the head in the first chunk.  Only
        the first chunk's copy in and the last chunk's copy out are not hidden
        behind products, so both are small: the first chunk holds the head
        (10 KB of x; its 304 KB of y go back while the rest runs) and eight
        layers, the last four layers (0.4 MB of y).  Every further chunk costs
        a call boundary (~12 us), so there are three.  (Measured on B200 over
        ten cuttings: this one 1.407 ms per step end to end, five equal chunks
        with the head last 1.453 ms; the copies alone take 0.139 ms.)
        Returns (products, x ranges, y ranges), ranges as element offsets into
        x_all / y_all."""
        per_x = 5120 + 6144 + 17408
        per_y = sum(N for _, _, N in synth.LAYER_PROJ)
        L = self.n_layers
        _, K, N, slots, sc = self.head
        head = (self.head_io[0], slots, sc, self.head_io[1])
        hx = (L * per_x, L * per_x + 5120)
        hy = (L * per_y, L * per_y + N)
        cuts = [0] + [round(f * L) for f in frac] + [L]
        out = []
        for c in range(len(cuts) - 1):
            l0, l1 = cuts[c], cuts[c + 1]
            if l1 <= l0 and c != 0:
                continue
            mats = [m for grp in self.groups[l0:l1] for m in grp]
            xr = [(l0 * per_x, l1 * per_x)] if l1 > l0 else []
            yr = [(l0 * per_y, l1 * per_y)] if l1 > l0 else []
            if c == 0:
                mats = [head] + mats
                xr, yr = [hx] + xr, [hy] + yr
            out.append((mats, xr, yr))
        return out

    def step_per_layer(self):
        """The same step as one grouped launch per layer plus the head."""
        T = self.T
        for grp in self.groups:
            T.tern_gemv_grouped(grp, 1)
        _, K, N, slots, sc = self.head
        T.tern_gemv(self.head_io[0], slots, sc, self.head_io[1])

    @property
    def launches_per_step(self):
        n = len(self.all_mats())
        return (n + STEP_PER_LAUNCH - 1) // STEP_PER_LAUNCH


def cuda_time(fn, iters, stream=None):
    s = stream or torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(iters):
        fn()
    e1.record(s)
    e1.synchronize()
    return e0.elapsed_time(e1) / iters


def proj_rows(T, model, peak_gbs, l2_bytes):
    """Per-projection GB/s at M = 1 and M in {2,4,8}: each timed launch uses a
    different layer's copy of the projection (64 distinct weight buffers,
    rotating through far more than the L2 size), in a CUDA graph."""
    out = {}
    s = torch.cuda.Stream()
    names = [p[0] for p in synth.LAYER_PROJ]
    xbuf = torch.randn(8 * 17408, device="cuda").half()
    ybuf = torch.empty(8 * 17408, dtype=torch.float16, device="cuda")
    ybuf_l = [torch.empty(8 * N, dtype=torch.float16, device="cuda") for _, _, N in synth.LAYER_PROJ]
    for M in (1, 2, 4, 8):
        for i, name in enumerate(names):
            _, K, N = synth.LAYER_PROJ[i]
            x = xbuf[:M * K].view(M, K)
            y = ybuf[:M * N].view(M, N)
            mats = [model.layers[l][i] for l in range(synth.N_LAYERS)]
            if M == 1:
                fns = [lambda m=m: T.tern_gemv(x[0], m[3], m[4], y[0]) for m in mats]
            else:
                fns = [lambda m=m: T.tern_gemm(x, m[3], m[4], y) for m in mats]
            ms = graph_time(fns, s)
            b = wbytes(K, N) + 2 * M * K + 2 * M * N
            out[f"{name}_M{M}"] = {"us": round(ms * 1e3, 3), "GBps": round(b / ms / 1e6, 1),
                                   "frac": round(b / ms / 1e6 / peak_gbs, 4)}
    # grouped shapes at M = 1
    for label, idx in (("qkv", [0, 1, 2]), ("gate_up", [4, 5]), ("layer", list(range(7)))):
        x = xbuf
        fns = []
        for l in range(synth.N_LAYERS):
            grp = [model.groups[l][i] for i in idx]
            fns.append(lambda grp=grp: T.tern_gemv_grouped(grp, 1))
        ms = graph_time(fns, s)
        b = sum(wbytes(synth.LAYER_PROJ[i][1], synth.LAYER_PROJ[i][2]) +
                2 * synth.LAYER_PROJ[i][1] + 2 * synth.LAYER_PROJ[i][2] for i in idx)
        out[f"{label}_M1"] = {"us": round(ms * 1e3, 3), "GBps": round(b / ms / 1e6, 1),
                              "frac": round(b / ms / 1e6 / peak_gbs, 4)}
    # grouped layers at M = 2, 4, 8 (verify batch): one launch per layer
    for M in (2, 4, 8):
        fns = []
        for l in range(synth.N_LAYERS):
            grp = []
            for i, (x, slots, sc, y) in enumerate(model.groups[l]):
                K = synth.LAYER_PROJ[i][1]
                N = synth.LAYER_PROJ[i][2]
                grp.append((xbuf[:M * K].view(M, K), slots, sc, ybuf_l[i][:M * N].view(M, N)))
            fns.append(lambda grp=grp, M=M: T.tern_gemv_grouped(grp, M))
        ms = graph_time(fns, s)
        b = sum(wbytes(K, N) + 2 * M * K + 2 * M * N for _, K, N in synth.LAYER_PROJ)
        out[f"layer_M{M}"] = {"us": round(ms * 1e3, 3), "GBps": round(b / ms / 1e6, 1),
                              "frac": round(b / ms / 1e6 / peak_gbs, 4)}
    # the verify step: every projection of all layers at M = 2, 4, 8 token
    # rows, one tern_gemv_step call (5 launches; at M = 8 the down
    # projections, whose eight rows of x do not fit, run as two K segments)
    for M in (2, 4, 8):
        mats, b = [], 0
        for l in range(synth.N_LAYERS):
            for i, (x, slots, sc, y) in enumerate(model.groups[l]):
                K, N = synth.LAYER_PROJ[i][1], synth.LAYER_PROJ[i][2]
                mats.append((xbuf[:M * K].view(M, K), slots, sc,
                             torch.empty(M, N, dtype=torch.float16, device="cuda")))
                b += wbytes(K, N) + 2 * M * K + 2 * M * N
        ms = graph_time([lambda mats=mats, M=M: T.tern_gemv_step(mats, M)], s, reps=5)
        out[f"verify_step_M{M}"] = {"ms": round(ms, 4), "GBps": round(b / ms / 1e6, 1),
                                    "frac": round(b / ms / 1e6 / peak_gbs, 4),
                                    "products": len(mats)}
        del mats
    # one layer (seven projections) through the step kernel, rotating layers
    fns = [lambda grp=grp: T.tern_gemv_step(grp) for grp in model.groups]
    ms = graph_time(fns, s)
    b = sum(wbytes(K, N) + 2 * K + 2 * N for _, K, N in synth.LAYER_PROJ)
    out["layer_step_kernel_M1"] = {"us": round(ms * 1e3, 3), "GBps": round(b / ms / 1e6, 1),
                                   "frac": round(b / ms / 1e6 / peak_gbs, 4)}
    # the whole decode step as one grouped launch per layer plus the head
    wb, xin, yout = step_bytes()
    ms = graph_time([model.step_per_layer], s, reps=5)
    out["decode_step_per_layer_launches"] = {"ms": round(ms, 4), "GBps": round((wb + xin + yout) / ms / 1e6, 1),
                                             "frac": round((wb + xin + yout) / ms / 1e6 / peak_gbs, 4),
                                             "launches": model.n_layers + 1}
    _, K, N, slots, sc = model.head
    # 206 MB of head weights per call: larger than L2, streamed cold each replay
    ms = graph_time([lambda: T.tern_gemv(model.head_io[0], slots, sc, model.head_io[1])], s, reps=20)
    b = wbytes(K, N) + 2 * K + 2 * N
    out["head_M1"] = {"us": round(ms * 1e3, 3), "GBps": round(b / ms / 1e6, 1),
                      "frac": round(b / ms / 1e6 / peak_gbs, 4)}
    return out


def b1_rows(T, model, peak_gbs, sm_mhz=None):
    """The 1-bit variant ({-1,+1} + fp16 scale per 128, 1.125 bits/weight)
    over the same shapes: every projection of the 64 layers plus the head in
    one tern_b1_gemv_step call, at M = 1 (decode) and M = 2, 4 (verify).
    Weights are random signs; x and y are the decode model's buffers.  The
    unpack costs as many integer instructions per weight as the ternary one
    (one AND per pair of weights), over half the bytes, so the row also
    reports the fraction of the integer-pipe bound (alu_frac): 2 logic
    instructions per cycle per SM, 34 per 2048 weights."""
    out = {}
    s = torch.cuda.Stream()
    mats, bmats = [], 0
    for l in range(model.n_layers):
        g = synth.gen(6000 + l, "cuda")
        for i, (x, slots, sc, y) in enumerate(model.groups[l]):
            _, K, N = synth.LAYER_PROJ[i]
            codes = synth.codes_sign(N, K, g, device="cuda")
            bits, bsc = T.tern_b1_pack(codes, synth.scales_uniform(N, K, g, device="cuda"))
            del codes
            mats.append((x, bits, bsc, y, K, N))
    g = synth.gen(6000 + synth.N_LAYERS, "cuda")
    _, K, N = synth.HEAD
    codes = synth.codes_sign(N, K, g, device="cuda")
    bits, bsc = T.tern_b1_pack(codes, synth.scales_uniform(N, K, g, device="cuda"))
    del codes
    mats.append((model.head_io[0], bits, bsc, model.head_io[1], K, N))
    torch.cuda.synchronize()
    nweights = sum(K * N for *_, K, N in mats)
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    mhz = sm_mhz or 1800.0
    alu_weights_per_s = props.multi_processor_count * mhz * 1e6 * 2 / 34 * 2048
    xbuf = torch.randn(4 * 17408, device="cuda").half()
    for M in (1, 2, 4):
        if M == 1:
            run = [(x, b, sc, y) for x, b, sc, y, _, _ in mats]
        else:
            run = [(xbuf[:M * K].view(M, K), b, sc, torch.empty(M, N, dtype=torch.float16, device="cuda"))
                   for _, b, sc, _, K, N in mats]
        b = sum(N * K // 8 + 2 * N * (K // GROUP) + 2 * M * K + 2 * M * N for *_, K, N in mats)
        ms = graph_time([lambda run=run, M=M: T.tern_b1_gemv_step(run, M)], s, reps=5)
        wps = nweights / (ms * 1e-3)
        out[f"b1_step_M{M}"] = {"ms": round(ms, 4), "GBps": round(b / ms / 1e6, 1),
                                "frac": round(b / ms / 1e6 / peak_gbs, 4),
                                "weights_per_s": float(f"{wps:.4g}"),
                                "alu_frac": round(wps / alu_weights_per_s, 4),
                                "products": len(run)}
        del run
    del mats
    torch.cuda.empty_cache()
    return out


def t5_rows(T, model, peak_gbs):
    """Five trits per byte (26 bytes per 128-weight group, 1.75 bits/weight)
    over the same shapes and codes distribution as the decode step (P(0) =
    0.4): every projection of the 64 layers plus the head in one
    tern_t5_gemv_step call, at M = 1 and M = 2 (M = 4 does not fit beside
    the decode table at K = 17408).  weights_per_s compares the decode rate
    with the 2-bit slots' (decode_step in the main line)."""
    out = {}
    s = torch.cuda.Stream()
    mats = []
    for l in range(model.n_layers):
        g = synth.gen(7000 + l, "cuda")
        for i, (x, slots, sc, y) in enumerate(model.groups[l]):
            _, K, N = synth.LAYER_PROJ[i]
            codes = synth.codes_sparse(N, K, g, device="cuda")
            packed, psc = T.tern_t5_pack(codes, synth.scales_uniform(N, K, g, device="cuda"))
            del codes
            mats.append((x, packed, psc, y, K, N))
    g = synth.gen(7000 + synth.N_LAYERS, "cuda")
    _, K, N = synth.HEAD
    codes = synth.codes_sparse(N, K, g, device="cuda")
    packed, psc = T.tern_t5_pack(codes, synth.scales_uniform(N, K, g, device="cuda"))
    del codes
    mats.append((model.head_io[0], packed, psc, model.head_io[1], K, N))
    torch.cuda.synchronize()
    nweights = sum(K * N for *_, K, N in mats)
    xbuf = torch.randn(2 * 17408, device="cuda").half()
    for M in (1, 2):
        if M == 1:
            run = [(x, b, sc, y) for x, b, sc, y, _, _ in mats]
        else:
            run = [(xbuf[:M * K].view(M, K), b, sc, torch.empty(M, N, dtype=torch.float16, device="cuda"))
                   for _, b, sc, _, K, N in mats]
        b = sum(N * (26 * K // GROUP) + 2 * N * (K // GROUP) + 2 * M * K + 2 * M * N for *_, K, N in mats)
        ms = graph_time([lambda run=run, M=M: T.tern_t5_gemv_step(run, M)], s, reps=5)
        out[f"t5_step_M{M}"] = {"ms": round(ms, 4), "GBps": round(b / ms / 1e6, 1),
                                "frac": round(b / ms / 1e6 / peak_gbs, 4),
                                "weights_per_s": float(f"{nweights / (ms * 1e-3):.4g}"),
                                "products": len(run)}
        del run
    del mats
    torch.cuda.empty_cache()
    return out


def pack_rows(T, peak_gbs):
    """tern_pack_g128 on a gate-sized matrix (17408 x 5120): int8 codes and
    fp16 scales in, 2-bit slots and scales out; GB/s of those bytes."""
    s = torch.cuda.Stream()
    N, K = 17408, 5120
    g = synth.gen(77, "cuda")
    codes = synth.codes_sparse(N, K, g, device="cuda")
    scales = synth.scales_uniform(N, K, g, device="cuda")
    slots = torch.empty(N, K // 4, dtype=torch.uint8, device="cuda")
    sc = torch.empty_like(scales)
    ms = graph_time([lambda: T.tern_pack_g128(codes, scales, slots, sc)], s, reps=20)
    b = N * K + 2 * N * (K // GROUP) * 2 + N * K // 4
    del codes
    return {"pack_17408x5120": {"us": round(ms * 1e3, 3), "GBps": round(b / ms / 1e6, 1),
                                "frac": round(b / ms / 1e6 / peak_gbs, 4)}}


def embed_rows(T, model, peak_gbs):
    """tern_embed_gather from the head's table (tied weights, 151936 x 5120):
    M = 1 (a decode token) and M = 2048 (a prompt); GB/s of slots + scales
    read and fp16 rows written."""
    out = {}
    s = torch.cuda.Stream()
    _, K, V, slots, sc = model.head
    g = torch.Generator(device="cuda")
    g.manual_seed(88)
    for M in (1, 2048):
        ids = torch.randint(0, V, (M,), generator=g, device="cuda", dtype=torch.int32)
        o = torch.empty(M, K, dtype=torch.float16, device="cuda")
        ms = graph_time([lambda ids=ids, o=o: T.tern_embed_gather(ids, slots, sc, K, out=o)] * 16, s, reps=5)
        b = M * (K // 4 + 2 * (K // GROUP) + 2 * K) + 4 * M
        out[f"embed_M{M}"] = {"us": round(ms * 1e3, 3), "GBps": round(b / ms / 1e6, 1),
                              "frac": round(b / ms / 1e6 / peak_gbs, 4)}
    return out


def prefill_rows(T, peak_tf):
    """Prefill GEMM (tensor cores) at M = 2048 and 8192 for both shapes:
    TFLOP/s = 2*M*N*K / device time, against the measured dense fp16 peak."""
    out = {}
    s = torch.cuda.Stream()
    for ci, (K, N) in enumerate(synth.PREFILL):
        g = synth.gen(3000 + 10 * ci, "cuda")
        codes = synth.codes_uniform(N, K, g, device="cuda")
        scales = synth.scales_uniform(N, K, g, device="cuda")
        slots, sc = T.tern_pack_g128(codes, scales)
        del codes
        for M in synth.PREFILL_M:
            x = synth.activations(M, K, g, device="cuda")
            y = torch.empty(M, N, dtype=torch.float16, device="cuda")
            ms = graph_time([lambda: T.tern_gemm(x, slots, sc, y)], s, reps=5)
            tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
            out[f"prefill_K{K}_N{N}_M{M}"] = {"ms": round(ms, 4), "TFLOPs": round(tf, 1),
                                              "frac": round(tf / peak_tf, 4)}
            del x, y
        del slots, sc
    torch.cuda.empty_cache()
    return out


def graph_time(fns, stream, reps=3, flush=0):
    """Average device time per call of fns (captured once into a graph, the
    graph replayed `reps` times; with `flush` > 0 an L2-sized buffer is
    rewritten before each call, and its cost is timed separately and removed)."""
    fl = torch.empty(max(flush, 1) // 4 * 2, dtype=torch.float32, device="cuda") if flush else None
    with torch.cuda.stream(stream):
        for f in fns:  # warm-up (and first-call setup) outside capture
            if fl is not None:
                fl.fill_(1.0)
            f()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for f in fns:
                if fl is not None:
                    fl.fill_(1.0)
                f()
        g.replay()
        stream.synchronize()
        t = cuda_time(g.replay, reps, stream)
        if fl is not None:
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2, stream=stream):
                for _ in fns:
                    fl.fill_(1.0)
            g2.replay()
            t -= cuda_time(g2.replay, reps, stream)
    return t / len(fns)


# --------------------------------------------------------------- oracle ---
_ORACLE_JOBS = None


def oracle_sample(target_s: float = 12.0, max_s: float = 30.0):
    """Time the fp64 oracle on a bounded sample of the decode step: the
    projections of one decode layer and a slice of the head, inputs drawn on the
    host and packed by the oracle itself (packing untimed), run in passes until
    `target_s` of oracle time (at least one matrix, at most `max_s`).
    Returns (GB/s, threads, description)."""
    global _ORACLE_JOBS
    import oracle
    orc = oracle.load()
    threads = os.cpu_count() or 1
    if _ORACLE_JOBS is None:
        _ORACLE_JOBS = _oracle_jobs(orc)
    packed = _ORACLE_JOBS
    done_bytes, t_total, mats = 0, 0.0, 0
    while t_total < target_s:
        for name, K, N, xb, sl, sc in packed:
            t0 = time.perf_counter()
            orc.matmul(xb, sl, sc, threads=threads)
            t_total += time.perf_counter() - t0
            done_bytes += wbytes(K, N) + 2 * K + 2 * N
            mats += 1
            if t_total >= target_s or t_total > max_s:
                break
        if t_total > max_s:
            break
    used = orc.threads_used
    desc = (f"{mats} matrix products from one decode layer (q,k,v,o,gate,up,down, M=1) and 16384 rows "
            f"of the 5120x151936 head, in that order, fp64 oracle, {used} OpenMP threads, {t_total:.1f} s")
    return done_bytes / t_total / 1e9, used, desc


def _orc_inputs(orc, x, codes, scales):
    xb = x.contiguous().view(torch.int16).numpy().view(np.uint16)
    sl, sc, _, _ = orc.pack(codes.numpy(), scales.view(torch.int16).numpy().view(np.uint16))
    return xb, sl, sc


def oracle_configs():
    """The oracle on each named workload, on one host thread and on all of
    them: the tiny GEMV, every decode-layer projection at M = 1, and the
    prefill GEMM K = 5120 -> N = 17408 timed on a few token rows and
    extrapolated by rows to M = 2048 and 8192 (labelled so).  Packing is not
    timed.  About 10 s of host time on 8 cores."""
    import oracle
    orc = oracle.load()
    allc = os.cpu_count() or 1
    out = {}

    def timed(xb, sl, sc, threads, reps):
        best = float("inf")
        for _ in range(reps):
            t0 = time.perf_counter()
            orc.matmul(xb, sl, sc, threads=threads)
            best = min(best, time.perf_counter() - t0)
        return best * 1e3

    xb, sl, sc = _orc_inputs(orc, *synth.tiny_gemv())
    out["tiny_gemv_M1_K512_N256"] = {"ms_1t": round(timed(xb, sl, sc, 1, 5), 4),
                                     "ms_all": round(timed(xb, sl, sc, allc, 5), 4)}
    for i, (name, K, N) in enumerate(synth.LAYER_PROJ):
        xb, sl, sc = _orc_inputs(orc, *synth.decode_proj(i))
        b = wbytes(K, N) + 2 * K + 2 * N
        m1, ma = timed(xb, sl, sc, 1, 1), timed(xb, sl, sc, allc, 1)
        out[f"decode_{name}_M1_K{K}_N{N}"] = {"ms_1t": round(m1, 2), "ms_all": round(ma, 2),
                                              "GBps_all": round(b / ma / 1e6, 3)}
    K, N = synth.PREFILL[0]
    x, codes, scales = synth.prefill(0, 2048)
    xb, sl, sc = _orc_inputs(orc, x, codes, scales)
    r1, ra = 1, 4
    per1 = timed(xb[:r1], sl, sc, 1, 1) / r1
    pera = timed(xb[:ra], sl, sc, allc, 1) / ra
    for M in synth.PREFILL_M:
        out[f"prefill_K{K}_N{N}_M{M}"] = {
            "ms_1t_extrapolated": round(per1 * M, 1), "ms_all_extrapolated": round(pera * M, 1),
            "TFLOPs_all_extrapolated": round(2 * M * N * K / (pera * M * 1e-3) / 1e12, 6),
            "timed_rows": {"1t": r1, "all": ra}}
    return out, orc.threads_used


def _oracle_jobs(orc):
    jobs = []
    for i, (name, K, N) in enumerate(synth.LAYER_PROJ):
        x, codes, scales = synth.case(1, K, N, seed=6000 + i, codes="sparse")
        jobs.append((name, K, N, x, codes, scales))
    _, K, N = synth.HEAD
    x, codes, scales = synth.case(1, K, 16384, seed=6100, codes="sparse")
    jobs.append(("head_slice", K, 16384, x, codes, scales))
    packed = []
    for name, K, N, x, codes, scales in jobs:
        xb = x.view(torch.int16).numpy().view(np.uint16)
        sl, sc, _, _ = orc.pack(codes.numpy(), scales.view(torch.int16).numpy().view(np.uint16))
        packed.append((name, K, N, xb, sl, sc))
    return packed


def run_reference(args):
    ws, rank, _ = dist_setup(args)
    if rank != 0:
        return 0
    wb, xin, yout = step_bytes()
    total = wb + xin + yout
    vals, times = [], []
    per_step = max(0.05, min(2.0, 150.0 / (args.warmup + args.steps)))  # whole run ~<= 3 min
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        gbs, used, desc = oracle_sample(target_s=per_step, max_s=3 * per_step)
        if i >= args.warmup:
            vals.append(gbs)
            times.append(time.perf_counter() - t0)
    gbs = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        # the time of each timed (sampled) step, as run; the full 6.01 GB step
        # at this rate would take ms_per_full_step_projected
        "ms_per_step": round(1e3 * statistics.mean(times), 3),
        "ms_per_full_step_projected": round(total / (gbs * 1e9) * 1e3, 1),
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "decode step: 64 layers x {q,k,v,o,gate,up,down} + head 5120->151936, "
                               "M=1, ternary-g128 2-bit slots; each step a bounded CPU sample of it "
                               f"(about {per_step:.2f} s of oracle time: projections of one layer and "
                               "rows of the head, in order), GB/s of the sampled bytes",
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": used, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- main ---
# The kernel that carries the decode step (every grouped layer and the head).
DOMINANT_KERNEL, DOMINANT_SOURCE = "gemv_step_kernel", "tern_gemv_step.cu"


def traffic_from_profile(avg_launch_bytes):
    """Per-launch DRAM bytes of the dominant kernel from the committed ncu
    summary, only if the kernel source is unchanged since the capture."""
    prof = os.path.join(ROOT, "profiles", f"{DOMINANT_KERNEL}.decode_step.txt")
    src = os.path.join(ROOT, "ternary_weight_only_b200", "csrc", DOMINANT_SOURCE)
    try:
        text = open(prof).read()
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
        m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
        m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
        m_a = re.search(r"algorithmic_bytes_per_launch:\s*([0-9.eE+]+)", text)
        if m_sha and m_b and m_a and m_sha.group(1) == sha:
            # DRAM bytes per algorithmic byte of the captured launch, applied
            # to the average launch of the step.
            return float(m_b.group(1)) / float(m_a.group(1)) * avg_launch_bytes
    except OSError:
        pass
    return None


def run_profile(args):
    """Small case for ncu captures: a few layers' grouped launches, eager."""
    torch.cuda.set_device(0)
    from ternary_weight_only_b200 import tern as T
    if args.gemv_variant:
        T.tern_set_option(T.TERN_OPT_GEMV_VARIANT, args.gemv_variant)
    model = DecodeModel(T, n_layers=args.profile_layers)
    _, hK, hN, hslots, hsc = model.head
    if args.profile_format != "tern":
        # the same products with 1-bit or five-per-byte weights, one step call
        pack = T.tern_b1_pack if args.profile_format == "b1" else T.tern_t5_pack
        draw = synth.codes_sign if args.profile_format == "b1" else synth.codes_sparse
        g = synth.gen(8800, "cuda")
        mats, nbytes = [], 0
        for x, slots, sc, y in model.all_mats():
            N, K = slots.shape[0], x.shape[-1]
            w, wsc = pack(draw(N, K, g, device="cuda"), synth.scales_uniform(N, K, g, device="cuda"))
            mats.append((x, w, wsc, y))
            nbytes += w.numel() + 2 * wsc.numel() + 2 * K + 2 * N
        step = T.tern_b1_gemv_step if args.profile_format == "b1" else T.tern_t5_gemv_step
        for _ in range(3):
            step(mats)
        torch.cuda.synchronize()
        print(json.dumps({"profile_layers": args.profile_layers, "profile_format": args.profile_format,
                          "bytes_per_launch": nbytes}))
        return 0
    for _ in range(3):
        if args.profile_step:
            model.step()
        elif args.profile_head:
            T.tern_gemv(model.head_io[0], hslots, hsc, model.head_io[1])
        else:
            for grp in model.groups:
                T.tern_gemv_grouped(grp, 1)
    torch.cuda.synchronize()
    layer = sum(wbytes(K, N) + 2 * K + 2 * N for _, K, N in synth.LAYER_PROJ)
    head = wbytes(hK, hN) + 2 * hK + 2 * hN
    if args.profile_step:
        per_launch = (args.profile_layers * layer + head) / model.launches_per_step
    else:
        per_launch = head if args.profile_head else layer
    print(json.dumps({"profile_layers": args.profile_layers, "profile_head": bool(args.profile_head),
                      "profile_step": bool(args.profile_step), "launches": model.launches_per_step,
                      "bytes_per_launch": per_launch}))
    return 0


def run_profile_prefill(args):
    """Small case for ncu captures of the tensor-core prefill kernel: one
    K = 5120 -> N = 17408 product at M token rows (the prefill workload's
    first shape), run three times."""
    torch.cuda.set_device(0)
    from ternary_weight_only_b200 import tern as T
    M, (K, N) = args.profile_prefill, synth.PREFILL[0]
    g = synth.gen(3000, "cuda")
    slots, sc = T.tern_pack_g128(synth.codes_uniform(N, K, g, device="cuda"),
                                 synth.scales_uniform(N, K, g, device="cuda"))
    x = synth.activations(M, K, g, device="cuda")
    y = torch.empty(M, N, dtype=torch.float16, device="cuda")
    for _ in range(3):
        T.tern_gemm(x, slots, sc, y)
    torch.cuda.synchronize()
    print(json.dumps({"profile_prefill": M, "K": K, "N": N, "flops_per_launch": 2 * M * N * K}))
    return 0


def run_tern(args):
    ws, rank, local = dist_setup(args)
    from ternary_weight_only_b200 import tern as T
    peak_gbs, peak_tf, peak_tf_s, peak_src = load_peaks()
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    l2 = getattr(props, "L2_cache_size", 126 * 1024 * 1024)

    model = DecodeModel(T)
    wb, xin, yout = step_bytes()
    total_bytes = wb + xin + yout

    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        model.step()  # first-call setup outside capture
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            model.step()
        # The weight packing above streams HBM for seconds.  On B200 the step
        # held back to back trips the power cap after ~60 ms (SM clock down to
        # ~1.55 GHz, the step ~1.07 ms instead of ~0.93 ms), so the timed steps
        # start from a rested GPU, as the burst copy that the roofline peak
        # comes from does; the back-to-back rate is reported as "sustained".
        stream.synchronize()
        time.sleep(REST_S)
        for _ in range(args.warmup):
            graph.replay()
        stream.synchronize()

        barrier(ws)
        torch.cuda.synchronize()
        clocks = ClockSampler(local)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with clocks:
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
            e1.synchronize()
        torch.cuda.synchronize()
        barrier(ws)
        ms_local = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms_local, ws)
    value = ws * total_bytes / (ms * 1e-3) / 1e9  # GB/s over all ranks (weak scaling)

    # ---- e2e: host inputs -> device, step, outputs -> host, every step ----
    # The step's products go in three chunks of consecutive layers (the head
    # with the first; DecodeModel.e2e_chunks); per chunk: copy its inputs in
    # (copy stream), run it (tern_gemv_step on the compute stream), copy its
    # outputs back (second copy stream), so that the copies of one chunk
    # overlap the products of the others.  One step is captured as one CUDA
    # graph.
    x_host = torch.empty(model.x_all.shape, dtype=torch.float16, pin_memory=True)
    x_host.copy_(model.x_all.cpu())
    y_host = torch.empty(model.y_all.shape, dtype=torch.float16, pin_memory=True)
    chunks = model.e2e_chunks()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_body():
        ev_in = []
        for (mats, xr, yr) in chunks:
            s_in.wait_stream(stream)
            with torch.cuda.stream(s_in):
                for a, b in xr:
                    model.x_all[a:b].copy_(x_host[a:b], non_blocking=True)
                e = torch.cuda.Event()
                e.record(s_in)
                ev_in.append(e)
        for (mats, xr, yr), e in zip(chunks, ev_in):
            stream.wait_event(e)
            T.tern_gemv_step(mats)
            d = torch.cuda.Event()
            d.record(stream)
            s_out.wait_event(d)
            with torch.cuda.stream(s_out):
                for a, b in yr:
                    y_host[a:b].copy_(model.y_all[a:b], non_blocking=True)
        stream.wait_stream(s_out)
        stream.wait_stream(s_in)

    with torch.cuda.stream(stream):
        e2e_body()  # first-call setup outside capture
        stream.synchronize()
        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e, stream=stream):
            e2e_body()
        stream.synchronize()
        time.sleep(REST_S)  # as for the device-timed steps
        for _ in range(max(3, args.warmup)):
            g_e2e.replay()
        stream.synchronize()
        barrier(ws)
        e2e_ms_local = cuda_time(g_e2e.replay, args.steps, stream)
        barrier(ws)
    torch.cuda.synchronize()
    assert torch.equal(y_host, model.y_all.cpu()), "e2e outputs differ from the device results"
    e2e_ms = max_over_ranks(e2e_ms_local, ws)
    e2e_value = ws * total_bytes / (e2e_ms * 1e-3) / 1e9

    # ---- sustained: the same step back to back once the power cap has
    # engaged (SUSTAIN_LEAD untimed steps, then SUSTAIN_STEPS timed) ----
    with torch.cuda.stream(stream):
        for _ in range(SUSTAIN_LEAD):
            graph.replay()
        stream.synchronize()
        clocks_sus = ClockSampler(local)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with clocks_sus:
            s0.record(stream)
            for _ in range(SUSTAIN_STEPS):
                graph.replay()
            s1.record(stream)
            s1.synchronize()
    sus_ms = max_over_ranks(s0.elapsed_time(s1) / SUSTAIN_STEPS, ws)
    sus_value = ws * total_bytes / (sus_ms * 1e-3) / 1e9
    if rank == 0 and ws == 1:
        time.sleep(REST_S)  # the per-shape rows below start rested too

    # ---- per-shape breakdown (rank 0 only, outside the timed region) ----
    # (one GPU only: under torchrun the other GPUs would sit idle meanwhile)
    rows = None
    if rank == 0 and ws == 1 and not args.no_rows:
        rows = proj_rows(T, model, peak_gbs, l2)
        rows.update(pack_rows(T, peak_gbs))
        rows.update(b1_rows(T, model, peak_gbs, (clocks.summary() or {}).get("sm_mhz")))
        rows.update(t5_rows(T, model, peak_gbs))
        rows.update(embed_rows(T, model, peak_gbs))
        rows.update(prefill_rows(T, peak_tf))

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        gbs, used, desc = oracle_sample()
        per_config, _ = oracle_configs()
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": used, "kind": "oracle", "sample": desc,
               "decode_step_ms_all_extrapolated": round(total_bytes / (gbs * 1e9) * 1e3, 1),
               "per_config": per_config}

    launches = model.launches_per_step * args.steps
    per_launch_ms = ms_local / model.launches_per_step
    achieved = total_bytes / model.launches_per_step / (per_launch_ms * 1e-3) / 1e9
    traffic = traffic_from_profile(total_bytes / model.launches_per_step)
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "u2+f16 weights, f16 x, f32 acc", "data": "synthetic",
            "config": {"workload": "decode step: 64 layers x {q 5120->6144, k/v 5120->1024, o 6144->5120, "
                                   "gate/up 5120->17408, down 17408->5120} + head 5120->151936; M=1; "
                                   "ternary-g128 2-bit slots; codes P(0)=0.4 P(+-1)=0.3, scales U[0.005,0.05], "
                                   "x N(0,1)",
                       "weights_bytes": wb, "bytes_per_step": total_bytes,
                       "l2": f"inputs {wb/1e9:.2f} GB >> L2 {l2/1e6:.0f} MB, no flush needed",
                       "launch": f"CUDA graph of {model.launches_per_step} launches/step (tern_gemv_step over all "
                                 f"{len(model.all_mats())} products, at most {STEP_PER_LAUNCH} per launch)",
                       "parallelism": f"replicas x{ws}" if ws > 1 else "1 GPU"},
            "pct_of_peak_hbm": round(100 * value / ws / peak_gbs, 2),
            "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "ms_per_step": round(e2e_ms, 4),
                    "h2d_bytes_per_step": int(model.x_all.numel() * 2),
                    "d2h_bytes_per_step": int(model.y_all.numel() * 2)},
            "roofline": {"bound": "hbm", "kernel": DOMINANT_KERNEL,
                         "achieved": round(achieved, 1), "peak": peak_gbs, "unit": "GB/s",
                         "frac": round(achieved / peak_gbs, 4), "traffic": round(traffic) if traffic else None,
                         "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else "fallback 6650 GB/s",
                         "per_launch": "device time of the timed region / launches (gaps included)"},
            "sustained": {"ms_per_step": round(sus_ms, 4), "value": round(sus_value, 1), "unit": "GB/s",
                          "frac": round(sus_value / ws / peak_gbs, 4), "steps": SUSTAIN_STEPS,
                          "after_steps": SUSTAIN_LEAD, "clocks": clocks_sus.summary(),
                          "note": f"timed steps start after {REST_S:.0f} s idle (burst, like the copy peak); "
                                  "back to back the power cap lowers the SM clock"},
            "cpu_baseline": cpu,
            "gpu_launches": launches,
            "clocks": clocks.summary(),
            "rows": rows,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        del graph
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["tern", "reference"], default="tern")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-shape breakdown")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--profile-layers", type=int, default=0,
                    help="profiling case: build this many layers, run their grouped launches 3x, exit")
    ap.add_argument("--profile-step", action="store_true",
                    help="profiling case: run the layers and the head as tern_gemv_step calls 3x")
    ap.add_argument("--profile-format", choices=["tern", "b1", "t5"], default="tern",
                    help="profiling case with --profile-layers: the step's products as 1-bit or five-per-byte "
                         "matrices in one step call (run 3x)")
    ap.add_argument("--profile-head", action="store_true",
                    help="profiling case: run the 5120x151936 head launch 3x instead of the layers")
    ap.add_argument("--profile-prefill", type=int, default=0, metavar="M",
                    help="profiling case: the prefill GEMM K=5120 -> N=17408 at M token rows, run 3x, exit")
    ap.add_argument("--gemv-variant", type=int, default=0,
                    help="profiling case only: bandwidth kernel variant (TERN_OPT_GEMV_VARIANT)")
    args = ap.parse_args()
    if args.profile_prefill > 0:
        return run_profile_prefill(args)
    if args.profile_layers > 0:
        return run_profile(args)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_tern(args)


if __name__ == "__main__":
    sys.exit(main())
