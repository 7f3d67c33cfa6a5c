"""Benchmark of the ternary linear layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload decode|prefill|fused|sweep|roundtrip|mlp|train]
                    [--layout foundry|format0|format1] [--ratio R] [--bias] [--impl ours|reference]

One JSON line on rank 0.  A *step* is one pass of the whole hot path over one
batch of synthetic input: quantise + pack the fp32 latent weights (absmean
gamma, 2-bit codes), quantise the activations per token, run the ternary
contraction with the fused rescale (and, for the fused workload, the
RMSNorm + FWHT prologue).

Default workload ("decode"): K = N = 4096, per-row gamma, W ~ N(0, 0.02),
activations ~ N(0, 1) with 0.1 % outliers x20, token batches M = 1 and M = 8.
A ring of L = 64 distinct layers keeps every working set above L2: per step the
64 fp32 weights (4 GiB) are re-packed (the packed ring is 256 MiB), each layer's
activation batches (its own buffers) are quantised, and each batch runs through
the GEMV of its layer.
Metric: algorithmic HBM bytes of the step / step time (GB/s).

The layers of the ring have their own weights, activations, outputs and
workspaces, so the calls within one segment (packs, activation quantisations,
contractions) are independent: they are issued with TQ_FLAG_INPUTS_READY (and
TQ_FLAG_WEIGHTS_STATIC for the contractions), which lets consecutive kernels
overlap.  For the small-M GEMVs the line also reports "chain": the
same launches as a chain of dependent layers (each kernel waits for the
previous one before reading), timed separately and not part of the step.

Timing: CUDA graphs for each segment (pack, activation quantisation, GEMV
M=1, GEMV M=8), CUDA events between segments on the launching stream, barrier
+ synchronize around the timed steps, max over ranks.  Per-kernel average
launch time = segment time / launches in the segment.

Other workloads: "prefill" (2048 x 11008 x 4096 GEMM, per-tensor gamma),
"fused" (RMSNorm + FWHT + int8 + GEMM, 512 x 5632 x 2048), "sweep" (M from 1
to 4096 at 8192^2), "roundtrip" (the FWHT module's int8 round trip), "mlp"
(the clamped SwiGLU block, 512 tokens, 1536 -> 6144 -> 1536) and "train" (the
input gradient of the prefill layer, the STE of its latent weights and the
stochastic flip of its codes); --layout, --ratio and --bias select the
packed-code layout, the threshold ternarisation rule and the bias epilogue.
Metric: TOPS (TFLOP/s for train) of the step's contractions / step time for
the GEMM workloads, GB/s for decode and roundtrip.

--impl reference times the CPU oracle (the plain C reference) on a bounded
sample of the same workload, on this host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ternary GEMM TOPS (M>=512) & packed-weight HBM GB/s (M<=16), % of roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_HBM = 6650.0
FALLBACK_BF16 = 1590.0
INT8_OVER_BF16 = 2.0  # nominal dense int8 (4.5 POPS) / bf16 (2.25 PFLOP/s)


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {"hbm": float(p["hbm_gbs"]), "bf16": float(p["bf16_tflops"]),
                "bf16_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm": FALLBACK_HBM, "bf16": FALLBACK_BF16, "bf16_sustained": 1400.0,
                "source": "fallback"}


KERNEL_FILES = {  # device sources of each kernel (besides tq_common.cuh)
    "pack": ["tq_pack.cuh"], "act_quant": ["tq_act.cuh"], "gemv": ["tq_gemv.cuh"],
    "gemm": ["tq_gemm.cuh"], "fused": ["tq_act.cuh", "tq_gemm.cuh"],
    "bwd": ["tq_train.cuh", "tq_gemm.cuh"], "ste": ["tq_train.cuh"], "flip": ["tq_train.cuh", "tq_xorshift_jump.h"],
}


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "ternary_bit_linear_b200", "csrc")
    for name in ["tq_common.cuh"] + KERNEL_FILES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_for(key: str):
    """DRAM bytes per launch ("kernel:workload") from the committed ncu
    summary, or None if that kernel's sources changed since it was taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)["kernels"][key]
        if t["source_hash"] != kernel_source_hash(key.split(":")[0]):
            return None
        return t["bytes"]
    except Exception:
        return None


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------
class ClockSampler:
    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        med = float(np.median(self.samples)) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
class Workload:
    """Builds device buffers and the per-segment launch lists of one step."""

    def __init__(self, name, tq, S, torch, dev, layers, layout=0, ratio=0.0, bias=False):
        self.name, self.tq, self.torch, self.dev = name, tq, torch, dev
        f32, u8, i8, i32 = torch.float32, torch.uint8, torch.int8, torch.int32
        self.segments = []  # (label, kernel_name, launches, algorithmic bytes or ops, [fns])
        self.bias = None
        self.chains = []    # (label, launches, bytes per launch, [fns]): dependent-layer GEMV chains
        if name == "decode":
            N = K = 4096
            self.N, self.K, self.Ms, self.L = N, K, [1, 8], layers
            self.per_row = True
            W = torch.from_numpy(S.decode_weights(N, K, seed=0))
            self.W = [W.to(dev) for _ in range(self.L)]  # distinct buffers, same values
            self.X = {M: torch.from_numpy(S.decode_acts(M, K, seed=0)) for M in self.Ms}
        elif name == "prefill":
            M, N, K = 2048, 11008, 4096
            self.N, self.K, self.Ms, self.L = N, K, [M], layers
            self.per_row = False
            W, X = S.prefill(M, N, K, seed=0)
            W = torch.from_numpy(W)
            self.W = [W.to(dev) for _ in range(self.L)]
            self.X = {M: torch.from_numpy(X)}
        elif name == "fused":
            M, N, K = 512, 5632, 2048
            self.N, self.K, self.Ms, self.L = N, K, [M], layers
            self.per_row = False
            W, X = S.fused(M, N, K, seed=0)
            W = torch.from_numpy(W)
            self.W = [W.to(dev) for _ in range(self.L)]
            self.X = {M: torch.from_numpy(X)}
        elif name == "sweep":
            N = K = 8192
            self.N, self.K, self.Ms, self.L = N, K, [1, 4, 16, 64, 512, 4096], layers
            self.per_row = True
            W = torch.from_numpy(S.sweep_weights(N, K, seed=0))
            self.W = [W.to(dev) for _ in range(self.L)]
            self.X = {M: torch.from_numpy(S.sweep_acts(M, K, seed=0)) for M in self.Ms}
        elif name == "mlp":
            # Hetman-2b's clamped SwiGLU block: d_model 1536, d_ffn 4 * 1536, 512 tokens
            M, D, F = 512, 1536, 6144
            self.N, self.K, self.Ms, self.L = D, D, [M], layers
            self.per_row = False
            self.layout, self.ratio = layout, ratio
            fl = tq.FLAG_FWHT | tq.FLAG_RMSNORM | (layout << 7)
            X = torch.from_numpy(S.fused(M, 16, D, seed=0)[1])
            shapes = [(F, D), (F, D), (D, F)]
            Wf = [torch.from_numpy(S.normal(sh, 0.02, 7 + i, sh[0])) for i, sh in enumerate(shapes)]
            self.W3 = [[w.to(dev) for w in Wf] for _ in range(layers)]
            self.P3 = [[(torch.empty((sh[0], sh[1] // 4), dtype=torch.uint8, device=dev),
                         torch.empty((1,), dtype=torch.float32, device=dev)) for sh in shapes] for _ in range(layers)]
            wsz = max(tq.pack_workspace_bytes(sh[0], sh[1], 0) for sh in shapes)
            self.pws3 = [torch.empty((wsz,), dtype=torch.uint8, device=dev) for _ in range(layers)]
            self.X = {M: X}
            self.Xd = {M: [X.to(dev) for _ in range(layers)]}
            self.y = {M: [torch.empty((M, D), dtype=torch.float32, device=dev) for _ in range(layers)]}
            self.mws = [torch.empty((tq.swiglu_workspace_bytes(M, D, F, fl),), dtype=torch.uint8, device=dev)
                        for _ in range(layers)]
            pack_bytes = sum(4 * a * b + a * b // 4 + 4 for a, b in shapes)
            self.segments.append(("pack", "pack", 3 * layers, layers * pack_bytes, 6 * layers, [
                lambda l=l, i=i: tq.quantize_ternary_pack_(self.W3[l][i], (layout << 7), self.P3[l][i][0],
                                                          self.P3[l][i][1], self.pws3[l])
                for l in range(layers) for i in range(3)]))
            ops = 2 * M * 3 * D * F
            self.segments.append(("mlp M=%d" % M, "mlp", layers, layers * ops, 5 * layers, [
                lambda l=l: tq.swiglu_mlp_(self.Xd[M][l], self.P3[l][0], self.P3[l][1], self.P3[l][2],
                                           fl | tq.FLAG_WEIGHTS_STATIC, self.y[M][l], self.mws[l])
                for l in range(layers)]))
            return
        elif name == "train":
            # one training step of the prefill layer (2048 tokens, 4096 -> 11008 features): the input
            # gradient dX = (dY * gamma) W, the STE gradient of the latent weights and the
            # stochastic flip of the packed codes (the weight-gradient GEMM X^T dY is a plain float
            # GEMM outside this library: its output G is a synthetic input here)
            M, N, K = 2048, 11008, 4096
            self.N, self.K, self.Ms, self.L = N, K, [M], layers
            self.per_row = False
            self.layout, self.ratio = layout, ratio
            fl = layout << 7
            W, _ = S.prefill(M, N, K, seed=0)
            dY = torch.from_numpy(S.normal((M, N), 1.0, 160, 0))
            G = torch.from_numpy(S.normal((N, K), 1.0, 161, 0))
            W = torch.from_numpy(W)
            self.Wl = [W.to(dev) for _ in range(layers)]
            self.G = [G.to(dev) for _ in range(layers)]
            self.gw = [torch.empty((N, K), dtype=f32, device=dev) for _ in range(layers)]
            self.packed = [torch.empty((N, K // 4), dtype=u8, device=dev) for _ in range(layers)]
            self.gamma = [torch.empty((1,), dtype=f32, device=dev) for _ in range(layers)]
            pws = torch.empty((tq.pack_workspace_bytes(N, K, 0),), dtype=u8, device=dev)
            for l in range(layers):
                tq.quantize_ternary_pack_(self.Wl[l], fl, self.packed[l], self.gamma[l], pws)
            self.X = {M: dY}
            self.Xd = {M: [dY.to(dev) for _ in range(layers)]}
            self.y = {M: [torch.empty((M, K), dtype=f32, device=dev) for _ in range(layers)]}
            self.bws = [torch.empty((tq.backward_input_workspace_bytes(M, N),), dtype=u8, device=dev)
                        for _ in range(layers)]
            self.rng = tq.seed(42)
            self.segments.append(("backward dX M=%d" % M, "bwd", layers, layers * 2 * M * N * K, 2 * layers, [
                lambda l=l: tq.ternary_backward_input_(self.Xd[M][l], self.packed[l], self.gamma[l], fl,
                                                       self.y[M][l], self.bws[l])
                for l in range(layers)]))
            self.segments.append(("ste", "ste", layers, layers * 12 * N * K, layers, [
                lambda l=l: tq.ste_backward_(self.G[l], self.Wl[l], self.gamma[l], 0, self.gw[l])
                for l in range(layers)]))
            self.segments.append(("flip", "flip", layers, layers * (4 * N * K + N * K // 2), layers, [
                lambda l=l: tq.ternary_stochastic_flip_(self.packed[l], self.G[l], 0.05, self.rng, fl)
                for l in range(layers)]))
            return
        elif name == "roundtrip":
            # the FWHT module's int8 round trip on the fused configuration's activations
            M, K = 512, 2048
            self.N, self.K, self.Ms, self.L = 0, K, [M], layers
            self.per_row = False
            self.layout, self.ratio = layout, ratio
            X = torch.from_numpy(S.fused(M, 16, K, seed=0)[1])
            self.X = {M: X}
            self.Xd = {M: [X.to(dev) for _ in range(layers)]}
            self.yr = [torch.empty((M, K), dtype=torch.float32, device=dev) for _ in range(layers)]
            self.y = {M: self.yr}
            self.segments.append(("fwht roundtrip", "roundtrip", layers, layers * 8 * M * K, layers, [
                lambda l=l: tq.fwht_roundtrip_(self.Xd[M][l], self.yr[l], 0.05, 40.0) for l in range(layers)]))
            return
        else:
            raise SystemExit(f"unknown workload {name}")
        N, K, L = self.N, self.K, self.L
        # packed-code layout (0 Foundry, 1 Hetman-2b Format 0, 2 Format 1) on every pack and contraction
        self.layout, self.ratio = layout, ratio
        self.flags = (tq.GAMMA_PER_ROW if self.per_row else 0) | (layout << 7)
        # the ring's layers share x and have their own weights and outputs:
        # independent calls, so the contractions may overlap one another
        self.ready_flags = self.flags | tq.FLAG_WEIGHTS_STATIC | tq.FLAG_INPUTS_READY
        self.packed = [torch.empty((N, K // 4), dtype=u8, device=dev) for _ in range(L)]
        self.gamma = [torch.empty((N if self.per_row else 1,), dtype=f32, device=dev) for _ in range(L)]
        nws = tq.pack_workspace_bytes(N, K, self.flags)
        # one workspace per layer: the ring's packs are independent calls
        self.pack_ws = [torch.empty((max(nws, 16),), dtype=u8, device=dev) for _ in range(L)]
        # every layer of the ring has its own activation batch (same values)
        self.Xd = {M: [x.to(dev) for _ in range(L)] for M, x in self.X.items()}
        self.xq = {M: [torch.empty((M, K), dtype=i8, device=dev) for _ in range(L)] for M in self.Ms}
        self.sx = {M: [torch.empty((M,), dtype=f32, device=dev) for _ in range(L)] for M in self.Ms}
        self.rs = {M: [torch.empty((M,), dtype=i32, device=dev) for _ in range(L)] for M in self.Ms}
        self.y = {M: [torch.empty((M, N), dtype=f32, device=dev) for _ in range(L)] for M in self.Ms}
        if name == "fused":
            fl = tq.FLAG_FWHT | tq.FLAG_RMSNORM
            # the ring's layers have their own x, y and workspace: independent calls
            self.fused_flags = fl | tq.FLAG_WEIGHTS_STATIC | tq.FLAG_INPUTS_READY | (layout << 7)
            self.fused_ws = [torch.empty((tq.fused_workspace_bytes(self.Ms[0], K, fl),), dtype=u8, device=dev)
                             for _ in range(L)]

        # --- segments of one step ---
        pack_bytes = 4 * N * K + N * K // 4 + 4 * (N if self.per_row else 1)
        pack_launches = 1 if self.per_row else 2  # per tensor: partial sums, then the pack pass
        if ratio > 0:  # threshold ternarisation (w > ratio * gamma) instead of round/clamp
            pack_fns = [lambda l=l: tq.quantize_ternary_pack_threshold_(
                self.W[l], self.flags | tq.FLAG_INPUTS_READY, ratio, self.packed[l], self.gamma[l], self.pack_ws[l])
                for l in range(L)]
        else:
            pack_fns = [lambda l=l: tq.quantize_ternary_pack_(self.W[l], self.flags | tq.FLAG_INPUTS_READY,
                                                              self.packed[l], self.gamma[l], self.pack_ws[l])
                        for l in range(L)]
        self.segments.append(("pack", "pack", L, L * pack_bytes, L * pack_launches, pack_fns))
        if name == "fused":
            M = self.Ms[0]
            ops = 2 * M * N * K
            self.segments.append(("fused M=%d" % M, "fused", L, L * ops, 2 * L, [
                lambda l=l: tq.bitlinear_fused_(self.Xd[M][l], self.packed[l], self.gamma[l],
                                                self.fused_flags, self.y[M][l], self.fused_ws[l])
                for l in range(L)]))
            return
        act_bytes = L * sum(4 * M * K + M * K + 8 * M for M in self.Ms)
        nact = L * len(self.Ms)
        self.segments.append(("act", "act_quant", nact, act_bytes, nact, [
            lambda M=M, l=l: tq.quantize_act_int8_(self.Xd[M][l], tq.FLAG_INPUTS_READY, 0.05, 40.0,
                                                   self.xq[M][l], self.sx[M][l], self.rs[M][l])
            for M in self.Ms for l in range(L)]))
        self.bias = [torch.full((N,), 0.25, dtype=f32, device=dev) for _ in range(L)] if bias else None
        for M in self.Ms:
            gemv = M <= 16
            work = (N * K // 4 + 4 * N * (1 if self.per_row else 0) + M * K + 8 * M + 4 * M * N) if gemv \
                else 2 * M * N * K
            if bias:  # the extra epilogue (y + bias[n]) through tq_ternary_gemm_ex
                fns = [lambda l=l, M=M: tq.ternary_gemm_ex_(self.xq[M][l], self.sx[M][l], self.rs[M][l],
                                                            self.packed[l], self.gamma[l], self.ready_flags,
                                                            self.y[M][l], bias=self.bias[l])
                       for l in range(L)]
            else:
                fns = [lambda l=l, M=M: tq.ternary_gemm_(self.xq[M][l], self.sx[M][l], self.rs[M][l],
                                                         self.packed[l], self.gamma[l], self.ready_flags,
                                                         self.y[M][l])
                       for l in range(L)]
            self.segments.append(("gemv M=%d" % M if gemv else "gemm M=%d" % M,
                                  "gemv" if gemv else "gemm", L, L * work, L, fns))
            if gemv:
                self.chains.append(("gemv M=%d" % M, L, work, [
                    lambda l=l, M=M: tq.ternary_gemm_(self.xq[M][l], self.sx[M][l], self.rs[M][l],
                                                      self.packed[l], self.gamma[l],
                                                      self.flags | tq.FLAG_WEIGHTS_STATIC, self.y[M][l])
                    for l in range(L)]))

    def step_bytes(self):
        return sum(s[3] for s in self.segments if s[1] in ("pack", "act_quant", "gemv", "roundtrip"))

    def step_ops(self):
        return sum(s[3] for s in self.segments if s[1] in ("gemm", "fused", "mlp", "bwd"))


def run_ours(args, rank, world, local_rank):
    import torch

    import ternary_bit_linear_b200 as tq
    from ternary_bit_linear_b200 import build as tqbuild
    from ternary_bit_linear_b200 import synthetic as S

    if rank == 0 or not os.path.exists(tqbuild.LIB):
        tqbuild.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    tq.load()
    wl = Workload(args.workload, tq, S, torch, dev, args.layers or WORKLOAD_SHAPES[args.workload][3],
                  LAYOUTS.index(args.layout), args.ratio, args.bias)
    stream = torch.cuda.Stream(device=dev)
    graphs = []
    with torch.cuda.stream(stream):
        for seg in wl.segments:  # eager warm-up of every launch, then capture
            for fn in seg[5]:
                fn()
        torch.cuda.synchronize()
        for seg in wl.segments:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for fn in seg[5]:
                    fn()
            graphs.append(g)
    torch.cuda.synchronize()

    def step():
        for g in graphs:
            g.replay()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    assert tq.device_status(stream) == 0

    nseg = len(graphs)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nseg + 1)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    with sampler:
        with torch.cuda.stream(stream):
            for k in range(args.steps):
                evs[k][0].record(stream)
                for i, g in enumerate(graphs):
                    g.replay()
                    evs[k][i + 1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    seg_ms = np.zeros(nseg)
    for k in range(args.steps):
        for i in range(nseg):
            seg_ms[i] += evs[k][i].elapsed_time(evs[k][i + 1])
    total_ms = float(seg_ms.sum())
    total_ms = allreduce_max(total_ms, world)
    ms_per_step = total_ms / args.steps
    assert tq.device_status(stream) == 0

    # --- end to end through the public API with host buffers ---
    e2e = run_e2e(args, wl, tq, torch, stream, graphs, world)
    chain = run_chains(args, wl, tq, torch, stream, world)

    pk = peaks()
    kernels = {}
    for (label, kname, launches, work, nlaunch, _), ms in zip(wl.segments, seg_ms):
        per_launch_ms = ms / args.steps / launches
        if kname in ("gemm", "fused", "mlp", "bwd"):
            ach = work / launches / (per_launch_ms * 1e-3) / 1e12
            # the input gradient contracts bf16 operands (the int8 kernels: twice the bf16 rate)
            peak = pk["bf16"] * (1.0 if kname == "bwd" else INT8_OVER_BF16)
            kernels[label] = {"bound": "tensor", "achieved": round(ach, 2), "peak": round(peak, 1),
                              "unit": "TOPS", "frac": round(ach / peak, 4),
                              "us_per_launch": round(per_launch_ms * 1e3, 3)}
        else:
            ach = work / launches / (per_launch_ms * 1e-3) / 1e9
            kernels[label] = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm"],
                              "unit": "GB/s", "frac": round(ach / pk["hbm"], 4),
                              "us_per_launch": round(per_launch_ms * 1e3, 3)}
            if kname == "flip":  # the xorshift64 chain keeps the ALU pipe busy before HBM
                kernels[label]["limiter"] = "alu pipe"
    dom = max(zip(wl.segments, seg_ms), key=lambda t: t[1])[0]
    dk = kernels[dom[0]]
    roofline = {"bound": dk["bound"], "achieved": dk["achieved"], "peak": dk["peak"],
                "unit": "GB/s" if dk["unit"] == "GB/s" else "TOPS", "frac": dk["frac"],
                "traffic": traffic_for(dom[1] + ":" + args.workload), "kernel": dom[0],
                "peak_source": pk["source"] + (" hbm_gbs (copy, burst)" if dk["bound"] == "hbm"
                                               else " bf16_tflops (bf16 operands)" if dom[1] == "bwd"
                                               else " bf16_tflops x2 (nominal int8/bf16 ratio)")}
    if wl.name in ("decode", "roundtrip"):
        value = wl.step_bytes() * world / (ms_per_step * 1e-3) / 1e9
        unit = "GB/s"
    else:
        value = wl.step_ops() * world / (ms_per_step * 1e-3) / 1e12
        unit = "TOPS"
    launches = sum(s[4] for s in wl.segments) * args.steps

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload, budget_s=args.cpu_seconds)
    clocks = sampler.summary()
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl.name == "train" else "int8",
        "data": "synthetic", "config": wl_config(wl, world),
        "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu,
        "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
    }
    if chain:
        out["chain"] = chain
    if rank == 0:
        print(json.dumps(out), flush=True)
    del graphs


WORKLOAD_SHAPES = {  # name -> (Ms, N, K, default ring of layers, per_row)
    "decode": ([1, 8], 4096, 4096, 64, True),
    "prefill": ([2048], 11008, 4096, 4, False),
    "fused": ([512], 5632, 2048, 8, False),
    "sweep": ([1, 4, 16, 64, 512, 4096], 8192, 8192, 8, True),
    "roundtrip": ([512], 0, 2048, 64, False),
    "mlp": ([512], 1536, 1536, 8, False),
    "train": ([2048], 11008, 4096, 4, False),
}


LAYOUTS = ["foundry", "format0", "format1"]  # packed-code layouts, flag value = index << 7


def config_for(name, layers, world, layout="foundry", ratio=0.0, bias=False):
    Ms, N, K, L, per_row = WORKLOAD_SHAPES[name]
    L = layers or L
    desc = {"decode": "decode GEMV: K=N=4096, per-row gamma, M in {1, 8}, ring of %d layers" % L,
            "prefill": "prefill GEMM: M=2048, N=11008, K=4096, per-tensor gamma, ring of %d layers" % L,
            "fused": "fused BitLinear: M=512, N=5632, K=2048, RMSNorm+FWHT-512, ring of %d layers" % L,
            "sweep": "M sweep over K=N=8192, per-row gamma, ring of %d layers" % L,
            "roundtrip": "FWHT module int8 round trip: 512 x 2048 Student-t(3), ring of %d batches" % L,
            "mlp": "clamped SwiGLU block of 3 BitLinears: 512 tokens, d_model 1536, d_ffn 6144, ring of %d" % L,
            "train": "training step of the prefill layer: dX = (dY gamma) W (M=2048, N=11008, K=4096), STE of "
                     "the latent weights, stochastic flip (T=0.05), ring of %d layers" % L}[name]
    return {"workload": desc, "M": Ms, "N": N, "K": K, "layers": L,
            "gamma": "per-row" if per_row else "per-tensor", "layout": layout,
            "ternarise": "threshold w > %g * gamma" % ratio if ratio > 0 else "round/clamp",
            "epilogue": "y + bias (tq_ternary_gemm_ex)" if bias else "y",
            "l2": ("inputs larger than L2 (no flush): per layer dY %d MiB, latent weights and their gradient "
                   "2 x %d MiB, packed %d MiB" % (Ms[0] * N * 4 >> 20, N * K * 4 >> 20, N * K // 4 >> 20)
                   if name == "train" else
                   "inputs larger than L2 (no flush): fp32 weights %d MiB, packed %d MiB per step" % (
                       L * N * K * 4 >> 20, L * N * K // 4 >> 20)),
            "parallelism": "replicas x%d" % world if world > 1 else "single GPU"}


def wl_config(wl, world):
    return config_for(wl.name, wl.L, world, LAYOUTS[wl.layout], wl.ratio, wl.bias is not None)


def run_chains(args, wl, tq, torch, stream, world):
    """Dependent-layer GEMV chains: per-launch time when every kernel waits
    for its predecessor's results (the latency-bound decode case)."""
    import torch as _t
    res = {}
    pk = peaks()
    for label, launches, work, fns in wl.chains:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for fn in fns:
                fn()
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for fn in fns:
                    fn()
            for _ in range(3):
                g.replay()
        torch.cuda.synchronize()
        reps = max(3, min(args.steps, 20))
        e0, e1 = _t.cuda.Event(enable_timing=True), _t.cuda.Event(enable_timing=True)
        barrier(world)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        ms = allreduce_max(e0.elapsed_time(e1), world) / (reps * launches)
        ach = work / (ms * 1e-3) / 1e9
        res[label] = {"us_per_launch": round(ms * 1e3, 3), "achieved": round(ach, 1), "unit": "GB/s",
                      "frac": round(ach / pk["hbm"], 4)}
        del g
    assert tq.device_status(stream) == 0
    return res


def run_e2e(args, wl, tq, torch, stream, graphs, world):
    """Same step through the public calls with pinned host inputs copied in and
    the step's outputs copied back inside the timed region."""
    host_x = {M: x.pin_memory() for M, x in wl.X.items()}
    outs = [y for M in wl.Ms for y in wl.y[M]]
    host_y = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for y in outs]
    h2d = sum(x.numel() * 4 * wl.L for x in host_x.values())
    d2h = sum(y.numel() * 4 for y in outs)
    steps = max(3, min(args.steps, 50))

    def one():
        for M in wl.Ms:
            for xd in wl.Xd[M]:
                xd.copy_(host_x[M], non_blocking=True)
        for g in graphs:
            g.replay()
        for y, hy in zip(outs, host_y):
            hy.copy_(y, non_blocking=True)

    with torch.cuda.stream(stream):
        one()
    torch.cuda.synchronize()
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(steps):
            one()
        t1.record(stream)
    torch.cuda.synchronize()
    ms = allreduce_max(t0.elapsed_time(t1), world) / steps
    if wl.name in ("decode", "roundtrip"):
        v, u = wl.step_bytes() * world / (ms * 1e-3) / 1e9, "GB/s"
    else:
        v, u = wl.step_ops() * world / (ms * 1e-3) / 1e12, "TOPS"
    return {"value": round(v, 2), "unit": u, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms, 4), "steps": steps}


# ---------------------------------------------------------------------------
# CPU oracle baseline / reference arm
# ---------------------------------------------------------------------------
def oracle_sample(workload):
    """One bounded unit of the workload on the oracle: returns (fn, work, what)."""
    import oracle
    from ternary_bit_linear_b200 import synthetic as S

    if workload == "decode":
        N = K = 4096
        W = S.decode_weights(N, K, seed=0)
        Xs = {M: S.decode_acts(M, K, seed=0) for M in (1, 8)}

        def fn():
            packed, gamma = oracle.quantize_pack(W, per_row=True)
            for M, X in Xs.items():
                xq, sx, _ = oracle.act_quant(X)
                oracle.dequant(oracle.matmul_addsub(xq, packed), gamma, sx, True)
        work = (4 * N * K + N * K // 4 + 4 * N) + sum(
            4 * M * K + M * K + 8 * M + N * K // 4 + 4 * N + M * K + 8 * M + 4 * M * N for M in (1, 8))
        return fn, work, "one full layer of the step (pack 4096x4096 per-row, act-quant + GEMV for M=1 and M=8)", "GB/s"
    if workload == "mlp":
        M, D, F = 512, 1536, 6144
        X = S.fused(M, 16, D, seed=0)[1]
        shapes = [(F, D), (F, D), (D, F)]
        packs = [oracle.quantize_pack(S.normal(sh, 0.02, 7 + i, sh[0]), per_row=False) for i, sh in enumerate(shapes)]
        rows = 2

        def fn():
            oracle.swiglu_mlp(X[:rows], packs[0], packs[1], packs[2], False)
        return fn, 2 * rows * 3 * D * F, "%d tokens through the block (weights pre-packed)" % rows, "TOPS"
    if workload == "train":
        M, N, K = 2048, 11008, 4096
        W, _ = S.prefill(M, N, K, seed=0)
        dY = S.normal((M, N), 1.0, 160, 0)
        packed, gamma = oracle.quantize_pack(W, per_row=False)
        rows = 2

        def fn():
            oracle.backward_input(dY[:rows], packed, gamma, False, K)
        return fn, 2 * rows * N * K, "%d tokens of the input gradient (weights pre-packed)" % rows, "TOPS"
    if workload == "roundtrip":
        M, K = 512, 2048
        X = S.fused(M, 16, K, seed=0)[1]
        rows = 64

        def fn():
            oracle.fwht_roundtrip(X[:rows])
        return fn, 8 * rows * K, "%d of the 512 rows of one batch" % rows, "GB/s"
    if workload in ("prefill", "fused", "sweep"):
        if workload == "prefill":
            M, N, K, per_row = 2048, 11008, 4096, False
            W, X = S.prefill(M, N, K, seed=0)
        elif workload == "fused":
            M, N, K, per_row = 512, 5632, 2048, False
            W, X = S.fused(M, N, K, seed=0)
        else:
            M, N, K, per_row = 4096, 8192, 8192, True
            W, X = S.sweep_weights(N, K, seed=0), S.sweep_acts(64, K, seed=0)
        rows = 8
        Xs = X[:rows]
        packed, gamma = oracle.quantize_pack(W, per_row=per_row)

        def fn():
            if workload == "fused":
                oracle.bitlinear(Xs, packed, gamma, per_row)
            else:
                xq, sx, _ = oracle.act_quant(Xs)
                oracle.dequant(oracle.matmul_addsub(xq, packed), gamma, sx, per_row)
        return fn, 2 * rows * N * K, "%d tokens of the contraction (weights pre-packed)" % rows, "TOPS"
    raise SystemExit(workload)


def cpu_baseline(workload, budget_s=15.0):
    fn, work, what, unit = oracle_sample(workload)
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or el / n * (n + 1) > 2 * budget_s:
            break
    scale = 1e9 if unit == "GB/s" else 1e12
    return {"value": round(work * n / el / scale, 6), "unit": unit, "cores": 1, "kind": "oracle",
            "sample": "%s, x%d, %.1f s, single-threaded C" % (what, n, el), "host_cores": os.cpu_count()}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle

    oracle.build()
    fn, work, what, unit = oracle_sample(args.workload)
    for _ in range(args.warmup):
        fn()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fn()
    el = time.perf_counter() - t0
    scale = 1e9 if unit == "GB/s" else 1e12
    v = work * args.steps / el / scale
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if args.workload == "train" else "int8",
        "data": "synthetic", "config": dict(config_for(args.workload, args.layers, world, args.layout), sample=what),
        "cpu_baseline": {"value": round(v, 6), "unit": unit, "cores": 1, "kind": "oracle",
                         "sample": what + " per step"},
        "e2e": {"value": round(v, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ---------------------------------------------------------------------------
def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def allreduce_max(v, world):
    if world <= 1:
        return v
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "prefill", "fused", "sweep", "roundtrip", "mlp", "train"])
    ap.add_argument("--bias", action="store_true",
                    help="contractions through tq_ternary_gemm_ex with a bias (the extra epilogue)")
    ap.add_argument("--ratio", type=float, default=0.0,
                    help="threshold ternarisation w > ratio * gamma (0: the round/clamp rule)")
    ap.add_argument("--layout", default="foundry", choices=LAYOUTS,
                    help="packed-code layout: Foundry's (default) or Hetman-2b's Format 0 / Format 1")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=0, help="ring of distinct layers (0: workload default)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
