"""Benchmark of the ternary linear layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload metric|decode|prefill|fused|sweep|pack|roundtrip|mlp|train]
                    [--decode-group G] [--layout foundry|format0|format1] [--ratio R] [--bias]
                    [--impl ours|reference]

One JSON line on rank 0.  The metric has two halves, and the default run
("metric") measures both:

  * decode (the line's value): packed-weight HBM GB/s of the small-M
    contraction.  K = N = 4096, per-row gamma, W ~ N(0, 0.02), activations
    ~ N(0, 1) with 0.1 % outliers x20, token batches M = 1 and M = 8.  A ring
    of L = 64 distinct layers (256 MiB of packed weights, twice L2) is packed
    once; a step quantises every layer's activation batches per token and runs
    them through the layer's GEMV.  Metric: algorithmic bytes of the step
    (packed weights, gamma, x_q, s_x, rowsum, y and the fp32 activations the
    quantiser reads) / step time.
  * prefill (the "prefill" record): int8 tensor-core TOPS of the M = 2048,
    N = 11008, K = 4096 GEMM (per-tensor gamma) over a ring of 4 layers; a
    step quantises the 2048 tokens and runs the GEMM of each layer.
    Metric: 2 M N K / step time.

Packing (gamma reduction, ternarisation, 2-bit packing) happens once per
weight in inference: it is timed in the same run as its own entry ("aux"),
outside the step.  The "pack" workload makes it the step.

The ring's layers have their own weights, activations, outputs and
workspaces, so the calls within one segment are independent: they carry
TQ_FLAG_INPUTS_READY (and TQ_FLAG_WEIGHTS_STATIC for the contractions), which
lets consecutive kernels overlap.  --decode-group G > 1 issues the decode
GEMVs as grouped calls of G same-shape layers (one activation pass and one
GEMV launch per group).  The small-M GEMVs are also timed one call per layer
("per_call") and as a chain of dependent layers ("chain": each kernel waits
for the previous one before reading), outside the step.

Timing: each segment is one CUDA graph; CUDA events between segments on the
launching stream; barrier + synchronize around the timed steps; max over
ranks.  Per-kernel average launch time = segment time / launches.

Other workloads: "fused" (RMSNorm + FWHT + int8 + GEMM, 512 x 5632 x 2048),
"sweep" (M from 1 to 4096 at 8192^2), "pack" (quantise + pack of the 8192^2
per-row and 11008 x 4096 per-tensor weights), "roundtrip" (the FWHT module's
int8 round trip), "mlp" (the clamped SwiGLU block, 512 tokens,
1536 -> 6144 -> 1536) and "train" (input gradient of the prefill layer, STE
of its latent weights, stochastic flip of its codes); --layout, --ratio and
--bias select the packed-code layout, the threshold ternarisation rule and the
bias epilogue.

--impl reference times the CPU oracle (the plain C reference) on a bounded
sample of the same workload, on all of this host's cores.
"""
from __future__ import annotations

import argparse
import concurrent.futures
import hashlib
import json
import os
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
SMS = 148
I8_MAC_PER_CLK_SM = 8192  # tcgen05 kind::i8 rate per SM, measured with an MMA-only probe


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
    "pack": ["tq_pack.cuh"], "act_quant": ["tq_act.cuh"], "gemv": ["tq_gemv.cuh", "tq_gemv_group.cuh", "tq_act.cuh"],
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
class Seg:
    """One CUDA graph of a workload: `units` kernel invocations of `kname`
    (algorithmic bytes or ops `work` in total), `launches` GPU kernel
    launches; `in_step`: part of the timed step (else timed on its own)."""

    def __init__(self, label, kname, units, work, launches, fns, in_step=True):
        self.label, self.kname, self.units, self.work = label, kname, units, work
        self.launches, self.fns, self.in_step = launches, fns, in_step


TENSOR_KERNELS = ("gemm", "fused", "mlp", "bwd")


class Workload:
    """Builds device buffers and the per-segment launch lists of one step."""

    def __init__(self, name, tq, S, torch, dev, layers, layout=0, ratio=0.0, bias=False, group=1):
        self.name, self.tq, self.torch, self.dev = name, tq, torch, dev
        self.layout, self.ratio, self.group = layout, ratio, group
        f32, u8, i8, i32 = torch.float32, torch.uint8, torch.int8, torch.int32
        self.segs = []
        self.bias = None
        self.chains = []    # (label, launches, bytes per launch, [fns]): dependent-layer GEMV chains
        self.L = layers
        if name == "decode":
            N = K = 4096
            self.N, self.K, self.Ms = N, K, [1, 8]
            self.per_row = True
            W = torch.from_numpy(S.decode_weights(N, K, seed=0))
            self.W = [W.to(dev) for _ in range(layers)]  # distinct buffers, same values
            self.X = {M: torch.from_numpy(S.decode_acts(M, K, seed=0)) for M in self.Ms}
        elif name == "prefill":
            M, N, K = 2048, 11008, 4096
            self.N, self.K, self.Ms = N, K, [M]
            self.per_row = False
            W, X = S.prefill(M, N, K, seed=0)
            W = torch.from_numpy(W)
            self.W = [W.to(dev) for _ in range(layers)]
            self.X = {M: torch.from_numpy(X)}
        elif name == "fused":
            M, N, K = 512, 5632, 2048
            self.N, self.K, self.Ms = N, K, [M]
            self.per_row = False
            W, X = S.fused(M, N, K, seed=0)
            W = torch.from_numpy(W)
            self.W = [W.to(dev) for _ in range(layers)]
            self.X = {M: torch.from_numpy(X)}
        elif name == "sweep":
            N = K = 8192
            self.N, self.K, self.Ms = N, K, [1, 4, 16, 64, 512, 4096]
            self.per_row = True
            W = torch.from_numpy(S.sweep_weights(N, K, seed=0))
            self.W = [W.to(dev) for _ in range(layers)]
            self.X = {M: torch.from_numpy(S.sweep_acts(M, K, seed=0)) for M in self.Ms}
        elif name == "pack":
            self._build_pack(S, layers)
            return
        elif name == "mlp":
            self._build_mlp(S, layers)
            return
        elif name == "train":
            self._build_train(S, layers)
            return
        elif name == "roundtrip":
            # the FWHT module's int8 round trip on the fused configuration's activations
            M, K = 512, 2048
            self.N, self.K, self.Ms = 0, K, [M]
            self.per_row = False
            X = torch.from_numpy(S.fused(M, 16, K, seed=0)[1])
            self.X = {M: X}
            self.Xd = {M: [X.to(dev) for _ in range(layers)]}
            self.yr = [torch.empty((M, K), dtype=f32, device=dev) for _ in range(layers)]
            self.y = {M: self.yr}
            self.segs.append(Seg("fwht roundtrip", "roundtrip", layers, layers * 8 * M * K, layers, [
                lambda l=l: tq.fwht_roundtrip_(self.Xd[M][l], self.yr[l], 0.05, 40.0) for l in range(layers)]))
            return
        else:
            raise SystemExit(f"unknown workload {name}")
        N, K, L = self.N, self.K, layers
        # packed-code layout (0 Foundry, 1 Hetman-2b Format 0, 2 Format 1) on every pack and contraction
        self.flags = (tq.GAMMA_PER_ROW if self.per_row else 0) | (layout << 7)
        # the ring's layers have their own weights, activations and outputs:
        # independent calls, so the contractions may overlap one another
        self.ready_flags = self.flags | tq.FLAG_WEIGHTS_STATIC | tq.FLAG_INPUTS_READY
        self.packed = [torch.empty((N, K // 4), dtype=u8, device=dev) for _ in range(L)]
        self.gamma = [torch.empty((N if self.per_row else 1,), dtype=f32, device=dev) for _ in range(L)]
        nws = tq.pack_workspace_bytes(N, K, self.flags)
        self.pack_ws = [torch.empty((max(nws, 16),), dtype=u8, device=dev) for _ in range(L)]
        # every layer's activations and outputs in one contiguous [L][M][.] buffer per batch size
        # (each layer uses its own slice): the end-to-end run copies them in and out in one piece
        self.Xall = {M: x.unsqueeze(0).expand(L, *x.shape).contiguous().to(dev) for M, x in self.X.items()}
        self.Yall = {M: torch.empty((L, M, N), dtype=f32, device=dev) for M in self.Ms}
        self.Xd = {M: [self.Xall[M][l] for l in range(L)] for M in self.Ms}
        self.y = {M: [self.Yall[M][l] for l in range(L)] for M in self.Ms}
        self.xq = {M: [torch.empty((M, K), dtype=i8, device=dev) for _ in range(L)] for M in self.Ms}
        self.sx = {M: [torch.empty((M,), dtype=f32, device=dev) for _ in range(L)] for M in self.Ms}
        self.rs = {M: [torch.empty((M,), dtype=i32, device=dev) for _ in range(L)] for M in self.Ms}

        # packing: once per weight (aux, outside the step)
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
        self.segs.append(Seg("pack", "pack", L, L * pack_bytes, L * pack_launches, pack_fns, in_step=False))
        if name == "fused":
            M = self.Ms[0]
            fl = tq.FLAG_FWHT | tq.FLAG_RMSNORM
            self.fused_flags = fl | tq.FLAG_WEIGHTS_STATIC | tq.FLAG_INPUTS_READY | (layout << 7)
            self.fused_ws = [torch.empty((tq.fused_workspace_bytes(M, K, fl),), dtype=u8, device=dev)
                             for _ in range(L)]
            self.segs.append(Seg("fused M=%d" % M, "fused", L, L * 2 * M * N * K, 2 * L, [
                lambda l=l: tq.bitlinear_fused_(self.Xd[M][l], self.packed[l], self.gamma[l],
                                                self.fused_flags, self.y[M][l], self.fused_ws[l])
                for l in range(L)]))
            return
        self.bias = [torch.full((N,), 0.25, dtype=f32, device=dev) for _ in range(L)] if bias else None
        for M in self.Ms:
            gemv = M <= 16
            act_bytes = 4 * M * K + M * K + 8 * M
            # the contraction's algorithmic bytes (GEMV) or ops (GEMM)
            work = (N * K // 4 + 4 * N * (1 if self.per_row else 0) + M * K + 8 * M + 4 * M * N) if gemv \
                else 2 * M * N * K
            if gemv and group > 1:
                self._grouped_gemv(M, act_bytes, work, group, True)
                if group < L and L <= 64:  # the whole ring in one call, for comparison
                    self._grouped_gemv(M, act_bytes, work, L, False)
            else:
                self.segs.append(Seg("act M=%d" % M, "act_quant", L, L * act_bytes, L, [
                    lambda M=M, l=l: tq.quantize_act_int8_(self.Xd[M][l], tq.FLAG_INPUTS_READY, 0.05, 40.0,
                                                           self.xq[M][l], self.sx[M][l], self.rs[M][l])
                    for l in range(L)]))
                self.segs.append(Seg(("gemv M=%d" if gemv else "gemm M=%d") % M, "gemv" if gemv else "gemm", L,
                                     L * work, L, self._contraction_fns(M, self.ready_flags)))
            if gemv:
                if group > 1:  # one call per layer, outside the step, for comparison
                    self.segs.append(Seg("gemv M=%d per call" % M, "gemv", L, L * work, L,
                                         self._contraction_fns(M, self.ready_flags), in_step=False))
                self.chains.append(("gemv M=%d" % M, L, work, self._contraction_fns(M, self.flags | tq.FLAG_WEIGHTS_STATIC)))

    def _contraction_fns(self, M, flags):
        tq = self.tq
        if self.bias is not None:  # the extra epilogue (y + bias[n]) through tq_ternary_gemm_ex
            return [lambda l=l: tq.ternary_gemm_ex_(self.xq[M][l], self.sx[M][l], self.rs[M][l], self.packed[l],
                                                     self.gamma[l], flags, self.y[M][l], bias=self.bias[l])
                    for l in range(self.L)]
        return [lambda l=l: tq.ternary_gemm_(self.xq[M][l], self.sx[M][l], self.rs[M][l], self.packed[l],
                                              self.gamma[l], flags, self.y[M][l])
                for l in range(self.L)]

    def _grouped_gemv(self, M, act_bytes, work, G, in_step):
        """Groups of G consecutive ring layers, each with its own activation
        batch: one call (activation pass + GEMV launch) per group.  Work per
        layer: the packed weights, gamma, the fp32 activations read and the
        outputs written, plus the x_q, s_x and rowsum the activation pass
        writes and the GEMV reads."""
        tq, torch, L, K, N = self.tq, self.torch, self.L, self.K, self.N
        assert L % G == 0
        ng = L // G
        # per group: contiguous slices x [G][M][K] and y [G][M][N] of the ring's buffers
        gx = [self.Xall[M][g * G:(g + 1) * G] for g in range(ng)]
        gy = [self.Yall[M][g * G:(g + 1) * G] for g in range(ng)]
        wsz = tq.grouped_workspace_bytes(G, M, K, 0)
        gws = [torch.empty((max(wsz, 16),), dtype=torch.uint8, device=self.dev) for _ in range(ng)]
        self.__dict__.setdefault("keep", []).append((gx, gy, gws))
        fl = self.ready_flags
        fns = [lambda g=g: tq.bitlinear_grouped_(gx[g], self.packed[g * G:(g + 1) * G], self.gamma[g * G:(g + 1) * G],
                                                 fl, gy[g], gws[g])
               for g in range(ng)]
        self.segs.append(Seg("gemv M=%d grouped x%d" % (M, G), "gemv", L, L * (work + act_bytes), 2 * ng, fns,
                             in_step=in_step))

    def _build_pack(self, S, layers):
        """Quantise + pack as the step: the 8192^2 sweep weight per row and the
        11008 x 4096 prefill weight per tensor, each over a ring of layers."""
        tq, torch, dev = self.tq, self.torch, self.dev
        self.N, self.K, self.Ms, self.per_row = 8192, 8192, [], True
        self.X, self.y = {}, {}
        for label, W, per_row in (("pack per-row 8192x8192", S.sweep_weights(8192, 8192, seed=0), True),
                                  ("pack per-tensor 11008x4096", S.prefill(1, 11008, 4096, seed=0)[0], False)):
            N, K = W.shape
            fl = (tq.GAMMA_PER_ROW if per_row else 0) | (self.layout << 7) | tq.FLAG_INPUTS_READY
            Wd = [torch.from_numpy(W).to(dev) for _ in range(layers)]
            P = [torch.empty((N, K // 4), dtype=torch.uint8, device=dev) for _ in range(layers)]
            g = [torch.empty((N if per_row else 1,), dtype=torch.float32, device=dev) for _ in range(layers)]
            ws = [torch.empty((max(16, tq.pack_workspace_bytes(N, K, fl)),), dtype=torch.uint8, device=dev)
                  for _ in range(layers)]
            self.__dict__.setdefault("keep", []).append((Wd, P, g, ws))
            work = 4 * N * K + N * K // 4 + 4 * (N if per_row else 1)
            self.segs.append(Seg(label, "pack", layers, layers * work, layers * (1 if per_row else 2), [
                lambda l=l, Wd=Wd, P=P, g=g, ws=ws, fl=fl: tq.quantize_ternary_pack_(Wd[l], fl, P[l], g[l], ws[l])
                for l in range(layers)]))

    def _build_mlp(self, S, layers):
        # Hetman-2b's clamped SwiGLU block: d_model 1536, d_ffn 4 * 1536, 512 tokens
        tq, torch, dev, layout = self.tq, self.torch, self.dev, self.layout
        M, D, F = 512, 1536, 6144
        self.N, self.K, self.Ms, self.per_row = D, D, [M], False
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
        self.segs.append(Seg("pack", "pack", 3 * layers, layers * pack_bytes, 6 * layers, [
            lambda l=l, i=i: tq.quantize_ternary_pack_(self.W3[l][i], (layout << 7), self.P3[l][i][0],
                                                      self.P3[l][i][1], self.pws3[l])
            for l in range(layers) for i in range(3)], in_step=False))
        ops = 2 * M * 3 * D * F
        self.segs.append(Seg("mlp M=%d" % M, "mlp", layers, layers * ops, 5 * layers, [
            lambda l=l: tq.swiglu_mlp_(self.Xd[M][l], self.P3[l][0], self.P3[l][1], self.P3[l][2],
                                       fl | tq.FLAG_WEIGHTS_STATIC, self.y[M][l], self.mws[l])
            for l in range(layers)]))

    def _build_train(self, S, layers):
        # one training step of the prefill layer (2048 tokens, 4096 -> 11008 features): the input
        # gradient dX = (dY * gamma) W, the STE gradient of the latent weights and the
        # stochastic flip of the packed codes (the weight-gradient GEMM X^T dY is a plain float
        # GEMM outside this library: its output G is a synthetic input here)
        tq, torch, dev, layout = self.tq, self.torch, self.dev, self.layout
        f32, u8 = torch.float32, torch.uint8
        M, N, K = 2048, 11008, 4096
        self.N, self.K, self.Ms, self.per_row = N, K, [M], False
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
        self.segs.append(Seg("backward dX M=%d" % M, "bwd", layers, layers * 2 * M * N * K, 2 * layers, [
            lambda l=l: tq.ternary_backward_input_(self.Xd[M][l], self.packed[l], self.gamma[l], fl,
                                                   self.y[M][l], self.bws[l])
            for l in range(layers)]))
        self.segs.append(Seg("ste", "ste", layers, layers * 12 * N * K, layers, [
            lambda l=l: tq.ste_backward_(self.G[l], self.Wl[l], self.gamma[l], 0, self.gw[l])
            for l in range(layers)]))
        self.segs.append(Seg("flip", "flip", layers, layers * (4 * N * K + N * K // 2), layers, [
            lambda l=l: tq.ternary_stochastic_flip_(self.packed[l], self.G[l], 0.05, self.rng, fl)
            for l in range(layers)]))

    def bytes_metric(self):
        return self.name in ("decode", "roundtrip", "pack")

    def step_work(self):
        """Algorithmic bytes (decode, roundtrip, pack) or ops of one step."""
        if self.bytes_metric():
            return sum(s.work for s in self.segs if s.in_step)
        return sum(s.work for s in self.segs if s.in_step and s.kname in TENSOR_KERNELS)


WORKLOAD_SHAPES = {  # name -> (Ms, N, K, default ring of layers, per_row)
    "decode": ([1, 8], 4096, 4096, 64, True),
    "prefill": ([2048], 11008, 4096, 4, False),
    "fused": ([512], 5632, 2048, 8, False),
    "sweep": ([1, 4, 16, 64, 512, 4096], 8192, 8192, 8, True),
    "pack": ([], 8192, 8192, 6, True),
    "roundtrip": ([512], 0, 2048, 64, False),
    "mlp": ([512], 1536, 1536, 8, False),
    "train": ([2048], 11008, 4096, 4, False),
}

LAYOUTS = ["foundry", "format0", "format1"]  # packed-code layouts, flag value = index << 7


def config_for(name, layers, world, layout="foundry", ratio=0.0, bias=False, group=1):
    Ms, N, K, L, per_row = WORKLOAD_SHAPES[name]
    L = layers or L
    grp = (", GEMV calls grouped %d layers per call (each layer its own activation batch)" % group
           if group > 1 else ", one GEMV call per layer")
    desc = {"decode": "decode GEMV: K=N=4096, per-row gamma, M in {1, 8}, ring of %d layers%s" % (L, grp),
            "prefill": "prefill GEMM: M=2048, N=11008, K=4096, per-tensor gamma, ring of %d layers" % L,
            "fused": "fused BitLinear: M=512, N=5632, K=2048, RMSNorm+FWHT-512, ring of %d layers" % L,
            "sweep": "M sweep over K=N=8192, per-row gamma, ring of %d layers%s" % (L, grp),
            "pack": "quantise+pack: 8192x8192 per-row (Laplace) and 11008x4096 per-tensor, ring of %d each" % L,
            "roundtrip": "FWHT module int8 round trip: 512 x 2048 Student-t(3), ring of %d batches" % L,
            "mlp": "clamped SwiGLU block of 3 BitLinears: 512 tokens, d_model 1536, d_ffn 6144, ring of %d" % L,
            "train": "training step of the prefill layer: dX = (dY gamma) W (M=2048, N=11008, K=4096), STE of "
                     "the latent weights, stochastic flip (T=0.05), ring of %d layers" % L}[name]
    if name == "train":
        l2 = ("inputs larger than L2 (no flush): per layer dY %d MiB, latent weights and their gradient "
              "2 x %d MiB, packed %d MiB" % (Ms[0] * N * 4 >> 20, N * K * 4 >> 20, N * K // 4 >> 20))
    elif name == "pack":
        l2 = "inputs larger than L2 (no flush): fp32 weights %d MiB per step" % (L * (8192 * 8192 + 11008 * 4096) * 4 >> 20)
    else:
        l2 = "inputs larger than L2 (no flush): packed weights %d MiB per step (packed once, outside the step)" % (
            L * N * K // 4 >> 20)
    return {"workload": desc, "M": Ms, "N": N, "K": K, "layers": L,
            "gamma": "per-row" if per_row else "per-tensor", "layout": layout,
            "ternarise": "threshold w > %g * gamma" % ratio if ratio > 0 else "round/clamp",
            "epilogue": "y + bias (tq_ternary_gemm_ex)" if bias else "y", "l2": l2,
            "parallelism": "replicas x%d" % world if world > 1 else "single GPU"}


def line_config(args, world):
    """`config` of the JSON line (both arms print the same one)."""
    main = "decode" if args.workload == "metric" else args.workload
    group = min(args.decode_group, args.layers or WORKLOAD_SHAPES[main][3]) if main in ("decode", "sweep") else 1
    cfg = config_for(main, args.layers, world, args.layout, args.ratio, args.bias, group)
    if args.workload == "metric":
        cfg["workload"] = "metric: " + cfg["workload"] + "; prefill GEMM record: M=2048, N=11008, K=4096"
    return cfg


# ---------------------------------------------------------------------------
# measurement
# ---------------------------------------------------------------------------
def capture(torch, stream, fns):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for fn in fns:
            fn()
    return g


def int8_peaks(pk, sm_mhz):
    """Two int8 dense peaks (TOPS): the measured bf16 burst x the nominal
    int8/bf16 ratio, and the clock-derived rate (SMs x MAC/clk/SM x 2 x the
    median SM clock sampled during the timed region)."""
    nominal = pk["bf16"] * INT8_OVER_BF16
    clock = 2 * I8_MAC_PER_CLK_SM * SMS * sm_mhz * 1e6 / 1e12 if sm_mhz else None
    return nominal, clock


def kernel_entry(seg, per_launch_ms, pk, sm_mhz):
    if seg.kname in TENSOR_KERNELS:
        ach = seg.work / seg.units / (per_launch_ms * 1e-3) / 1e12
        if seg.kname == "bwd":  # fp16 operands on the tensor cores
            return {"bound": "tensor", "achieved": round(ach, 2), "peak": round(pk["bf16"], 1), "unit": "TFLOP/s",
                    "frac": round(ach / pk["bf16"], 4), "us_per_launch": round(per_launch_ms * 1e3, 3)}
        nominal, clock = int8_peaks(pk, sm_mhz)
        e = {"bound": "tensor", "achieved": round(ach, 2), "peak": round(nominal, 1), "unit": "TOPS",
             "frac": round(ach / nominal, 4), "us_per_launch": round(per_launch_ms * 1e3, 3)}
        if clock:
            e["peak_clock"] = round(clock, 1)
            e["frac_clock"] = round(ach / clock, 4)
        return e
    ach = seg.work / seg.units / (per_launch_ms * 1e-3) / 1e9
    e = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm"], "unit": "GB/s",
         "frac": round(ach / pk["hbm"], 4), "us_per_launch": round(per_launch_ms * 1e3, 3)}
    if seg.kname == "flip":  # the xorshift64 chain keeps the ALU pipe busy before HBM
        e["limiter"] = "alu pipe"
    return e


def roofline_of(wl, seg, kernels, pk):
    """The roofline record of the step's dominant contraction (else its
    longest segment)."""
    k = kernels[seg.label]
    r = {"bound": k["bound"], "achieved": k["achieved"], "peak": k["peak"], "unit": k["unit"], "frac": k["frac"],
         "traffic": traffic_for(seg.kname + ":" + wl.name), "kernel": seg.label}
    if k["bound"] == "hbm":
        r["peak_source"] = pk["source"] + " hbm_gbs (copy, burst)"
        if seg.kname == "gemv":
            r["algorithmic_bytes"] = (
                "per layer of the grouped call (activation pass + GEMV): packed N*K/4 + gamma 4N + fp32 "
                "activations 4MK + x_q written and read 2MK + s_x, rowsum written and read 16M + y 4MN"
                if "grouped" in seg.label else
                "per layer: packed N*K/4 + gamma 4N + x_q M*K + s_x, rowsum 8M + y 4MN")
    elif seg.kname == "bwd":
        r["peak_source"] = pk["source"] + " bf16_tflops (fp16 operands)"
    else:
        r["peak_source"] = pk["source"] + " bf16_tflops x2 (nominal int8/bf16 ratio); peak_clock = 148 SMs x " \
                           "8192 MAC/clk x 2 x median SM clock of the timed region"
        for key in ("peak_clock", "frac_clock"):
            if key in k:
                r[key] = k[key]
    return r


def measure(args, wl, torch, tq, stream, world, local_rank):
    """Warm up, time the step (its segments' graphs back to back), then the
    aux segments and chains on their own.  Returns the record of this workload."""
    step_segs = [s for s in wl.segs if s.in_step]
    aux_segs = [s for s in wl.segs if not s.in_step]
    with torch.cuda.stream(stream):
        for seg in wl.segs:  # eager warm-up of every launch (aux first: it packs the weights)
            if not seg.in_step:
                for fn in seg.fns:
                    fn()
        for seg in step_segs:
            for fn in seg.fns:
                fn()
        torch.cuda.synchronize()
        graphs = [capture(torch, stream, s.fns) for s in step_segs]
        aux_graphs = [capture(torch, stream, s.fns) for s in aux_segs]
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            for g in graphs:
                g.replay()
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
    total_ms = allreduce_max(float(seg_ms.sum()), world)
    ms_per_step = total_ms / args.steps
    assert tq.device_status(stream) == 0
    clocks = sampler.summary()

    pk = peaks()
    kernels = {}
    for seg, ms in zip(step_segs, seg_ms):
        kernels[seg.label] = kernel_entry(seg, ms / args.steps / seg.units, pk, clocks["sm_mhz"])
    aux = {}
    reps = max(3, min(args.steps, 20))
    for seg, g in zip(aux_segs, aux_graphs):
        with torch.cuda.stream(stream):
            for _ in range(2):
                g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier(world)
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        ms = allreduce_max(e0.elapsed_time(e1), world) / reps
        aux[seg.label] = kernel_entry(seg, ms / seg.units, pk, clocks["sm_mhz"])
    assert tq.device_status(stream) == 0

    contr = [(s, ms) for s, ms in zip(step_segs, seg_ms) if s.kname in ("gemv",) + TENSOR_KERNELS]
    dom = max(contr or list(zip(step_segs, seg_ms)), key=lambda t: t[1])[0]
    work = wl.step_work() * world
    if wl.bytes_metric():
        value, unit = work / (ms_per_step * 1e-3) / 1e9, "GB/s"
    else:
        value, unit = work / (ms_per_step * 1e-3) / 1e12, ("TFLOP/s" if wl.name == "train" else "TOPS")
    rec = {"value": round(value, 2), "unit": unit, "ms_per_step": round(ms_per_step, 5),
           "roofline": roofline_of(wl, dom, kernels, pk), "kernels": kernels,
           "gpu_launches": sum(s.launches for s in step_segs) * args.steps, "clocks": clocks}
    if aux:
        rec["aux"] = aux
    rec["e2e"] = run_e2e(args, wl, torch, stream, graphs, world)
    chain = run_chains(args, wl, tq, torch, stream, world)
    if chain:
        rec["chain"] = chain
    del graphs, aux_graphs
    return rec


def run_chains(args, wl, tq, torch, stream, world):
    """Dependent-layer GEMV chains: per-launch time when every kernel waits
    for its predecessor's results (the latency-bound decode case)."""
    res = {}
    pk = peaks()
    for label, launches, work, fns in wl.chains:
        with torch.cuda.stream(stream):
            for fn in fns:
                fn()
            torch.cuda.synchronize()
            g = capture(torch, stream, fns)
            for _ in range(3):
                g.replay()
        torch.cuda.synchronize()
        reps = max(3, min(args.steps, 20))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
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


def run_e2e(args, wl, torch, stream, graphs, world):
    """Same step through the public calls with pinned host inputs copied in and
    the step's outputs copied back inside the timed region."""
    ins, outs = [], []
    for M in wl.Ms:
        if getattr(wl, "Xall", None) is not None:
            ins.append(wl.Xall[M])
            outs.append(wl.Yall[M])
        else:
            ins += wl.Xd[M]
            outs += wl.y[M]
    host_in = [x.cpu().pin_memory() for x in ins]
    host_out = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for y in outs]
    h2d = sum(x.numel() * x.element_size() for x in ins)
    d2h = sum(y.numel() * y.element_size() for y in outs)
    steps = max(3, min(args.steps, 50))

    def one():
        for xd, hx in zip(ins, host_in):
            xd.copy_(hx, non_blocking=True)
        for g in graphs:
            g.replay()
        for y, hy in zip(outs, host_out):
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
    work = wl.step_work() * world
    if wl.bytes_metric():
        v, u = work / (ms * 1e-3) / 1e9, "GB/s"
    else:
        v, u = work / (ms * 1e-3) / 1e12, ("TFLOP/s" if wl.name == "train" else "TOPS")
    return {"value": round(v, 2), "unit": u, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms, 4), "steps": steps}


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
    stream = torch.cuda.Stream(device=dev)
    layout = LAYOUTS.index(args.layout)
    main = "decode" if args.workload == "metric" else args.workload
    group = min(args.decode_group, args.layers or WORKLOAD_SHAPES[main][3]) if main in ("decode", "sweep") else 1
    layers = args.layers or WORKLOAD_SHAPES[main][3]
    wl = Workload(main, tq, S, torch, dev, layers, layout, args.ratio, args.bias, group)
    rec = measure(args, wl, torch, tq, stream, world, local_rank)
    cfg = line_config(args, world)
    prefill = None
    if args.workload == "metric":  # the M >= 512 half of the metric, same run
        del wl
        torch.cuda.empty_cache()
        pl = args.prefill_layers or WORKLOAD_SHAPES["prefill"][3]
        wp = Workload("prefill", tq, S, torch, dev, pl, layout, args.ratio, args.bias)
        prefill = measure(args, wp, torch, tq, stream, world, local_rank)
        prefill["config"] = config_for("prefill", pl, world, args.layout, args.ratio, args.bias)
        del wp

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(main, budget_s=args.cpu_seconds)
    out = {
        "metric": METRIC, "value": rec["value"], "unit": rec["unit"], "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": rec["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if main == "train" else "int8", "data": "synthetic", "config": cfg,
        "roofline": rec["roofline"], "kernels": rec["kernels"], "cpu_baseline": cpu, "e2e": rec["e2e"],
        "gpu_launches": rec["gpu_launches"], "clocks": rec["clocks"],
    }
    for k in ("aux", "chain"):
        if k in rec:
            out[k] = rec[k]
    if prefill is not None:
        out["prefill"] = prefill
    if rank == 0:
        print(json.dumps(out), flush=True)


# ---------------------------------------------------------------------------
# CPU oracle baseline / reference arm
# ---------------------------------------------------------------------------
def _chunks(n, parts):
    b = [n * i // parts for i in range(parts + 1)]
    return [(b[i], b[i + 1]) for i in range(parts) if b[i + 1] > b[i]]


def oracle_sample(workload):
    """One bounded unit of the workload on the oracle: (fn(threads), work, what,
    unit).  fn runs the unit on `threads` host threads, each calling the
    unchanged oracle functions on its own slice of rows (the oracle's C calls
    release the interpreter lock); threads = 1 is the plain sequential oracle."""
    import oracle
    from ternary_bit_linear_b200 import synthetic as S

    def par(threads, n, body):
        if threads <= 1:
            body(0, n)
            return
        with concurrent.futures.ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda c: body(*c), _chunks(n, threads)))

    if workload in ("decode", "metric"):
        N = K = 4096
        W = S.decode_weights(N, K, seed=0)
        Xs = {M: S.decode_acts(M, K, seed=0) for M in (1, 8)}

        packed, gamma = oracle.quantize_pack(W, per_row=True)  # once, as in inference

        def fn(threads):
            q = {M: oracle.act_quant(X) for M, X in Xs.items()}

            def body(r0, r1):  # output rows r0..r1 of the layer
                for M, (xq, sx, _) in q.items():
                    oracle.dequant(oracle.matmul_addsub(xq, packed[r0:r1]), gamma[r0:r1], sx, True)
            par(threads, N, body)
        work = sum(4 * M * K + M * K + 8 * M + N * K // 4 + 4 * N + M * K + 8 * M + 4 * M * N for M in (1, 8))
        return fn, work, "one layer of the decode step: act-quant + GEMV for M=1 and M=8 at 4096x4096", "GB/s"
    if workload == "pack":
        N = K = 8192
        W = S.sweep_weights(N, K, seed=0)[:1024]

        def fn(threads):
            par(threads, W.shape[0], lambda r0, r1: oracle.quantize_pack(W[r0:r1], per_row=True))
        return fn, W.shape[0] * (4 * K + K // 4 + 4), "1024 of the 8192 rows of the per-row 8192^2 pack", "GB/s"
    if workload == "mlp":
        M, D, F = 512, 1536, 6144
        X = S.fused(M, 16, D, seed=0)[1]
        shapes = [(F, D), (F, D), (D, F)]
        packs = [oracle.quantize_pack(S.normal(sh, 0.02, 7 + i, sh[0]), per_row=False) for i, sh in enumerate(shapes)]

        def fn(threads):
            rows = 2 * max(1, threads)
            par(threads, rows, lambda r0, r1: oracle.swiglu_mlp(X[r0:r1], packs[0], packs[1], packs[2], False))
        return fn, None, "2 tokens per thread through the block (weights pre-packed)", "TOPS", \
            (lambda threads: 2 * 2 * max(1, threads) * 3 * D * F)
    if workload == "train":
        M, N, K = 2048, 11008, 4096
        W, _ = S.prefill(M, N, K, seed=0)
        dY = S.normal((M, N), 1.0, 160, 0)
        packed, gamma = oracle.quantize_pack(W, per_row=False)

        def fn(threads):
            rows = 2 * max(1, threads)
            par(threads, rows, lambda r0, r1: oracle.backward_input(dY[r0:r1], packed, gamma, False, K))
        return fn, None, "2 tokens per thread of the input gradient (weights pre-packed)", "TFLOP/s", \
            (lambda threads: 2 * 2 * max(1, threads) * N * K)
    if workload == "roundtrip":
        M, K = 512, 2048
        X = S.fused(M, 16, K, seed=0)[1]
        rows = 64

        def fn(threads):
            par(threads, rows, lambda r0, r1: oracle.fwht_roundtrip(X[r0:r1]))
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
            W, X = S.sweep_weights(N, K, seed=0), S.sweep_acts(256, K, seed=0)
        packed, gamma = oracle.quantize_pack(W, per_row=per_row)

        def fn(threads):
            rows = 2 * max(1, threads)

            def body(r0, r1):
                if workload == "fused":
                    oracle.bitlinear(X[r0:r1], packed, gamma, per_row)
                else:
                    xq, sx, _ = oracle.act_quant(X[r0:r1])
                    oracle.dequant(oracle.matmul_addsub(xq, packed), gamma, sx, per_row)
            par(threads, rows, body)
        return fn, None, "2 tokens per thread of the contraction (weights pre-packed)", "TOPS", \
            (lambda threads: 2 * 2 * max(1, threads) * N * K)
    raise SystemExit(workload)


def _time_oracle(sample, threads, budget_s):
    fn, work, what, unit = sample[:4]
    work_of = sample[4] if len(sample) > 4 else (lambda t: work)
    n, t0 = 0, time.perf_counter()
    while True:
        fn(threads)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or el / n * (n + 1) > 2 * budget_s:
            break
    scale = 1e9 if unit == "GB/s" else 1e12
    return work_of(threads) * n / el / scale, n, el, what, unit


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(workload, budget_s=15.0):
    """The oracle on this host: single-threaded, then on all cores (rows split
    across threads).  The line's value is the all-core figure."""
    sample = oracle_sample(workload)
    cores = host_cores()
    v1, n1, el1, what, unit = _time_oracle(sample, 1, budget_s / 2)
    va, na, ela, _, _ = _time_oracle(sample, cores, budget_s / 2)
    return {"value": round(va, 6), "unit": unit, "cores": cores, "kind": "oracle",
            "sample": "%s, x%d in %.1f s on %d threads (rows split across threads; plain C)" % (what, na, ela, cores),
            "single_core": {"value": round(v1, 6), "unit": unit, "cores": 1,
                            "sample": "x%d in %.1f s, one thread" % (n1, el1)}}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle

    oracle.build()
    main = "decode" if args.workload == "metric" else args.workload
    sample = oracle_sample(main)
    cores = host_cores()
    fn, work, what, unit = sample[:4]
    work_of = sample[4] if len(sample) > 4 else (lambda t: work)
    for _ in range(args.warmup):
        fn(cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fn(cores)
    el = time.perf_counter() - t0
    scale = 1e9 if unit == "GB/s" else 1e12
    v = work_of(cores) * args.steps / el / scale
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if main == "train" else "int8", "data": "synthetic",
        "config": dict(line_config(args, world), sample=what),
        "cpu_baseline": {"value": round(v, 6), "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": what + " per step, rows split across %d threads" % cores},
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
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="metric", choices=["metric"] + list(WORKLOAD_SHAPES))
    ap.add_argument("--decode-group", type=int, default=8,
                    help="small-M GEMVs (decode, sweep) as grouped calls of G same-shape layers (1: one call per layer)")
    ap.add_argument("--bias", action="store_true",
                    help="contractions through tq_ternary_gemm_ex with a bias (the extra epilogue)")
    ap.add_argument("--ratio", type=float, default=0.0,
                    help="threshold ternarisation w > ratio * gamma (0: the round/clamp rule)")
    ap.add_argument("--layout", default="foundry", choices=LAYOUTS,
                    help="packed-code layout: Foundry's (default) or Hetman-2b's Format 0 / Format 1")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=0, help="ring of distinct layers (0: workload default)")
    ap.add_argument("--prefill-layers", type=int, default=0, help="ring of the metric run's prefill record")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
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
