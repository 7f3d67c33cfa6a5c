"""Run one kernel of the hot path a few times on a chosen shape -- the small,
self-contained command that ncu captures are taken on.

    python -m ternary_bit_linear_b200.profile_case --kernel gemv --M 8 --N 4096 --K 4096 --reps 3 [--ready]
    python -m ternary_bit_linear_b200.profile_case --kernel grouped --G 64 --M 8 --N 4096 --K 4096 --reps 3

Training kernels: bwd (input gradient, dY [M][N] against the packed [N][K]),
ste and flip (latent weights / gradient [N][K]).

Inputs are random device tensors of the workloads' distributions (values do
not affect timing); every call goes through the C ABI.  Exits non-zero if a
call fails or the device status word reports a timeout.
"""
from __future__ import annotations

import argparse

import torch

import ternary_bit_linear_b200 as tq


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", required=True,
                    choices=["pack_row", "pack_tensor", "act", "fwht", "gemv", "gemm", "grouped", "fused", "bwd", "ste",
                             "flip"])
    ap.add_argument("--G", type=int, default=8, help="layers per grouped call")
    ap.add_argument("--M", type=int, default=8)
    ap.add_argument("--N", type=int, default=4096)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--ready", action="store_true",
                    help="contractions with TQ_FLAG_INPUTS_READY (independent calls: the streaming GEMV)")
    a = ap.parse_args()
    tq.load()
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    M, N, K = a.M, a.N, a.K
    W = torch.randn((N, K), generator=g, device=dev) * 0.02
    X = torch.randn((M, K), generator=g, device=dev)
    per_row = a.kernel != "pack_tensor"
    packed, gamma = tq.quantize_ternary_pack(W, per_row=per_row)
    xq, sx, rs = tq.quantize_act_int8(X)
    y = torch.empty((M, N), device=dev)
    flags = tq.GAMMA_PER_ROW if per_row else 0
    ws = torch.empty((max(16, tq.fused_workspace_bytes(M, K, tq.FLAG_FWHT | tq.FLAG_RMSNORM)),),
                     dtype=torch.uint8, device=dev)
    pws = torch.empty((max(16, tq.pack_workspace_bytes(N, K, flags)),), dtype=torch.uint8, device=dev)
    Xr = torch.empty_like(X)
    if a.kernel == "grouped":  # G distinct packed copies of the layer, one activation batch per layer
        Pg = [packed.clone() for _ in range(a.G)]
        Gg = [gamma.clone() for _ in range(a.G)]
        Xg = X.unsqueeze(0).expand(a.G, M, K).contiguous()
        Yg = torch.empty((a.G, M, N), device=dev)
        gfl = flags | tq.FLAG_WEIGHTS_STATIC | tq.FLAG_INPUTS_READY
        gws = torch.empty((tq.grouped_workspace_bytes(a.G, M, K, gfl),), dtype=torch.uint8, device=dev)
    if a.kernel in ("bwd", "ste", "flip"):
        dY = torch.randn((M, N), generator=g, device=dev)
        dX = torch.empty((M, K), device=dev)
        bws = torch.empty((tq.backward_input_workspace_bytes(M, N),), dtype=torch.uint8, device=dev)
        G = torch.randn((N, K), generator=g, device=dev)
        GW = torch.empty_like(G)
        state = tq.seed(42)
    torch.cuda.synchronize()
    for _ in range(a.reps):
        if a.kernel in ("pack_row", "pack_tensor"):
            tq.quantize_ternary_pack_(W, flags, packed, gamma, pws)
        elif a.kernel == "act":
            tq.quantize_act_int8_(X, 0, 0.05, 40.0, xq, sx, rs)
        elif a.kernel == "fwht":
            tq.fwht512_(X, Xr)
        elif a.kernel in ("gemv", "gemm"):
            ready = tq.FLAG_WEIGHTS_STATIC | tq.FLAG_INPUTS_READY if a.ready else 0
            tq.ternary_gemm_(xq, sx, rs, packed, gamma, flags | ready, y)
        elif a.kernel == "grouped":
            tq.bitlinear_grouped_(Xg, Pg, Gg, gfl, Yg, gws)
        elif a.kernel == "bwd":
            tq.ternary_backward_input_(dY, packed, gamma, flags, dX, bws)
        elif a.kernel == "ste":
            tq.ste_backward_(G, W, gamma, flags, GW)
        elif a.kernel == "flip":
            state = tq.ternary_stochastic_flip_(packed, G, 0.05, state)
        else:
            tq.bitlinear_fused_(X, packed, gamma, tq.FLAG_FWHT | tq.FLAG_RMSNORM, y, ws)
    torch.cuda.synchronize()
    st = tq.device_status()
    if st != 0:
        raise SystemExit(f"device status {st}")
    print(f"{a.kernel} M={M} N={N} K={K} reps={a.reps} ok")


if __name__ == "__main__":
    main()
