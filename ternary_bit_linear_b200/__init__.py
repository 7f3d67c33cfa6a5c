"""Python binding of libtq -- the B200 (sm_100a) ternary linear layer.

Argument marshalling only: every function forwards torch CUDA tensors (their
device pointers) and the current CUDA stream to the C ABI declared in
include/tq.h and raises on a non-OK status.  All arithmetic runs in the CUDA
kernels of libtq.so.  There is no CPU fallback: if the library is missing or
the device is not sm_100, calls fail loudly.

The library is built in-tree by ``python -m ternary_bit_linear_b200.build``
(or ``__graft_entry__.build()``).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

GAMMA_PER_ROW = 1 << 0
FLAG_FWHT = 1 << 1
FLAG_RMSNORM = 1 << 2
FLAG_ETA_CLAMP = 1 << 3
FLAG_SANITIZE_NONFINITE = 1 << 4
FLAG_WEIGHTS_STATIC = 1 << 5
FLAG_INPUTS_READY = 1 << 6
# packed-code layouts (flag bits 7-8): Foundry's (default), Hetman-2b "Format 0" and "Format 1"
ENC_FOUNDRY = 0 << 7
ENC_FORMAT0 = 1 << 7
ENC_FORMAT1 = 2 << 7
ENC_MASK = 3 << 7
FLAG_ACCUMULATE = 1 << 9  # tq_ternary_backward_input: dX += result
FLAG_SHARED_INPUT = 1 << 10  # tq_bitlinear_grouped: one activation batch for all layers

STATUS = {0: "TQ_OK", 1: "TQ_ERR_NULL", 2: "TQ_ERR_SHAPE", 3: "TQ_ERR_ALIGN", 4: "TQ_ERR_ARG",
          5: "TQ_ERR_CUDA", 6: "TQ_ERR_DEVICE", 7: "TQ_ERR_TIMEOUT"}

# Entry points declared in include/tq.h, with their ctypes signatures.
_P, _I64, _U, _F, _I, _SZ = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint, ctypes.c_float,
                              ctypes.c_int, ctypes.c_size_t)
SIGNATURES = {
    "tq_quantize_ternary_pack": (_I, [_P, _I64, _I64, _U, _P, _P, _P, _SZ, _P]),
    "tq_pack_workspace_bytes": (_SZ, [_I64, _I64, _U]),
    "tq_quantize_ternary_pack_threshold": (_I, [_P, _I64, _I64, _U, _F, _P, _P, _P, _SZ, _P]),
    "tq_quantize_ternary_pack_noalloc": (_I, [_P, _I64, _I64, _U, _P, _P, _P]),
    "tq_quantize_ternary_pack_abs_threshold": (_I, [_P, _I64, _I64, _U, _F, _P, _P, _P]),
    "tq_quantize_act_int8": (_I, [_P, _I64, _I64, _U, _F, _F, _P, _P, _P, _P]),
    "tq_fwht512": (_I, [_P, _P, _I64, _I64, _I, _P]),
    "tq_fwht_roundtrip": (_I, [_P, _P, _I64, _I64, _F, _F, _P, _P]),
    "tq_ternary_gemm": (_I, [_P, _P, _P, _P, _P, _U, _I64, _I64, _I64, _P, _P, _P]),
    "tq_ternary_gemm_ex": (_I, [_P, _P, _P, _P, _P, _U, _I64, _I64, _I64, _P, _P, _I, _P, _P, _P]),
    "tq_bitlinear_fused": (_I, [_P, _P, _F, _F, _F, _U, _P, _P, _I64, _I64, _I64, _P, _P, _P,
                                _P, _SZ, _P]),
    "tq_fused_workspace_bytes": (_SZ, [_I64, _I64, _U]),
    "tq_swiglu_mlp": (_I, [_P, _I64, _I64, _I64, _U, _F, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "tq_swiglu_workspace_bytes": (_SZ, [_I64, _I64, _I64, _U]),
    "tq_bitlinear_grouped": (_I, [_P, _I64, _P, _P, _U, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "tq_grouped_workspace_bytes": (_SZ, [_I64, _I64, _I64, _U]),
    "tq_ternary_backward_input": (_I, [_P, _P, _P, _P, _U, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "tq_backward_input_workspace_bytes": (_SZ, [_I64, _I64]),
    "tq_ste_backward": (_I, [_P, _P, _P, _I64, _I64, _F, _U, _P, _P]),
    "tq_ternary_stochastic_flip": (_I, [_P, _P, _I64, _I64, _F, ctypes.POINTER(ctypes.c_uint64), _U, _P]),
    "tq_seed": (None, [ctypes.POINTER(ctypes.c_uint64), ctypes.c_uint64]),
    "tq_get_device_status": (_I, [_P]),
    "tq_selftest_wait_timeout": (_I, [ctypes.c_uint64, _I, _P]),
    "tq_status_string": (ctypes.c_char_p, [_I]),
    "tq_version": (_I, []),
}

_lib = None


class TqError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        msg = _lib.tq_status_string(code).decode() if _lib is not None else ""
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({msg})")


def load():
    """Load libtq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libtq.so not built ({LIB_PATH}); run "
                               "`python -m ternary_bit_linear_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, code: int):
    if code != 0:
        raise TqError(fn, code)


def _need(t, dtype, shape, name):
    if t is None:
        return
    if not t.is_cuda or t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


# ---------------------------------------------------------------------------
# Raw C-ABI calls (tensors in, status checked); the caller owns every buffer.
# ---------------------------------------------------------------------------

def pack_workspace_bytes(N: int, K: int, flags: int) -> int:
    return load().tq_pack_workspace_bytes(N, K, flags)


def fused_workspace_bytes(M: int, K: int, flags: int) -> int:
    return load().tq_fused_workspace_bytes(M, K, flags)


def quantize_ternary_pack_(w, flags, packed, gamma, workspace=None, stream=None):
    import torch

    N, K = w.shape
    _need(w, torch.float32, (N, K), "w")
    _need(packed, torch.uint8, (N, K // 4), "packed")
    _need(gamma, torch.float32, (N if flags & GAMMA_PER_ROW else 1,), "gamma")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("tq_quantize_ternary_pack",
           load().tq_quantize_ternary_pack(_ptr(w), N, K, flags, _ptr(packed), _ptr(gamma),
                                           _ptr(workspace), ws_bytes, _stream(stream)))


def quantize_ternary_pack_threshold_(w, flags, ratio, packed, gamma, workspace=None, stream=None):
    import torch

    N, K = w.shape
    _need(w, torch.float32, (N, K), "w")
    _need(packed, torch.uint8, (N, K // 4), "packed")
    _need(gamma, torch.float32, (N if flags & GAMMA_PER_ROW else 1,), "gamma")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("tq_quantize_ternary_pack_threshold",
           load().tq_quantize_ternary_pack_threshold(_ptr(w), N, K, flags, float(ratio), _ptr(packed),
                                                     _ptr(gamma), _ptr(workspace), ws_bytes,
                                                     _stream(stream)))


def quantize_ternary_pack_abs_threshold_(w, flags, threshold, packed, gamma, stream=None):
    import torch

    N, K = w.shape
    _need(w, torch.float32, (N, K), "w")
    _need(packed, torch.uint8, (N, K // 4), "packed")
    _need(gamma, torch.float32, (1,), "gamma")
    _check("tq_quantize_ternary_pack_abs_threshold",
           load().tq_quantize_ternary_pack_abs_threshold(_ptr(w), N, K, flags, float(threshold), _ptr(packed),
                                                         _ptr(gamma), _stream(stream)))


def quantize_act_int8_(x, flags, eta_min, eta_max, xq, s_x, rowsum, stream=None):
    import torch

    M, K = x.shape
    _need(x, torch.float32, (M, K), "x")
    _need(xq, torch.int8, (M, K), "xq")
    _need(s_x, torch.float32, (M,), "s_x")
    _need(rowsum, torch.int32, (M,), "rowsum")
    _check("tq_quantize_act_int8",
           load().tq_quantize_act_int8(_ptr(x), M, K, flags, eta_min, eta_max, _ptr(xq),
                                       _ptr(s_x), _ptr(rowsum), _stream(stream)))


def fwht512_(x, y, normalize=True, stream=None):
    import torch

    rows, K = x.shape
    _need(x, torch.float32, (rows, K), "x")
    _need(y, torch.float32, (rows, K), "y")
    _check("tq_fwht512", load().tq_fwht512(_ptr(x), _ptr(y), rows, K, int(bool(normalize)),
                                           _stream(stream)))


def ternary_gemm_(xq, s_x, rowsum, packed, gamma, flags, y, acc=None, stream=None):
    import torch

    M, K = xq.shape
    N = packed.shape[0]
    _need(xq, torch.int8, (M, K), "xq")
    _need(packed, torch.uint8, (N, K // 4), "packed")
    _need(y, torch.float32, (M, N), "y")
    _need(acc, torch.int32, (M, N), "acc")
    _check("tq_ternary_gemm",
           load().tq_ternary_gemm(_ptr(xq), _ptr(s_x), _ptr(rowsum), _ptr(packed), _ptr(gamma),
                                  flags, M, N, K, _ptr(y), _ptr(acc), _stream(stream)))


def ternary_gemm_ex_(xq, s_x, rowsum, packed, gamma, flags, y, acc=None, bias=None, acc_bias=None,
                     out_shift=0, stream=None):
    import torch

    M, K = xq.shape
    N = packed.shape[0]
    _need(xq, torch.int8, (M, K), "xq")
    _need(packed, torch.uint8, (N, K // 4), "packed")
    _need(y, torch.float32, (M, N), "y")
    _need(acc, torch.int32, (M, N), "acc")
    _need(bias, torch.float32, (N,), "bias")
    _need(acc_bias, torch.int32, (N,), "acc_bias")
    _check("tq_ternary_gemm_ex",
           load().tq_ternary_gemm_ex(_ptr(xq), _ptr(s_x), _ptr(rowsum), _ptr(packed), _ptr(gamma), flags, M, N, K,
                                     _ptr(bias), _ptr(acc_bias), int(out_shift), _ptr(y), _ptr(acc),
                                     _stream(stream)))


def bitlinear_fused_(x, packed, gamma, flags, y, workspace, rms_gain=None, rms_eps=1e-6,
                     eta_min=0.05, eta_max=40.0, xq_out=None, s_x_out=None, stream=None):
    import torch

    M, K = x.shape
    N = packed.shape[0]
    _need(x, torch.float32, (M, K), "x")
    _need(y, torch.float32, (M, N), "y")
    _check("tq_bitlinear_fused",
           load().tq_bitlinear_fused(_ptr(x), _ptr(rms_gain), rms_eps, eta_min, eta_max, flags,
                                     _ptr(packed), _ptr(gamma), M, N, K, _ptr(y), _ptr(xq_out),
                                     _ptr(s_x_out), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(),
                                     _stream(stream)))


def fwht_roundtrip_(x, y, eta_min=0.05, eta_max=40.0, eta_out=None, stream=None):
    import torch

    rows, K = x.shape
    _need(x, torch.float32, (rows, K), "x")
    _need(y, torch.float32, (rows, K), "y")
    _need(eta_out, torch.float32, (rows,), "eta_out")
    _check("tq_fwht_roundtrip",
           load().tq_fwht_roundtrip(_ptr(x), _ptr(y), rows, K, float(eta_min), float(eta_max), _ptr(eta_out),
                                    _stream(stream)))


def swiglu_workspace_bytes(M: int, d_model: int, d_ffn: int, flags: int) -> int:
    return int(load().tq_swiglu_workspace_bytes(M, d_model, d_ffn, flags))


def grouped_workspace_bytes(G: int, M: int, K: int, flags: int) -> int:
    return int(load().tq_grouped_workspace_bytes(G, M, K, flags))


def bitlinear_grouped_(x, packed, gamma, flags, y, workspace, stream=None):
    """G same-shape layers: x [G, M, K] (or [M, K] with FLAG_SHARED_INPUT),
    packed / gamma: sequences of G device tensors, y [G, M, N]."""
    import torch

    G = len(packed)
    if len(gamma) != G:
        raise ValueError("packed and gamma must have one entry per layer")
    M, K = x.shape[-2], x.shape[-1]
    N = packed[0].shape[0]
    _need(x, torch.float32, (M, K) if flags & FLAG_SHARED_INPUT else (G, M, K), "x")
    _need(y, torch.float32, (G, M, N), "y")
    for p in packed:
        _need(p, torch.uint8, (N, K // 4), "packed")
    arr = ctypes.c_void_p * G
    pp = arr(*[p.data_ptr() for p in packed])
    gp = arr(*[g.data_ptr() for g in gamma])
    _check("tq_bitlinear_grouped",
           load().tq_bitlinear_grouped(_ptr(x), G, ctypes.cast(pp, ctypes.c_void_p), ctypes.cast(gp, ctypes.c_void_p),
                                       flags, M, N, K, _ptr(y), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream)))


def grouped_intermediates(workspace, G: int, M: int, K: int, flags: int) -> dict:
    """x_q (back in plain [Gx, M, K] order), s_x and rowsum from the
    workspace of tq_bitlinear_grouped (the layout the header states)."""
    import torch

    Gx = 1 if flags & FLAG_SHARED_INPUT else G
    al = lambda b: (b + 255) & ~255
    o1 = al(Gx * M * K)
    o2 = o1 + al(Gx * M * 4)
    raw = workspace[:Gx * M * K].view(Gx * M, K // 16, 4, 4)
    c = torch.arange(K // 16, device=workspace.device)
    pos = c ^ (2 * ((c >> 3) & 1))
    xq = raw[:, pos].transpose(2, 3).reshape(Gx, M, K).view(torch.int8)
    sx = workspace[o1:o1 + Gx * M * 4].view(torch.float32).view(Gx, M)
    rs = workspace[o2:o2 + Gx * M * 4].view(torch.int32).view(Gx, M)
    return {"xq": xq, "s_x": sx, "rowsum": rs}


def swiglu_intermediates(workspace, M: int, d_model: int, d_ffn: int) -> dict:
    """Views of what tq_swiglu_mlp leaves in its workspace (the layout the
    header states: eight parts, each starting on a 256-byte boundary)."""
    import torch

    sizes = [(M * d_model, torch.int8, (M, d_model), "xq1"), (M, torch.float32, (M,), "s_x1"),
             (M, torch.int32, (M,), "rowsum1"), (M * d_ffn, torch.float32, (M, d_ffn), "y_gate"),
             (M * d_ffn, torch.float32, (M, d_ffn), "y_up"), (M * d_ffn, torch.int8, (M, d_ffn), "xq2"),
             (M, torch.float32, (M,), "s_x2"), (M, torch.int32, (M,), "rowsum2")]
    out, off = {}, 0
    for n, dt, shape, name in sizes:
        nb = n * torch.tensor([], dtype=dt).element_size()
        out[name] = workspace[off:off + nb].view(dt).view(shape)
        off += (nb + 255) & ~255
    if off > workspace.numel():
        raise ValueError("workspace smaller than tq_swiglu_workspace_bytes")
    return out


def swiglu_mlp_(x, gate, up, down, flags, y, workspace, clamp_val=10.0, act_out=None, stream=None):
    """gate, up, down: (packed, gamma) pairs."""
    import torch

    M, D = x.shape
    F = gate[0].shape[0]
    _need(x, torch.float32, (M, D), "x")
    _need(y, torch.float32, (M, D), "y")
    _need(act_out, torch.float32, (M, F), "act_out")
    _need(gate[0], torch.uint8, (F, D // 4), "gate packed")
    _need(up[0], torch.uint8, (F, D // 4), "up packed")
    _need(down[0], torch.uint8, (D, F // 4), "down packed")
    _check("tq_swiglu_mlp",
           load().tq_swiglu_mlp(_ptr(x), M, D, F, flags, float(clamp_val), _ptr(gate[0]), _ptr(gate[1]),
                                _ptr(up[0]), _ptr(up[1]), _ptr(down[0]), _ptr(down[1]), _ptr(y), _ptr(act_out),
                                _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def backward_input_workspace_bytes(M: int, N: int) -> int:
    return load().tq_backward_input_workspace_bytes(M, N)


def ternary_backward_input_(dY, packed, gamma, flags, dX, workspace, row_scale=None, stream=None):
    import torch

    M, N = dY.shape
    K = packed.shape[1] * 4
    _need(dY, torch.float32, (M, N), "dY")
    _need(packed, torch.uint8, (N, K // 4), "packed")
    _need(gamma, torch.float32, (N if flags & GAMMA_PER_ROW else 1,), "gamma")
    _need(row_scale, torch.float32, (M,), "row_scale")
    _need(dX, torch.float32, (M, K), "dX")
    ws_bytes = workspace.numel() * workspace.element_size()
    _check("tq_ternary_backward_input",
           load().tq_ternary_backward_input(_ptr(dY), _ptr(packed), _ptr(gamma), _ptr(row_scale), flags, M, N, K,
                                            _ptr(dX), _ptr(workspace), ws_bytes, _stream(stream)))


def ste_backward_(grad, w, gamma, flags, out, tau=1.0, stream=None):
    import torch

    N, K = w.shape
    _need(grad, torch.float32, (N, K), "grad")
    _need(w, torch.float32, (N, K), "w")
    _need(gamma, torch.float32, (N if flags & GAMMA_PER_ROW else 1,), "gamma")
    _need(out, torch.float32, (N, K), "out")
    _check("tq_ste_backward", load().tq_ste_backward(_ptr(grad), _ptr(w), _ptr(gamma), N, K, float(tau), flags,
                                                     _ptr(out), _stream(stream)))


def seed(value: int) -> int:
    """fq_seed: the xorshift64 state for `value`."""
    st = ctypes.c_uint64(0)
    load().tq_seed(ctypes.byref(st), ctypes.c_uint64(value))
    return st.value


def ternary_stochastic_flip_(packed, grad, temperature, state: int, flags=0, stream=None) -> int:
    """Flips `packed` in place; returns the generator state after the N*K draws."""
    import torch

    N, K = grad.shape
    _need(grad, torch.float32, (N, K), "grad")
    _need(packed, torch.uint8, (N, K // 4), "packed")
    st = ctypes.c_uint64(state)
    _check("tq_ternary_stochastic_flip",
           load().tq_ternary_stochastic_flip(_ptr(packed), _ptr(grad), N, K, float(temperature), ctypes.byref(st),
                                             flags, _stream(stream)))
    return st.value


def device_status(stream=None) -> int:
    """Synchronises the stream; returns and clears the device status word."""
    return load().tq_get_device_status(_stream(stream))


def selftest_wait_timeout(limit_ns: int, sleeping: bool = False, stream=None):
    """Launch the bounded-wait self-test (a wait that nothing completes, given
    up after limit_ns); the next device_status() reports TQ_ERR_TIMEOUT."""
    _check("tq_selftest_wait_timeout",
           load().tq_selftest_wait_timeout(int(limit_ns), int(bool(sleeping)), _stream(stream)))


# ---------------------------------------------------------------------------
# Allocating conveniences (torch allocates; the kernels compute).
# ---------------------------------------------------------------------------

def quantize_ternary_pack(w, per_row: bool, sanitize: bool = False, stream=None):
    import torch

    N, K = w.shape
    flags = (GAMMA_PER_ROW if per_row else 0) | (FLAG_SANITIZE_NONFINITE if sanitize else 0)
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=w.device)
    gamma = torch.empty((N if per_row else 1,), dtype=torch.float32, device=w.device)
    nws = pack_workspace_bytes(N, K, flags)
    ws = torch.empty((max(nws, 16),), dtype=torch.uint8, device=w.device) if nws else None
    quantize_ternary_pack_(w, flags, packed, gamma, ws, stream)
    return packed, gamma


def quantize_act_int8(x, clamp_eta: bool = False, eta_min: float = 0.05, eta_max: float = 40.0,
                      sanitize: bool = False, stream=None):
    import torch

    M, K = x.shape
    flags = (FLAG_ETA_CLAMP if clamp_eta else 0) | (FLAG_SANITIZE_NONFINITE if sanitize else 0)
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s_x = torch.empty((M,), dtype=torch.float32, device=x.device)
    rowsum = torch.empty((M,), dtype=torch.int32, device=x.device)
    quantize_act_int8_(x, flags, eta_min, eta_max, xq, s_x, rowsum, stream)
    return xq, s_x, rowsum


def fwht512(x, normalize: bool = True, stream=None):
    import torch

    y = torch.empty_like(x)
    fwht512_(x, y, normalize, stream)
    return y


def ternary_gemm(xq, s_x, rowsum, packed, gamma, per_row: bool, with_acc: bool = False,
                 stream=None):
    import torch

    M, N = xq.shape[0], packed.shape[0]
    y = torch.empty((M, N), dtype=torch.float32, device=xq.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=xq.device) if with_acc else None
    ternary_gemm_(xq, s_x, rowsum, packed, gamma, GAMMA_PER_ROW if per_row else 0, y, acc, stream)
    return (y, acc) if with_acc else y


def bitlinear_fused(x, packed, gamma, per_row: bool, rmsnorm: bool = True, fwht: bool = True,
                    rms_gain=None, rms_eps: float = 1e-6, clamp_eta: bool = False,
                    eta_min: float = 0.05, eta_max: float = 40.0, sanitize: bool = False,
                    return_xq: bool = False, stream=None):
    import torch

    M, K = x.shape
    N = packed.shape[0]
    flags = ((GAMMA_PER_ROW if per_row else 0) | (FLAG_RMSNORM if rmsnorm else 0) |
             (FLAG_FWHT if fwht else 0) | (FLAG_ETA_CLAMP if clamp_eta else 0) |
             (FLAG_SANITIZE_NONFINITE if sanitize else 0))
    y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    ws = torch.empty((fused_workspace_bytes(M, K, flags),), dtype=torch.uint8, device=x.device)
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device) if return_xq else None
    sx = torch.empty((M,), dtype=torch.float32, device=x.device) if return_xq else None
    bitlinear_fused_(x, packed, gamma, flags, y, ws, rms_gain, rms_eps, eta_min, eta_max, xq, sx,
                     stream)
    return (y, xq, sx) if return_xq else y
