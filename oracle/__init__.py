"""CPU oracle for the ternary linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The CUDA
path (``ternary_bit_linear_b200``) never imports it and shares no code with it.

The arithmetic lives in ``tq_oracle.c`` (plain C, single-threaded, one
function per step of the pages' method, each citing the page and section it
follows).  This module compiles it with gcc on first use and wraps each
function for numpy arrays.  Function names follow the C file.

Parity pins for every function are in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq_oracle.c")
_LIB = os.path.join(_HERE, "libtq_oracle.so")

EPS = np.float32(1e-6)

_lib = None


def build(force: bool = False) -> str:
    """Compile tq_oracle.c into libtq_oracle.so beside it (gcc, IEEE fp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call([
            "gcc", "-O2", "-std=gnu99", "-fPIC", "-shared", "-ffp-contract=off",
            "-fno-fast-math", "-o", tmp, _SRC, "-lm",
        ])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        F = ctypes.c_float
        _lib.tqo_absmean_gamma.argtypes = [P, I64, F]
        _lib.tqo_absmean_gamma.restype = F
        _lib.tqo_sanitize_weights.argtypes = [P, I64, P]
        _lib.tqo_ternary_codes.argtypes = [P, I64, I64, P, I, P]
        _lib.tqo_pack.argtypes = [P, I64, I64, P]
        _lib.tqo_unpack.argtypes = [P, I64, I64, P]
        _lib.tqo_unpack.restype = I64
        _lib.tqo_quantize_pack.argtypes = [P, I64, I64, I, I, P, P]
        _lib.tqo_quantize_pack_format.argtypes = [P, I64, I64, I, I, I, P, P]
        _lib.tqo_quantize_pack_threshold.argtypes = [P, I64, I64, I, I, I, F, P, P]
        _lib.tqo_quantize_pack_abs_threshold.argtypes = [P, I64, I64, I, I, F, P, P]
        _lib.tqo_dequant_bias.argtypes = [P, P, I, P, P, I64, I64, P]
        _lib.tqo_int_epilogue.argtypes = [P, P, I, I64, I64, P]
        _lib.tqo_fwht_roundtrip.argtypes = [P, I64, I64, F, F, P, P]
        _lib.tqo_swiglu_act.argtypes = [P, P, I64, F, P]
        _lib.tqo_ternary_codes_threshold.argtypes = [P, I64, I64, P, I, F, P]
        _lib.tqo_pack_format.argtypes = [P, I64, I64, I, P]
        _lib.tqo_unpack_format.argtypes = [P, I64, I64, I, P]
        _lib.tqo_matmul_addsub_format.argtypes = [P, P, I64, I64, I64, I, P]
        _lib.tqo_act_quant.argtypes = [P, I64, I64, I, F, F, P, P, P]
        _lib.tqo_matmul_dense.argtypes = [P, P, I64, I64, I64, P]
        _lib.tqo_matmul_addsub.argtypes = [P, P, I64, I64, I64, P]
        _lib.tqo_dequant.argtypes = [P, P, I, P, I64, I64, P]
        _lib.tqo_sanitize_acts.argtypes = [P, I64, F, P]
        _lib.tqo_rmsnorm.argtypes = [P, P, I64, I64, F, P]
        _lib.tqo_fwht512.argtypes = [P, P, I64, I64, I]
        U64P = ctypes.POINTER(ctypes.c_uint64)
        _lib.tqo_backward_input.argtypes = [P, P, I, P, I, P, I, I64, I64, I64, P]
        _lib.tqo_ste_backward.argtypes = [P, P, P, I, F, I, I64, I64, P]
        _lib.tqo_xorshift64.argtypes = [U64P]
        _lib.tqo_xorshift64.restype = ctypes.c_uint64
        _lib.tqo_seed.argtypes = [U64P, ctypes.c_uint64]
        _lib.tqo_stochastic_flip.argtypes = [P, I, P, F, I64, I64, U64P]
        _lib.tqo_bitlinear.argtypes = [P, P, F, I, I, I, I, F, F, P, P, I, I64, I64, I64,
                                       P, P, P, P]
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# weights
# --------------------------------------------------------------------------

def absmean_gamma(w, eps=EPS) -> np.float32:
    """fp32 nearest to mean(|w|) (ties to even), then max(eps)."""
    w, pw = _c(w, np.float32)
    return np.float32(_load().tqo_absmean_gamma(pw, w.size, float(eps)))


def sanitize_weights(w):
    w, pw = _c(w, np.float32)
    out = np.empty_like(w)
    _load().tqo_sanitize_weights(pw, w.size, out.ctypes.data_as(ctypes.c_void_p))
    return out


def ternary_codes(w, gamma, per_row: bool):
    w, pw = _c(w, np.float32)
    N, K = w.shape
    g, pg = _c(np.atleast_1d(gamma), np.float32)
    q = np.empty((N, K), np.int8)
    _load().tqo_ternary_codes(pw, N, K, pg, int(per_row), q.ctypes.data_as(ctypes.c_void_p))
    return q


def pack(q):
    q, pq = _c(q, np.int8)
    N, K = q.shape
    assert K % 4 == 0
    out = np.empty((N, K // 4), np.uint8)
    _load().tqo_pack(pq, N, K, out.ctypes.data_as(ctypes.c_void_p))
    return out


def unpack(packed, K: int):
    """Returns (codes int8 [N,K], number of reserved 0b11 fields seen)."""
    packed, pp = _c(packed, np.uint8)
    N = packed.shape[0]
    assert packed.shape[1] * 4 == K
    q = np.empty((N, K), np.int8)
    n_res = _load().tqo_unpack(pp, N, K, q.ctypes.data_as(ctypes.c_void_p))
    return q, int(n_res)


def quantize_pack(w, per_row: bool, sanitize: bool = False, encoding: int = 0):
    """Returns (packed uint8 [N, K/4], gamma float32 [N] or [1]).  encoding:
    0 Foundry's layout, 1 Hetman-2b "Format 0", 2 Hetman-2b "Format 1"."""
    w, pw = _c(w, np.float32)
    N, K = w.shape
    packed = np.empty((N, K // 4), np.uint8)
    gamma = np.empty((N if per_row else 1,), np.float32)
    _load().tqo_quantize_pack_format(pw, N, K, int(per_row), int(sanitize), int(encoding),
                                     packed.ctypes.data_as(ctypes.c_void_p),
                                     gamma.ctypes.data_as(ctypes.c_void_p))
    return packed, gamma


def ternary_codes_threshold(w, gamma, per_row: bool, ratio: float):
    w, pw = _c(w, np.float32)
    N, K = w.shape
    g, pg = _c(np.atleast_1d(gamma), np.float32)
    q = np.empty((N, K), np.int8)
    _load().tqo_ternary_codes_threshold(pw, N, K, pg, int(per_row), float(ratio),
                                        q.ctypes.data_as(ctypes.c_void_p))
    return q


def quantize_pack_threshold(w, per_row: bool, ratio: float, sanitize: bool = False, encoding: int = 0):
    """Threshold rule (code = sign(w) where |w| > fp32(ratio * gamma)); returns
    (packed, gamma) like quantize_pack."""
    w, pw = _c(w, np.float32)
    N, K = w.shape
    packed = np.empty((N, K // 4), np.uint8)
    gamma = np.empty((N if per_row else 1,), np.float32)
    _load().tqo_quantize_pack_threshold(pw, N, K, int(per_row), int(sanitize), int(encoding), float(ratio),
                                        packed.ctypes.data_as(ctypes.c_void_p),
                                        gamma.ctypes.data_as(ctypes.c_void_p))
    return packed, gamma


def quantize_pack_abs_threshold(w, threshold: float, sanitize: bool = False, encoding: int = 0):
    """Foundry's manual threshold (fq_quantize_ternary_threshold): code =
    sign(w) where |w| > threshold, scale gamma[0] = threshold; returns
    (packed, gamma) like quantize_pack."""
    w, pw = _c(w, np.float32)
    N, K = w.shape
    packed = np.empty((N, K // 4), np.uint8)
    gamma = np.empty((1,), np.float32)
    _load().tqo_quantize_pack_abs_threshold(pw, N, K, int(sanitize), int(encoding), float(threshold),
                                            packed.ctypes.data_as(ctypes.c_void_p),
                                            gamma.ctypes.data_as(ctypes.c_void_p))
    return packed, gamma


def pack_format(q, encoding: int):
    q, pq = _c(q, np.int8)
    N, K = q.shape
    assert K % 4 == 0
    out = np.empty((N, K // 4), np.uint8)
    _load().tqo_pack_format(pq, N, K, int(encoding), out.ctypes.data_as(ctypes.c_void_p))
    return out


def unpack_format(packed, K: int, encoding: int):
    packed, pp = _c(packed, np.uint8)
    N = packed.shape[0]
    assert packed.shape[1] * 4 == K
    q = np.empty((N, K), np.int8)
    _load().tqo_unpack_format(pp, N, K, int(encoding), q.ctypes.data_as(ctypes.c_void_p))
    return q


# --------------------------------------------------------------------------
# activations, contraction, epilogue
# --------------------------------------------------------------------------

def act_quant(x, clamp_eta: bool = False, eta_min: float = 0.05, eta_max: float = 40.0):
    """Returns (x_q int8 [M,K], s_x float32 [M], rowsum int32 [M])."""
    x, px = _c(x, np.float32)
    M, K = x.shape
    xq = np.empty((M, K), np.int8)
    sx = np.empty((M,), np.float32)
    rs = np.empty((M,), np.int32)
    _load().tqo_act_quant(px, M, K, int(clamp_eta), float(eta_min), float(eta_max),
                          xq.ctypes.data_as(ctypes.c_void_p), sx.ctypes.data_as(ctypes.c_void_p),
                          rs.ctypes.data_as(ctypes.c_void_p))
    return xq, sx, rs


def matmul_dense(xq, q):
    xq, px = _c(xq, np.int8)
    q, pq = _c(q, np.int8)
    M, K = xq.shape
    N = q.shape[0]
    acc = np.empty((M, N), np.int32)
    _load().tqo_matmul_dense(px, pq, M, N, K, acc.ctypes.data_as(ctypes.c_void_p))
    return acc


def matmul_addsub(xq, packed):
    xq, px = _c(xq, np.int8)
    packed, pp = _c(packed, np.uint8)
    M, K = xq.shape
    N = packed.shape[0]
    assert packed.shape[1] * 4 == K
    acc = np.empty((M, N), np.int32)
    _load().tqo_matmul_addsub(px, pp, M, N, K, acc.ctypes.data_as(ctypes.c_void_p))
    return acc


def matmul_addsub_format(xq, packed, encoding: int):
    xq, px = _c(xq, np.int8)
    packed, pp = _c(packed, np.uint8)
    M, K = xq.shape
    N = packed.shape[0]
    assert packed.shape[1] * 4 == K
    acc = np.empty((M, N), np.int32)
    _load().tqo_matmul_addsub_format(px, pp, M, N, K, int(encoding), acc.ctypes.data_as(ctypes.c_void_p))
    return acc


def dequant(acc, gamma, s_x, per_row: bool):
    acc, pa = _c(acc, np.int32)
    M, N = acc.shape
    g, pg = _c(np.atleast_1d(gamma), np.float32)
    sx, ps = _c(s_x, np.float32)
    y = np.empty((M, N), np.float32)
    _load().tqo_dequant(pa, pg, int(per_row), ps, M, N, y.ctypes.data_as(ctypes.c_void_p))
    return y


def sanitize_acts(x, eta_max: float = 40.0):
    x, px = _c(x, np.float32)
    out = np.empty_like(x)
    _load().tqo_sanitize_acts(px, x.size, float(eta_max), out.ctypes.data_as(ctypes.c_void_p))
    return out


def rmsnorm(x, gain=None, eps: float = 1e-6):
    x, px = _c(x, np.float32)
    M, K = x.shape
    pg = None
    if gain is not None:
        gain, pg = _c(gain, np.float32)
    out = np.empty_like(x)
    _load().tqo_rmsnorm(px, pg, M, K, float(eps), out.ctypes.data_as(ctypes.c_void_p))
    return out


def fwht512(x, normalize: bool = True):
    x, px = _c(x, np.float32)
    rows, K = x.shape
    assert K % 512 == 0
    y = np.empty_like(x)
    _load().tqo_fwht512(px, y.ctypes.data_as(ctypes.c_void_p), rows, K, int(normalize))
    return y


def dequant_bias(acc, gamma, s_x, per_row: bool, bias=None):
    acc, pa = _c(acc, np.int32)
    M, N = acc.shape
    g, pg = _c(np.atleast_1d(gamma), np.float32)
    sx, ps = _c(s_x, np.float32)
    pb = None
    if bias is not None:
        bias, pb = _c(bias, np.float32)
    y = np.empty((M, N), np.float32)
    _load().tqo_dequant_bias(pa, pg, int(per_row), ps, pb, M, N, y.ctypes.data_as(ctypes.c_void_p))
    return y


def int_epilogue(acc, bias=None, out_shift: int = 0):
    acc, pa = _c(acc, np.int32)
    M, N = acc.shape
    pb = None
    if bias is not None:
        bias, pb = _c(bias, np.int32)
    out = np.empty((M, N), np.int32)
    _load().tqo_int_epilogue(pa, pb, int(out_shift), M, N, out.ctypes.data_as(ctypes.c_void_p))
    return out


def fwht_roundtrip(x, eta_min: float = 0.05, eta_max: float = 40.0):
    """Returns (y float32 [rows, K], eta float32 [rows])."""
    x, px = _c(x, np.float32)
    rows, K = x.shape
    assert K % 512 == 0
    y = np.empty_like(x)
    eta = np.empty((rows,), np.float32)
    _load().tqo_fwht_roundtrip(px, rows, K, float(eta_min), float(eta_max), y.ctypes.data_as(ctypes.c_void_p),
                               eta.ctypes.data_as(ctypes.c_void_p))
    return y, eta


def bitlinear(x, packed, gamma, per_row: bool, rms_gain=None, rms_eps: float = 1e-6,
              use_rmsnorm: bool = True, use_fwht: bool = True, sanitize: bool = False,
              clamp_eta: bool = False, eta_min: float = 0.05, eta_max: float = 40.0):
    """Whole layer on pre-packed weights.  Returns (y, x_q, s_x, acc)."""
    x, px = _c(x, np.float32)
    M, K = x.shape
    packed, pp = _c(packed, np.uint8)
    N = packed.shape[0]
    g, pg = _c(np.atleast_1d(gamma), np.float32)
    pr = None
    if rms_gain is not None:
        rms_gain, pr = _c(rms_gain, np.float32)
    y = np.empty((M, N), np.float32)
    xq = np.empty((M, K), np.int8)
    sx = np.empty((M,), np.float32)
    acc = np.empty((M, N), np.int32)
    _load().tqo_bitlinear(px, pr, float(rms_eps), int(use_rmsnorm), int(use_fwht),
                          int(sanitize), int(clamp_eta), float(eta_min), float(eta_max),
                          pp, pg, int(per_row), M, N, K,
                          y.ctypes.data_as(ctypes.c_void_p), xq.ctypes.data_as(ctypes.c_void_p),
                          sx.ctypes.data_as(ctypes.c_void_p), acc.ctypes.data_as(ctypes.c_void_p))
    return y, xq, sx, acc


def swiglu_act(gate, up, clamp_val: float = 10.0):
    gate, pg = _c(gate, np.float32)
    up, pu = _c(up, np.float32)
    assert gate.shape == up.shape
    out = np.empty_like(gate)
    _load().tqo_swiglu_act(pg, pu, gate.size, float(clamp_val), out.ctypes.data_as(ctypes.c_void_p))
    return out


def swiglu_mlp(x, gate, up, down, per_row: bool, clamp_val: float = 10.0, use_rmsnorm: bool = True,
               use_fwht: bool = True):
    """Hetman-2b section 6 SwiGLUClamped.forward with three BitLinear layers
    (each: bitlinear above) on pre-packed (packed, gamma) pairs.  Returns
    (y, activated-and-clamped, x_q of the down projection)."""
    kw = dict(use_rmsnorm=use_rmsnorm, use_fwht=use_fwht)
    yg = bitlinear(x, gate[0], gate[1], per_row, **kw)[0]
    yu = bitlinear(x, up[0], up[1], per_row, **kw)[0]
    act = swiglu_act(yg, yu, clamp_val)
    y, xq, _, _ = bitlinear(act, down[0], down[1], per_row, **kw)
    return y, act, xq, yg, yu


# ---------------------------------------------------------------------------
# Training: gradient through the layer, STE, stochastic flip (tq_oracle.c)
# ---------------------------------------------------------------------------
def backward_input(dY, packed, gamma, per_row: bool, K: int, row_scale=None, dX_in=None, encoding: int = 0):
    """dX [M, K] float32 = (dX_in or 0) + row_scale[m] * sum_n fp32(dY[m, n] * gamma_n) * q[n, k]
    (Foundry fq_matmul_ternary_backward_input)."""
    dY, pd = _c(dY, np.float32)
    M, N = dY.shape
    packed, pp = _c(packed, np.uint8)
    assert packed.shape == (N, K // 4)
    g, pg = _c(np.atleast_1d(gamma), np.float32)
    pr = None
    if row_scale is not None:
        row_scale, pr = _c(row_scale, np.float32)
    dX = np.zeros((M, K), np.float32) if dX_in is None else np.array(dX_in, dtype=np.float32, order="C", copy=True)
    _load().tqo_backward_input(pd, pp, int(encoding), pg, int(per_row), pr, int(dX_in is not None), M, N, K,
                               dX.ctypes.data_as(ctypes.c_void_p))
    return dX


def ste_backward(grad, w, gamma, per_row: bool, tau: float = 1.0, sanitize: bool = False):
    """Hetman-2b AbsmeanWeightQuantizer.backward: (grad / gamma) * (1 or 0.1)."""
    grad, pgr = _c(grad, np.float32)
    w, pw = _c(w, np.float32)
    N, K = w.shape
    assert grad.shape == w.shape
    g, pg = _c(np.atleast_1d(gamma), np.float32)
    out = np.empty_like(w)
    _load().tqo_ste_backward(pgr, pw, pg, int(per_row), float(tau), int(sanitize), N, K,
                             out.ctypes.data_as(ctypes.c_void_p))
    return out


def seed(value: int) -> int:
    st = ctypes.c_uint64(0)
    _load().tqo_seed(ctypes.byref(st), ctypes.c_uint64(value))
    return st.value


def xorshift64(state: int, count: int = 1):
    """Returns (list of `count` outputs, state after them)."""
    st = ctypes.c_uint64(state)
    out = [_load().tqo_xorshift64(ctypes.byref(st)) for _ in range(count)]
    return out, st.value


def stochastic_flip(packed, grad, temperature: float, state: int, encoding: int = 0):
    """Foundry fq_ternary_stochastic_flip on a copy of `packed`.  Returns
    (new packed, state after the N*K draws)."""
    grad, pgr = _c(grad, np.float32)
    N, K = grad.shape
    out = np.array(packed, dtype=np.uint8, order="C", copy=True)
    assert out.shape == (N, K // 4)
    st = ctypes.c_uint64(state)
    _load().tqo_stochastic_flip(out.ctypes.data_as(ctypes.c_void_p), int(encoding), pgr, float(temperature),
                                N, K, ctypes.byref(st))
    return out, st.value
