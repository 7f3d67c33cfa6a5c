"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no arithmetic of the ternary method; it only draws numbers.
Every value is a pure function of (seed, stream, index), so any slice of any
tensor can be regenerated independently and the CPU oracle and the CUDA path
see identical inputs.

Generator (counter based, splitmix64 mixing):
    base      = mix64(seed * 0x9E3779B97F4A7C15 + stream * 0xC2B2AE3D27D4EB4F
                      + 0x632BE59BD9B4E019)
    bits(i)   = mix64(base + (i + 1) * 0x9E3779B97F4A7C15)
    mix64(z)  = splitmix64 finaliser: z ^= z>>30; z *= 0xBF58476D1CE4E5B9;
                z ^= z>>27; z *= 0x94D049BB133111EB; z ^= z>>31   (mod 2^64)
    uniform   = ((bits >> 11) + 0.5) * 2^-53            in (0, 1)
Distributions (computed in float64, rounded once to float32):
    normal(0, s)      Box-Muller on uniforms (2i, 2i+1): s*sqrt(-2 ln u1)*cos(2 pi u2)
    student_t(df=3)   z0 / sqrt((z1^2 + z2^2 + z3^2) / 3), z_j normals of sub-streams
    laplace(0, b)     u = uniform - 1/2;  -b * sign(u) * ln(1 - 2|u|)
    outliers          element scaled by `factor` where uniform(outlier stream) < p
"""
from __future__ import annotations

import numpy as np

_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_GOLD = np.uint64(0x9E3779B97F4A7C15)
_STREAM = np.uint64(0xC2B2AE3D27D4EB4F)
_OFF = np.uint64(0x632BE59BD9B4E019)
_CHUNK = 1 << 22

# stream ids used by the workloads below
STREAM_W = 1
STREAM_X = 2
STREAM_OUTLIER = 3
STREAM_GAIN = 4


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * _M1
    z = z ^ (z >> np.uint64(27))
    z = z * _M2
    return z ^ (z >> np.uint64(31))


def _base(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        b = np.array([seed], np.uint64) * _GOLD + np.array([stream], np.uint64) * _STREAM + _OFF
        return _mix64(b)[0]


def uniform(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """float64 uniforms in (0, 1) for counter indices start .. start+count-1."""
    base = _base(seed, stream)
    out = np.empty(count, np.float64)
    with np.errstate(over="ignore"):
        for c0 in range(0, count, _CHUNK):
            n = min(_CHUNK, count - c0)
            idx = np.arange(start + c0 + 1, start + c0 + 1 + n, dtype=np.uint64)
            bits = _mix64(base + idx * _GOLD)
            out[c0:c0 + n] = ((bits >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)
    return out


def _normal64(seed: int, stream: int, count: int) -> np.ndarray:
    out = np.empty(count, np.float64)
    for c0 in range(0, count, _CHUNK):
        n = min(_CHUNK, count - c0)
        u = uniform(seed, stream, 2 * c0, 2 * n)
        out[c0:c0 + n] = np.sqrt(-2.0 * np.log(u[0::2])) * np.cos(2.0 * np.pi * u[1::2])
    return out


def normal(shape, std: float, seed: int, stream: int) -> np.ndarray:
    n = int(np.prod(shape))
    return (_normal64(seed, stream, n) * std).astype(np.float32).reshape(shape)


def student_t3(shape, seed: int, stream: int) -> np.ndarray:
    n = int(np.prod(shape))
    z0 = _normal64(seed, stream * 16 + 0, n)
    s = np.zeros(n, np.float64)
    for j in (1, 2, 3):
        z = _normal64(seed, stream * 16 + j, n)
        s += z * z
    return (z0 / np.sqrt(s / 3.0)).astype(np.float32).reshape(shape)


def laplace(shape, b: float, seed: int, stream: int) -> np.ndarray:
    n = int(np.prod(shape))
    u = uniform(seed, stream, 0, n) - 0.5
    return (-b * np.sign(u) * np.log1p(-2.0 * np.abs(u))).astype(np.float32).reshape(shape)


def with_outliers(x: np.ndarray, p: float, factor: float, seed: int, stream: int) -> np.ndarray:
    u = uniform(seed, stream, 0, x.size).reshape(x.shape)
    y = x.copy()
    sel = u < p
    y[sel] = (x[sel].astype(np.float64) * factor).astype(np.float32)
    return y


# --------------------------------------------------------------------------
# The five workloads (weights W are [N, K] row-major, activations X [M, K])
# --------------------------------------------------------------------------

def single_layer(seed: int = 0):
    """256x512 weights ~N(0, 0.02), per-tensor gamma; 4x512 activations ~N(0, 1)."""
    W = normal((256, 512), 0.02, seed, STREAM_W)
    X = normal((4, 512), 1.0, seed, STREAM_X)
    return W, X


def decode_weights(N: int = 4096, K: int = 4096, seed: int = 0):
    """Decode GEMV weights ~N(0, 0.02), per-row gamma."""
    return normal((N, K), 0.02, seed, STREAM_W)


def decode_acts(M: int, K: int = 4096, seed: int = 0):
    """Decode activations ~N(0, 1) with 0.1 % of elements scaled by 20."""
    x = normal((M, K), 1.0, seed, STREAM_X)
    return with_outliers(x, 1e-3, 20.0, seed, STREAM_OUTLIER)


def prefill(M: int = 2048, N: int = 11008, K: int = 4096, seed: int = 0):
    """Prefill GEMM: X ~N(0, 1), W ~N(0, 0.02), per-tensor gamma."""
    return normal((N, K), 0.02, seed, STREAM_W), normal((M, K), 1.0, seed, STREAM_X)


def fused(M: int = 512, N: int = 5632, K: int = 2048, seed: int = 0):
    """Fused BitLinear: X ~Student-t(3), W ~N(0, 0.02), per-tensor gamma."""
    return normal((N, K), 0.02, seed, STREAM_W), student_t3((M, K), seed, STREAM_X)


def sweep_weights(N: int = 8192, K: int = 8192, seed: int = 0):
    """M sweep weights ~Laplace(0, 0.02), per-row gamma."""
    return laplace((N, K), 0.02, seed, STREAM_W)


def sweep_acts(M: int, K: int = 8192, seed: int = 0):
    return normal((M, K), 1.0, seed, STREAM_X)
