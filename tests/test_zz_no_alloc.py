"""tq_quantize_ternary_pack_noalloc: the packing entry point for callers that
cannot allocate device memory -- a runtime whose allocator has reserved all of
HBM up front, a host that only receives device pointers from someone else, or
a path where a cudaMalloc (and the device synchronisation it may bring) is not
allowed.  It must give the same packed bytes and gamma as
tq_quantize_ternary_pack, which takes its scratch from the caller, and as the
CPU oracle; and since every call shares one fixed scratch array inside the
library, calls made one after another must each be right.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process.  Its
argument checks (the size limit among them) are CPU tests in test_abi_cpu.py.
"""
import ctypes

import numpy as np
import pytest

import oracle
from ternary_bit_linear_b200 import synthetic as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

LIMIT = 2048 * 65536  # per-tensor weights the fixed scratch array covers


def noalloc_pack(tq, w, flags):
    N, K = w.shape
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=w.device)
    gamma = torch.empty((N if flags & tq.GAMMA_PER_ROW else 1,), dtype=torch.float32,
                        device=w.device)
    rc = tq.load().tq_quantize_ternary_pack_noalloc(
        ctypes.c_void_p(w.data_ptr()), N, K, flags, ctypes.c_void_p(packed.data_ptr()),
        ctypes.c_void_p(gamma.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, packed, gamma


def workspace_pack(tq, w, flags):
    N, K = w.shape
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=w.device)
    gamma = torch.empty((N if flags & tq.GAMMA_PER_ROW else 1,), dtype=torch.float32, device=w.device)
    ws = torch.empty((max(tq.pack_workspace_bytes(N, K, flags), 16),), dtype=torch.uint8, device=w.device)
    tq.quantize_ternary_pack_(w, flags, packed, gamma, ws)
    return packed, gamma


def cases():
    tie = np.ones((1024, 4096), np.float32)
    tie[512, 7] = 1.25  # per-tensor mean 1 + 2^-24: an exact fp32 tie (exact path)
    bad = S.normal((40, 1024), 0.02, 0, 63)
    bad[0, 0], bad[3, 9], bad[7, 100], bad[39, 1023] = np.nan, np.inf, -np.inf, np.nan
    return [("normal", S.normal((2048, 4096), 0.02, 0, 61), 0),     # many partial sums
            ("ragged", S.laplace((129, 4160), 0.05, 0, 62), 0),     # few partial sums, ragged
            ("tie", tie, 0),
            ("nonfinite", bad, 1),                                   # TQ_FLAG_SANITIZE_NONFINITE
            ("format0", S.normal((96, 2048), 0.02, 0, 64), 1 << 7),  # Hetman-2b layouts
            ("format1", S.normal((96, 2048), 0.02, 0, 65), 2 << 7)]


@pytest.mark.parametrize("per_row", [False, True])
def test_noalloc_matches_workspace_version_and_oracle(cuda_lib, per_row):
    tq = cuda_lib
    for name, W, extra in cases():  # calls in a row share the library's scratch
        flags = (tq.GAMMA_PER_ROW if per_row else 0) | (tq.FLAG_SANITIZE_NONFINITE if extra & 1 else 0) \
            | (extra & tq.ENC_MASK)
        w = torch.from_numpy(W).cuda()
        rc, packed, gamma = noalloc_pack(tq, w, flags)
        assert rc == 0, tq.STATUS.get(rc, rc)
        ref_packed, ref_gamma = workspace_pack(tq, w, flags)
        torch.cuda.synchronize()
        assert torch.equal(gamma, ref_gamma), name
        assert torch.equal(packed, ref_packed), name
        p_o, g_o = oracle.quantize_pack(W, per_row=per_row, sanitize=bool(extra & 1), encoding=(extra >> 7) & 3)
        assert np.array_equal(gamma.cpu().numpy(), g_o), name
        assert np.array_equal(packed.cpu().numpy(), p_o), name
    assert tq.device_status() == 0


def test_noalloc_at_the_limit_twice(cuda_lib):
    """N * K exactly at the limit: every one of the 2048 slots holds a partial
    sum.  Two calls in a row (the second on other values) against the
    workspace version."""
    tq = cuda_lib
    N, K = LIMIT // 65536, 65536
    for seed in (66, 67):  # a 2048 x 4096 block repeated along K (generating 2^27 values is slow)
        w = torch.from_numpy(S.normal((N, 4096), 0.02, 0, seed)).cuda().repeat(1, K // 4096).contiguous()
        rc, packed, gamma = noalloc_pack(tq, w, 0)
        assert rc == 0, tq.STATUS.get(rc, rc)
        ref_packed, ref_gamma = workspace_pack(tq, w, 0)
        torch.cuda.synchronize()
        assert torch.equal(gamma, ref_gamma) and torch.equal(packed, ref_packed)
        del w, packed, ref_packed
    assert tq.device_status() == 0
