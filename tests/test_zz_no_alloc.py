"""tq_quantize_ternary_pack_noalloc: the packing entry point for callers that
cannot allocate device memory (their allocator owns all of HBM, they only
receive device pointers, or a cudaMalloc is not allowed on their path).  It
must give the same packed bytes and gamma as tq_quantize_ternary_pack, which
takes its scratch from the caller, and it shares one fixed scratch array
between calls -- so two calls in a row must each be right.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

from ternary_bit_linear_b200 import synthetic as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

MAX_ELEMS = 2048 * 65536  # per-tensor limit stated in include/tq.h


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


@pytest.mark.parametrize("per_row", [False, True])
def test_noalloc_matches_workspace_version_twice(cuda_lib, per_row):
    tq = cuda_lib
    flags = tq.GAMMA_PER_ROW if per_row else 0
    tie = np.ones((1024, 4096), np.float32)
    tie[512, 7] = 1.25  # per-tensor mean 1 + 2^-24: an exact fp32 tie (exact path)
    cases = [S.normal((2048, 4096), 0.02, 0, 61),        # many partial sums
             S.laplace((129, 4160), 0.05, 0, 62),        # ragged, few partial sums
             tie]
    for W in cases:  # two calls in a row share the library's scratch
        w = torch.from_numpy(W).cuda()
        rc, packed, gamma = noalloc_pack(tq, w, flags)
        assert rc == 0, tq.STATUS.get(rc, rc)
        ref_packed, ref_gamma = tq.quantize_ternary_pack(w, per_row=per_row)
        torch.cuda.synchronize()
        assert torch.equal(gamma, ref_gamma)
        assert torch.equal(packed, ref_packed)
    assert tq.device_status() == 0


def test_noalloc_rejects_oversized_per_tensor_call(cuda_lib):
    tq = cuda_lib
    N, K = MAX_ELEMS // 65536 + 1, 65536  # one row past the limit; never touched
    fake = ctypes.c_void_p(1 << 40)
    rc = tq.load().tq_quantize_ternary_pack_noalloc(fake, N, K, 0, fake, fake, None)
    assert rc == 2  # TQ_ERR_SHAPE, nothing launched
