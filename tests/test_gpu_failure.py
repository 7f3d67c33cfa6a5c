"""Failure detection on the GPU without a fault: a kernel's bounded wait that
nothing completes gives up after its limit, records TQ_ERR_TIMEOUT in the
per-device status word and returns; the host reads the status (once: reading
clears it), and the context stays usable -- a normal call right after is
bit-exact against the oracle.  The wait is the library's own bounded wait
(spinning and suspending forms), run by the tq_selftest_wait_timeout kernel on
an mbarrier that is never arrived on."""
import time

import numpy as np
import pytest

import oracle
from ternary_bit_linear_b200 import synthetic as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TQ_ERR_TIMEOUT = 7


def normal_call_is_exact(tq):
    W = S.normal((96, 512), 0.02, 140, 1)
    X = S.decode_acts(4, 512, seed=141)
    packed, gamma = tq.quantize_ternary_pack(torch.from_numpy(W).cuda(), per_row=True)
    xq, sx, rs = tq.quantize_act_int8(torch.from_numpy(X).cuda())
    for M in (4,):
        y, acc = tq.ternary_gemm(xq, sx, rs, packed, gamma, per_row=True, with_acc=True)
        torch.cuda.synchronize()
        p_ref, g_ref = oracle.quantize_pack(W, per_row=True)
        xq_ref, _, _ = oracle.act_quant(X)
        assert np.array_equal(packed.cpu().numpy(), p_ref)
        assert np.array_equal(acc.cpu().numpy(), oracle.matmul_addsub(xq_ref, p_ref))
    return True


@pytest.mark.parametrize("sleeping", [False, True])
def test_bounded_wait_gives_up_and_reports(cuda_lib, sleeping):
    tq = cuda_lib
    assert tq.device_status() == 0  # clean start
    limit_ns = 2_000_000  # 2 ms
    t0 = time.perf_counter()
    tq.selftest_wait_timeout(limit_ns, sleeping)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert waited >= limit_ns * 1e-9 * 0.9, waited  # it really waited ...
    assert waited < 5.0                              # ... and then gave up
    assert tq.device_status() == TQ_ERR_TIMEOUT      # recorded once
    assert tq.device_status() == 0                   # reading cleared it
    assert normal_call_is_exact(tq)                  # the context is intact
    assert tq.device_status() == 0


def test_timeout_status_survives_later_work_until_read(cuda_lib):
    """The status word is sticky: work after the timed-out kernel does not
    clear it; only tq_get_device_status does."""
    tq = cuda_lib
    assert tq.device_status() == 0
    tq.selftest_wait_timeout(100_000)
    normal_call_is_exact(tq)
    assert tq.device_status() == TQ_ERR_TIMEOUT
    assert tq.device_status() == 0
