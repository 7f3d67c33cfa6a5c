"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Bars (from the method's contract):
  * packed bytes, gamma, int8 codes, s_x, rowsum, int32 accumulators and the
    FWHT output: bit-exact;
  * fp32 outputs y: max relative error 1e-5;
  * after the fused RMSNorm + FWHT prologue: int8 codes within 1 LSB on at most
    1e-4 of the elements (the RMSNorm sum of squares is reduced in a different
    order than the oracle's).
Oracle-side inputs (packed weights, x_q) are produced by the oracle and fed to
the GPU kernels that consume them; nothing produced by the GPU is fed to the
oracle.
"""
import functools
import math

import numpy as np
import pytest

import oracle
from ternary_bit_linear_b200 import synthetic as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

REL = 1e-5


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def assert_y_close(y, y_ref):
    y, y_ref = np.asarray(y, np.float64), np.asarray(y_ref, np.float64)
    zero = y_ref == 0
    assert np.all(y[zero] == 0), "y must be exactly 0 where acc == 0"
    rel = np.abs(y[~zero] - y_ref[~zero]) / np.abs(y_ref[~zero])
    assert rel.size == 0 or rel.max() <= REL, f"max rel err {rel.max():.3e}"


@functools.lru_cache(maxsize=None)
def cached(name, *args):
    return getattr(S, name)(*args)


# ---------------------------------------------------------------------------
# quantise + pack
# ---------------------------------------------------------------------------

PACK_SHAPES = [(1, 64), (3, 192), (17, 512), (129, 4160), (64, 8192), (5, 8256), (2, 65536)]


@pytest.mark.parametrize("N,K", PACK_SHAPES)
@pytest.mark.parametrize("per_row", [True, False])
def test_pack_matches_oracle(cuda_lib, N, K, per_row):
    W = S.normal((N, K), 0.02, 7, 100 + N)
    if N > 2:
        W[1] = S.laplace((K,), 0.05, 7, 200 + N)
        W[2] = 0.0  # all-zero row: gamma -> 1e-6, all codes 0
    packed, gamma = cuda_lib.quantize_ternary_pack(dev(W), per_row=per_row)
    p_ref, g_ref = oracle.quantize_pack(W, per_row=per_row)
    assert np.array_equal(host(gamma), g_ref)
    assert np.array_equal(host(packed), p_ref)


def test_pack_sanitize_nonfinite(cuda_lib):
    W = S.normal((8, 512), 0.02, 3, 31)
    W[0, 0], W[1, 7], W[2, 9], W[5, 511] = np.nan, np.inf, -np.inf, np.nan
    for per_row in (True, False):
        packed, gamma = cuda_lib.quantize_ternary_pack(dev(W), per_row=per_row, sanitize=True)
        p_ref, g_ref = oracle.quantize_pack(W, per_row=per_row, sanitize=True)
        assert np.array_equal(host(gamma), g_ref) and np.array_equal(host(packed), p_ref)


def test_pack_exact_ties():
    import ternary_bit_linear_b200 as tq

    u23 = np.float32(2.0 ** -23)
    rows = []
    base = np.tile(np.array([1.0, -1.0], np.float32), 30)
    # gamma = 1 exactly: ties at 0.5 and 1.5, then just above 0.5 (paired so the mean stays 1)
    rows.append(np.concatenate([[0.5, -0.5, 1.5, -1.5], base]))
    rows.append(np.concatenate([[0.5 + u23, -(0.5 + u23), 1.5 - u23, -(1.5 - u23)], base]))
    # gamma = 0.75 exactly: tie at 0.375, just above at 0.375 + 2^-23
    base75 = np.tile(np.array([0.75, -0.75], np.float32), 30)
    rows.append(np.concatenate([[0.375, -0.375, 1.125, -1.125], base75]))
    rows.append(np.concatenate([[0.375 + u23, -(0.375 + u23), 1.125 - u23, -(1.125 - u23)], base75]))
    W = np.array(rows, np.float32)
    packed, gamma = tq.quantize_ternary_pack(dev(W), per_row=True)
    p_ref, g_ref = oracle.quantize_pack(W, per_row=True)
    assert g_ref.tolist() == [1.0, 1.0, 0.75, 0.75]
    q_ref, _ = oracle.unpack(p_ref, 64)
    assert q_ref[:, :4].tolist() == [[0, 0, 1, -1], [1, -1, 1, -1], [0, 0, 1, -1], [1, -1, 1, -1]]
    assert np.array_equal(host(gamma), g_ref) and np.array_equal(host(packed), p_ref)


@pytest.mark.parametrize("N,K", [(1, 64), (17, 512), (129, 4160), (64, 8192), (5, 8256), (2, 65536)])
@pytest.mark.parametrize("t", [0.05, 0.0, 0.02])
def test_pack_abs_threshold_matches_oracle(cuda_lib, N, K, t):
    """Foundry's manual threshold: bytes and the stored scale bit-exact, in both
    pack kernels (K <= 8192 team kernel, larger K the row kernel)."""
    tq = cuda_lib
    W = S.laplace((N, K), 0.03, 8, 300 + N)
    if N > 2:  # weights exactly at +-t and one float beyond
        W[1, :4] = [t, -t, np.nextafter(np.float32(t), np.float32(1)), -np.nextafter(np.float32(t), np.float32(1))]
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    gamma = torch.empty((1,), dtype=torch.float32, device="cuda")
    tq.quantize_ternary_pack_abs_threshold_(dev(W), 0, t, packed, gamma)
    p_ref, g_ref = oracle.quantize_pack_abs_threshold(W, t)
    assert np.array_equal(host(gamma), g_ref)
    assert np.array_equal(host(packed), p_ref)


@pytest.mark.parametrize("enc", [1, 2])
def test_pack_abs_threshold_layouts_and_sanitize(cuda_lib, enc):
    tq = cuda_lib
    W = S.normal((40, 1024), 0.02, 9, 41)
    W[0, 0], W[3, 5], W[7, 9] = np.nan, np.inf, -np.inf
    packed = torch.empty((40, 256), dtype=torch.uint8, device="cuda")
    gamma = torch.empty((1,), dtype=torch.float32, device="cuda")
    tq.quantize_ternary_pack_abs_threshold_(dev(W), tq.FLAG_SANITIZE_NONFINITE | (enc << 7), 0.01, packed, gamma)
    p_ref, g_ref = oracle.quantize_pack_abs_threshold(W, 0.01, sanitize=True, encoding=enc)
    assert np.array_equal(host(gamma), g_ref) and np.array_equal(host(packed), p_ref)
    assert tq.device_status() == 0


def test_pack_dense_threshold_sweep(cuda_lib):
    # Row r: one probe value w_r followed by 63 entries of +-1.  Its gamma is
    # (|w_r| + 63) / 64, and w_r / gamma crosses 0.5 at w_r = 63/127.  4096
    # consecutive fp32 probes around that point (and their negatives) exercise
    # the exact rounding boundary of the code decision.
    centre = np.float32(63.0 / 127.0)
    bits = centre.view(np.int32) + np.arange(-2048, 2048, dtype=np.int32)
    probes = bits.view(np.float32)
    probes = np.concatenate([probes, -probes])
    filler = np.tile(np.array([1.0, -1.0], np.float32), 32)[:63]
    W = np.concatenate([probes[:, None], np.tile(filler, (probes.size, 1))], axis=1).astype(np.float32)
    packed, gamma = cuda_lib.quantize_ternary_pack(dev(W), per_row=True)
    p_ref, g_ref = oracle.quantize_pack(W, per_row=True)
    q_ref, _ = oracle.unpack(p_ref, 64)
    assert 0 < (q_ref[:, 0] != 0).sum() < probes.size  # the sweep straddles the boundary
    assert np.array_equal(host(gamma), g_ref) and np.array_equal(host(packed), p_ref)


@pytest.mark.parametrize("which", ["decode", "prefill", "fused", "sweep"])
def test_pack_full_size(cuda_lib, which):
    if which == "decode":
        W, per_row = cached("decode_weights", 4096, 4096), True
    elif which == "prefill":
        W, per_row = cached("prefill", 2048, 11008, 4096)[0], False
    elif which == "fused":
        W, per_row = cached("fused", 512, 5632, 2048)[0], False
    else:
        W, per_row = cached("sweep_weights", 8192, 8192), True
    packed, gamma = cuda_lib.quantize_ternary_pack(dev(W), per_row=per_row)
    p_ref, g_ref = oracle.quantize_pack(W, per_row=per_row)
    assert np.array_equal(host(gamma), g_ref)
    assert np.array_equal(host(packed), p_ref)


# ---------------------------------------------------------------------------
# activation quantisation and FWHT
# ---------------------------------------------------------------------------

ACT_SHAPES = [(1, 64), (3, 192), (4, 512), (8, 4096), (17, 4160), (2, 8192), (5, 8256), (3, 65536),
              # many tokens: the persistent ring kernel (rows streamed through shared memory)
              (300, 64), (401, 1088), (297, 4160), (600, 8192), (1000, 2048)]


@pytest.mark.parametrize("M,K", ACT_SHAPES)
@pytest.mark.parametrize("clamp", [False, True])
def test_act_quant_matches_oracle(cuda_lib, M, K, clamp):
    X = S.decode_acts(M, K, seed=11)
    if M > 2:
        X[1] = 0.0  # zero token
        X[2] *= np.float32(1e-4)  # tiny token (eta clamp lower bound when clamping)
    xq, sx, rs = cuda_lib.quantize_act_int8(dev(X), clamp_eta=clamp)
    xq_ref, sx_ref, rs_ref = oracle.act_quant(X, clamp_eta=clamp)
    assert np.array_equal(host(xq), xq_ref)
    assert np.array_equal(host(sx), sx_ref)
    assert np.array_equal(host(rs), rs_ref)


def test_act_quant_golden_ties_and_sanitize(cuda_lib):
    x = np.zeros((2, 64), np.float32)
    x[0, :8] = [1.0, 0.5, -0.5, 0.25, 0.125, -1.0, 0.0, 0.75]
    x[1] = S.normal((64,), 1.0, 1, 5)
    x[1, 3], x[1, 9], x[1, 10] = np.nan, np.inf, -np.inf
    xq, sx, rs = cuda_lib.quantize_act_int8(dev(x), sanitize=True, eta_max=40.0)
    xs = oracle.sanitize_acts(x, 40.0)
    xq_ref, sx_ref, rs_ref = oracle.act_quant(xs)
    assert xq_ref[0, :8].tolist() == [127, 64, -64, 32, 16, -127, 0, 95]
    assert np.array_equal(host(xq), xq_ref) and np.array_equal(host(sx), sx_ref)
    assert np.array_equal(host(rs), rs_ref)


def test_act_quant_many_tokens_sanitize(cuda_lib):
    M, K = 700, 4096
    X = S.decode_acts(M, K, seed=12)
    X[5, 3], X[40, 9], X[41, 10], X[699, 4095] = np.nan, np.inf, -np.inf, np.nan
    X[6] = np.inf
    xq, sx, rs = cuda_lib.quantize_act_int8(dev(X), sanitize=True, eta_max=40.0)
    xq_ref, sx_ref, rs_ref = oracle.act_quant(oracle.sanitize_acts(X, 40.0))
    assert np.array_equal(host(xq), xq_ref) and np.array_equal(host(sx), sx_ref)
    assert np.array_equal(host(rs), rs_ref)


def test_act_quant_prefill_full_size(cuda_lib):
    X = cached("prefill", 2048, 11008, 4096)[1]
    xq, sx, rs = cuda_lib.quantize_act_int8(dev(X))
    xq_ref, sx_ref, rs_ref = oracle.act_quant(X)
    assert np.array_equal(host(xq), xq_ref) and np.array_equal(host(sx), sx_ref)
    assert np.array_equal(host(rs), rs_ref)


@pytest.mark.parametrize("rows,K", [(1, 512), (8, 1536), (33, 2048), (4, 8192), (3, 65536)])
@pytest.mark.parametrize("normalize", [True, False])
def test_fwht_bit_exact(cuda_lib, rows, K, normalize):
    X = S.student_t3((rows, K), 2, 40 + rows)
    y = cuda_lib.fwht512(dev(X), normalize=normalize)
    assert np.array_equal(host(y), oracle.fwht512(X, normalize=normalize))


def test_fwht_in_place_and_spike(cuda_lib):
    x = np.zeros((1, 512), np.float32)
    x[0, 256] = 100.0
    t = dev(x)
    cuda_lib.fwht512_(t, t, True)
    y = host(t)
    assert np.array_equal(y, oracle.fwht512(x))
    assert abs(np.abs(y).max() - 100.0 / math.sqrt(512.0)) < 1e-4


# ---------------------------------------------------------------------------
# contraction (GEMV for M <= 16, tcgen05 GEMM above)
# ---------------------------------------------------------------------------

def run_gemm(tq, W, X, per_row):
    p_ref, g_ref = oracle.quantize_pack(W, per_row=per_row)
    xq_ref, sx_ref, rs_ref = oracle.act_quant(X)
    y, acc = tq.ternary_gemm(dev(xq_ref), dev(sx_ref), dev(rs_ref), dev(p_ref), dev(g_ref),
                             per_row=per_row, with_acc=True)
    return host(y), host(acc), (p_ref, g_ref, xq_ref, sx_ref)


GEMM_CASES = [
    # GEMV (M <= 16)
    (1, 1, 64), (1, 17, 192), (2, 128, 512), (3, 129, 1088), (5, 200, 4096), (8, 384, 4160),
    (9, 64, 8192), (15, 33, 2048), (16, 256, 4096), (16, 31, 8192), (1, 4096, 4096),
    # tcgen05 GEMM
    (17, 128, 512), (33, 130, 640), (64, 256, 1024), (65, 129, 4096), (100, 17, 192),
    (128, 384, 2048), (129, 128, 64), (255, 200, 1088), (256, 256, 4096), (300, 384, 1536),
    (513, 257, 512), (12, 128, 8256), (1000, 1, 128),
]


@pytest.mark.parametrize("M,N,K", GEMM_CASES)
@pytest.mark.parametrize("per_row", [True, False])
def test_gemm_matches_oracle(cuda_lib, M, N, K, per_row):
    W = S.normal((N, K), 0.02, 5, 1000 + N)
    X = S.decode_acts(M, K, seed=6)
    y, acc, (p_ref, g_ref, xq_ref, sx_ref) = run_gemm(cuda_lib, W, X, per_row)
    acc_ref = oracle.matmul_addsub(xq_ref, p_ref)
    assert np.array_equal(acc, acc_ref)
    assert_y_close(y, oracle.dequant(acc_ref, g_ref, sx_ref, per_row))


# Independent calls (TQ_FLAG_INPUTS_READY, M <= 8, K <= 4096) take the narrow
# streaming GEMV: runs of strips per CTA, one group of warps per strip, two
# strips in flight per group.  Shapes: one 64-byte step, a ragged last step,
# ragged last strips, runs shorter than the groups, and long runs (N = 16400:
# 33 strips per CTA, a ragged tail run).
STREAM_CASES = [(1, 1, 64), (3, 17, 1088), (8, 1000, 4096), (1, 4096, 4096), (5, 16400, 2048),
                (8, 64, 256), (2, 16384, 4096)]


@pytest.mark.parametrize("M,N,K", STREAM_CASES)
@pytest.mark.parametrize("per_row", [True, False])
def test_gemv_stream_matches_oracle(cuda_lib, M, N, K, per_row):
    tq = cuda_lib
    W = S.normal((N, K), 0.02, 7, 2000 + N)
    X = S.decode_acts(M, K, seed=8)
    p_ref, g_ref = oracle.quantize_pack(W, per_row=per_row)
    xq_ref, sx_ref, rs_ref = oracle.act_quant(X)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    fl = (tq.GAMMA_PER_ROW if per_row else 0) | tq.FLAG_WEIGHTS_STATIC | tq.FLAG_INPUTS_READY
    ins = [dev(a) for a in (xq_ref, sx_ref, rs_ref, p_ref, g_ref)]  # alive until the sync below
    tq.ternary_gemm_(*ins, fl, y, acc)
    acc_ref = oracle.matmul_addsub(xq_ref, p_ref)
    assert np.array_equal(host(acc), acc_ref)
    assert_y_close(host(y), oracle.dequant(acc_ref, g_ref, sx_ref, per_row))
    assert tq.device_status() == 0


def test_gemm_extreme_codes(cuda_lib):
    # all +1 / all -1 / all 0 weight rows and +-127 activations: |acc| = 127*K
    K, N, M = 4096, 130, 40
    W = np.zeros((N, K), np.float32)
    W[0::3] = 1.0
    W[1::3] = -1.0
    X = np.where(S.normal((M, K), 1.0, 1, 9) > 0, 1.0, -1.0).astype(np.float32)
    X[0] = 1.0
    for m_sub in (M, 4):  # tcgen05 GEMM and GEMV
        y, acc, (p_ref, g_ref, xq_ref, sx_ref) = run_gemm(cuda_lib, W, X[:m_sub], True)
        acc_ref = oracle.matmul_addsub(xq_ref, p_ref)
        assert acc_ref[0, 0] == 127 * K
        assert np.array_equal(acc, acc_ref)
        assert_y_close(y, oracle.dequant(acc_ref, g_ref, sx_ref, True))


def sampled_gemm_check(tq, W, X, per_row, sample):
    p_ref, g_ref = oracle.quantize_pack(W, per_row=per_row)
    xq_ref, sx_ref, rs_ref = oracle.act_quant(X)
    y, acc = tq.ternary_gemm(dev(xq_ref), dev(sx_ref), dev(rs_ref), dev(p_ref), dev(g_ref),
                             per_row=per_row, with_acc=True)
    y, acc = host(y), host(acc)
    acc_ref = oracle.matmul_addsub(xq_ref[sample], p_ref)
    assert np.array_equal(acc[sample], acc_ref)
    assert_y_close(y[sample], oracle.dequant(acc_ref, g_ref, sx_ref[sample], per_row))
    # every row (sampled or not) obeys the rescale identity exactly in fp32 terms
    g = g_ref if per_row else np.full(W.shape[0], g_ref[0], np.float32)
    y_from_acc = acc.astype(np.float32) * (g[None, :] * sx_ref[:, None])
    assert np.array_equal(y, y_from_acc.astype(np.float32))


@pytest.mark.parametrize("M", [1, 8])
def test_decode_full_size(cuda_lib, M):
    W = cached("decode_weights", 4096, 4096)
    X = S.decode_acts(M, 4096, seed=0)
    sampled_gemm_check(cuda_lib, W, X, True, np.arange(M))


def test_prefill_full_size_sampled(cuda_lib):
    W, X = cached("prefill", 2048, 11008, 4096)
    sampled_gemm_check(cuda_lib, W, X, False, np.arange(0, 2048, 97))


@pytest.mark.parametrize("M", [1, 4, 16, 64, 512, 4096])
def test_sweep_full_size_sampled(cuda_lib, M):
    W = cached("sweep_weights", 8192, 8192)
    X = S.sweep_acts(M, 8192, seed=0)
    sample = np.arange(M) if M <= 16 else np.unique(np.r_[0, np.arange(3, M, max(1, M // 12)), M - 1])
    sampled_gemm_check(cuda_lib, W, X, True, sample)


# ---------------------------------------------------------------------------
# fused layer
# ---------------------------------------------------------------------------

def check_fused(tq, X, W, per_row, sample=None, **kw):
    p_ref, g_ref = oracle.quantize_pack(W, per_row=per_row)
    okw = dict(kw)
    for k in ("return_xq",):
        okw.pop(k, None)
    rmsnorm = okw.pop("rmsnorm", True)
    fwht = okw.pop("fwht", True)
    gain = okw.get("rms_gain")
    y, xq, sx = tq.bitlinear_fused(dev(X), dev(p_ref), dev(g_ref), per_row=per_row,
                                   rmsnorm=rmsnorm, fwht=fwht, return_xq=True,
                                   **{k: (dev(v) if k == "rms_gain" and v is not None else v)
                                      for k, v in okw.items()})
    y, xq, sx = host(y), host(xq), host(sx)
    rows = np.arange(X.shape[0]) if sample is None else sample
    y_ref, xq_ref, sx_ref, acc_ref = oracle.bitlinear(X[rows], p_ref, g_ref, per_row,
                                                      use_rmsnorm=rmsnorm, use_fwht=fwht, **okw)
    d = np.abs(xq[rows].astype(np.int32) - xq_ref.astype(np.int32))
    assert d.max() <= 1
    assert (d != 0).sum() <= 1e-4 * d.size
    rel_sx = np.abs(sx[rows] - sx_ref) / sx_ref
    assert rel_sx.max() <= REL
    flips = (d != 0).sum(axis=1)
    if flips.sum() == 0 and np.array_equal(sx[rows], sx_ref):
        assert_y_close(y[rows], y_ref)
    else:  # a flipped code moves acc by at most 1 per flip
        g = g_ref if per_row else np.full(W.shape[0], g_ref[0], np.float32)
        bound = flips[:, None] * g[None, :] * sx_ref[:, None] * (1 + 1e-5) + REL * np.abs(y_ref) \
            + np.abs(y_ref) * rel_sx[:, None]
        assert np.all(np.abs(y[rows] - y_ref) <= bound)


@pytest.mark.parametrize("M,N,K", [(1, 64, 512), (3, 300, 1536), (16, 128, 2048), (17, 200, 1024),
                                   (200, 130, 512), (40, 64, 8192)])
def test_fused_matches_oracle(cuda_lib, M, N, K):
    W = S.normal((N, K), 0.02, 9, N)
    X = S.student_t3((M, K), 9, 7)
    check_fused(cuda_lib, X, W, False)


@pytest.mark.parametrize("variant", ["no_rms", "no_fwht", "plain", "gain", "clamp", "sanitize",
                                     "per_row"])
def test_fused_variants(cuda_lib, variant):
    M, N, K = 20, 96, 1024
    W = S.normal((N, K), 0.02, 10, 1)
    X = S.student_t3((M, K), 10, 2)
    kw = {}
    per_row = False
    if variant == "no_rms":
        kw["rmsnorm"] = False
    elif variant == "no_fwht":
        kw["fwht"] = False
    elif variant == "plain":
        kw.update(rmsnorm=False, fwht=False)
        K2 = 640
        W, X = W[:, :K2].copy(), X[:, :K2].copy()
    elif variant == "gain":
        kw["rms_gain"] = S.normal((K,), 1.0, 10, 3)
    elif variant == "clamp":
        kw["clamp_eta"] = True
        X[3] *= np.float32(1e-3)
        X[4] *= np.float32(500.0)
    elif variant == "sanitize":
        kw["sanitize"] = True
        X[0, 1], X[2, 5], X[7, 1023] = np.nan, np.inf, -np.inf
    elif variant == "per_row":
        per_row = True
    check_fused(cuda_lib, X, W, per_row, **kw)


def test_fused_full_size(cuda_lib):
    W, X = cached("fused", 512, 5632, 2048)
    check_fused(cuda_lib, X, W, False, sample=np.arange(0, 512, 37))


def test_device_status_clean(cuda_lib):
    assert cuda_lib.device_status() == 0


# ---------------------------------------------------------------------------
# exact-midpoint gamma (the double-double fallback) and launch ordering
# ---------------------------------------------------------------------------

def midpoint_rows(K, seed):
    """Rows whose mean |w| is exactly an fp32 rounding midpoint (ties to even)."""
    one, u = np.float32(1.0), np.float32(2.0 ** -23)
    signs = np.where(S.normal((4, K), 1.0, seed, 77) > 0, 1.0, -1.0).astype(np.float32)
    rows = np.empty((4, K), np.float32)
    rows[0] = np.tile([one, one + u], K // 2)              # mean 1 + 2^-24  -> 1 (even)
    rows[1] = np.tile([one + u, one + 2 * u], K // 2)      # mean 1 + 1.5u   -> 1 + 2u (even)
    rows[2] = np.tile([np.float32(0.75), np.float32(0.75) + u / 2], K // 2)  # tie below 1
    rows[3] = np.tile([np.float32(3.0), np.float32(3.0) + 2 * u], K // 2)    # mean 3 + u -> 3 (even)
    return rows * signs


@pytest.mark.parametrize("K", [512, 4096, 8256])
def test_pack_midpoint_means_take_exact_path(cuda_lib, K):
    W = midpoint_rows(K, K)
    packed, gamma = cuda_lib.quantize_ternary_pack(dev(W), per_row=True)
    p_ref, g_ref = oracle.quantize_pack(W, per_row=True)
    assert g_ref.tolist() == [1.0, float(np.float32(1.0 + 2.0 ** -22)), 0.75, 3.0]
    assert np.array_equal(host(gamma), g_ref) and np.array_equal(host(packed), p_ref)
    # per tensor: the whole matrix's mean is a midpoint too when built from one row kind
    Wt = np.tile(W[1:2], (64, 1))
    packed, gamma = cuda_lib.quantize_ternary_pack(dev(Wt), per_row=False)
    p_ref, g_ref = oracle.quantize_pack(Wt, per_row=False)
    assert g_ref[0] == np.float32(1.0 + 2.0 ** -22)
    assert np.array_equal(host(gamma), g_ref) and np.array_equal(host(packed), p_ref)


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (8, 1000, 4096), (16, 257, 8192), (3, 33, 192)])
def test_gemv_static_weights_flag_same_result(cuda_lib, M, N, K):
    tq = cuda_lib
    W = S.normal((N, K), 0.02, 12, N)
    X = S.decode_acts(M, K, seed=13)
    p_ref, g_ref = oracle.quantize_pack(W, per_row=True)
    xq_ref, sx_ref, rs_ref = oracle.act_quant(X)
    args = [dev(a) for a in (xq_ref, sx_ref, rs_ref, p_ref, g_ref)]
    y0 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    y1 = torch.empty_like(y0)
    tq.ternary_gemm_(*args, tq.GAMMA_PER_ROW, y0)
    tq.ternary_gemm_(*args, tq.GAMMA_PER_ROW | tq.FLAG_WEIGHTS_STATIC, y1)
    assert torch.equal(y0, y1)
    acc_ref = oracle.matmul_addsub(xq_ref, p_ref)
    assert_y_close(host(y1), oracle.dequant(acc_ref, g_ref, sx_ref, True))


def test_dependent_calls_back_to_back(cuda_lib):
    """Re-pack into the same buffer and contract it five times without any host
    synchronisation: every kernel must see its predecessor's writes (and not
    overwrite what the predecessor is still reading)."""
    tq = cuda_lib
    N, K, M = 384, 2048, 8
    X = dev(S.decode_acts(M, K, seed=21))
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    gamma = torch.empty((1,), dtype=torch.float32, device="cuda")
    ws = torch.empty((tq.pack_workspace_bytes(N, K, 0),), dtype=torch.uint8, device="cuda")
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty((M,), dtype=torch.float32, device="cuda")
    rs = torch.empty((M,), dtype=torch.int32, device="cuda")
    ys = []
    Ws = [S.normal((N, K), 0.02, 30 + i, 1) for i in range(5)]
    for i, W in enumerate(Ws):
        tq.quantize_ternary_pack_(dev(W), 0, packed, gamma, ws)
        tq.quantize_act_int8_(X, 0, 0.05, 40.0, xq, sx, rs)
        for Mi in (M, 40):  # GEMV and tcgen05 GEMM consumers of the same buffers
            Xi = X if Mi == M else dev(S.decode_acts(Mi, K, seed=22))
            if Mi != M:
                xq2 = torch.empty((Mi, K), dtype=torch.int8, device="cuda")
                sx2 = torch.empty((Mi,), dtype=torch.float32, device="cuda")
                rs2 = torch.empty((Mi,), dtype=torch.int32, device="cuda")
                tq.quantize_act_int8_(Xi, 0, 0.05, 40.0, xq2, sx2, rs2)
                y = torch.empty((Mi, N), dtype=torch.float32, device="cuda")
                tq.ternary_gemm_(xq2, sx2, rs2, packed, gamma, 0, y)
            else:
                y = torch.empty((Mi, N), dtype=torch.float32, device="cuda")
                tq.ternary_gemm_(xq, sx, rs, packed, gamma, 0, y)
            ys.append((i, Mi, y))
    torch.cuda.synchronize()
    for i, Mi, y in ys:
        p_ref, g_ref = oracle.quantize_pack(Ws[i], per_row=False)
        Xn = S.decode_acts(M, K, seed=21) if Mi == M else S.decode_acts(Mi, K, seed=22)
        xq_ref, sx_ref, _ = oracle.act_quant(Xn)
        acc_ref = oracle.matmul_addsub(xq_ref, p_ref)
        assert_y_close(host(y), oracle.dequant(acc_ref, g_ref, sx_ref, False))
    assert tq.device_status() == 0


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (8, 1000, 4096), (16, 257, 8192), (300, 384, 1536)])
def test_inputs_ready_flag_same_result_and_order(cuda_lib, M, N, K):
    """Independent contractions that share one activation (q/k/v style), each
    with its own output, launched with TQ_FLAG_INPUTS_READY back to back; then
    a flag-less consumer re-packs into the first weight buffer.  Every result
    must equal the flag-less one, and the re-pack must not overtake them."""
    tq = cuda_lib
    X = S.decode_acts(M, K, seed=41)
    xq_ref, sx_ref, rs_ref = oracle.act_quant(X)
    xq, sx, rs = dev(xq_ref), dev(sx_ref), dev(rs_ref)
    Ws = [S.normal((N, K), 0.02, 42 + i, N) for i in range(4)]
    refs = [oracle.quantize_pack(W, per_row=True) for W in Ws]
    P = [(dev(p), dev(g)) for p, g in refs]
    fl = tq.GAMMA_PER_ROW | tq.FLAG_WEIGHTS_STATIC
    torch.cuda.synchronize()
    ys = [torch.empty((M, N), dtype=torch.float32, device="cuda") for _ in Ws]
    for (p, g), y in zip(P, ys):
        tq.ternary_gemm_(xq, sx, rs, p, g, fl | tq.FLAG_INPUTS_READY, y)
    # a flag-less call right behind them overwrites the first weights
    ws = torch.empty((max(16, tq.pack_workspace_bytes(N, K, tq.GAMMA_PER_ROW)),), dtype=torch.uint8,
                     device="cuda")
    tq.quantize_ternary_pack_(dev(Ws[1]), tq.GAMMA_PER_ROW, P[0][0], P[0][1], ws)
    y_after = torch.empty((M, N), dtype=torch.float32, device="cuda")
    tq.ternary_gemm_(xq, sx, rs, P[0][0], P[0][1], tq.GAMMA_PER_ROW, y_after)
    for (p_ref, g_ref), y in zip(refs, ys):
        acc_ref = oracle.matmul_addsub(xq_ref, p_ref)
        assert_y_close(host(y), oracle.dequant(acc_ref, g_ref, sx_ref, True))
    assert torch.equal(y_after, ys[1])
    assert tq.device_status() == 0


@pytest.mark.parametrize("M,K", [(4, 512), (512, 2048)])
def test_fused_inputs_ready_same_result_and_order(cuda_lib, M, K):
    """Independent fused layers (own x, y and workspace; N = K) launched with
    TQ_FLAG_INPUTS_READY back to back, then a flag-less fused call that takes
    the first layer's output as its input: every result equals the flag-less
    one, and the dependent call sees the finished output."""
    tq = cuda_lib
    N = K
    fl = tq.FLAG_FWHT | tq.FLAG_RMSNORM
    p_ref, g_ref = oracle.quantize_pack(S.normal((N, K), 0.02, 61, N), per_row=False)
    packed, gamma = dev(p_ref), dev(g_ref)
    xs = [dev(S.student_t3((M, K), 62 + i, 4 * M)) for i in range(3)]

    def new_ws():
        return torch.empty((tq.fused_workspace_bytes(M, K, fl),), dtype=torch.uint8, device="cuda")

    def new_y():
        return torch.empty((M, N), dtype=torch.float32, device="cuda")

    torch.cuda.synchronize()
    # every buffer of a flagged call stays allocated until the stream is
    # drained: the caching allocator would hand a freed block to the next
    # call on the same stream while the flagged call may still run
    ys = [new_y() for _ in xs]
    wss = [new_ws() for _ in xs]
    for x, y, ws in zip(xs, ys, wss):
        tq.bitlinear_fused_(x, packed, gamma, fl | tq.FLAG_INPUTS_READY, y, ws)
    y_dep = new_y()
    tq.bitlinear_fused_(ys[0], packed, gamma, fl, y_dep, new_ws())
    torch.cuda.synchronize()
    refs = [new_y() for _ in xs]
    for x, r in zip(xs, refs):
        tq.bitlinear_fused_(x, packed, gamma, fl, r, new_ws())
    r_dep = new_y()
    tq.bitlinear_fused_(refs[0], packed, gamma, fl, r_dep, new_ws())
    for i, (y, r) in enumerate(zip(ys + [y_dep], refs + [r_dep])):
        bad = (y != r).sum().item()
        assert bad == 0, "call %d: %d of %d outputs differ" % (i, bad, y.numel())
    assert tq.device_status() == 0


@pytest.mark.parametrize("per_row", [True, False])
def test_pack_inputs_ready_layers_then_dependent_reader(cuda_lib, per_row):
    """Pack several layers with TQ_FLAG_INPUTS_READY (each with its own buffers
    and workspace), then contract the last one right behind them without the
    flag: bytes and gamma must equal the oracle's, in order."""
    tq = cuda_lib
    N, K, L = 1000, 2048, 5
    Ws = [S.normal((N, K), 0.02, 60 + i, N) for i in range(L)]
    flags = (tq.GAMMA_PER_ROW if per_row else 0)
    nws = max(16, tq.pack_workspace_bytes(N, K, flags))
    bufs = [(torch.empty((N, K // 4), dtype=torch.uint8, device="cuda"),
             torch.empty((N if per_row else 1,), dtype=torch.float32, device="cuda"),
             torch.empty((nws,), dtype=torch.uint8, device="cuda")) for _ in range(L)]
    Wd = [dev(W) for W in Ws]
    torch.cuda.synchronize()
    for W, (p, g, ws) in zip(Wd, bufs):
        tq.quantize_ternary_pack_(W, flags | tq.FLAG_INPUTS_READY, p, g, ws)
    M = 8
    X = S.decode_acts(M, K, seed=61)
    xq_ref, sx_ref, rs_ref = oracle.act_quant(X)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    tq.ternary_gemm_(dev(xq_ref), dev(sx_ref), dev(rs_ref), bufs[-1][0], bufs[-1][1], flags, y)
    for W, (p, g, _) in zip(Ws, bufs):
        p_ref, g_ref = oracle.quantize_pack(W, per_row=per_row)
        assert np.array_equal(host(p), p_ref)
        assert np.array_equal(host(g), g_ref)
    p_ref, g_ref = oracle.quantize_pack(Ws[-1], per_row=per_row)
    acc_ref = oracle.matmul_addsub(xq_ref, p_ref)
    assert_y_close(host(y), oracle.dequant(acc_ref, g_ref, sx_ref, per_row))
    assert tq.device_status() == 0


# Shapes whose tile choice (tokens per tile, from the launcher's cost model on
# 148 SMs) is 128, 256, 256 and 256, all ragged in M, N and K; in the last one the
# last token tile holds 68 tokens and the last feature tile 92 features.
@pytest.mark.parametrize("M,N,K", [(383, 11000, 192), (500, 5600, 320), (1000, 4000, 192), (580, 4956, 192)])
def test_gemm_tile_sizes_sampled(cuda_lib, M, N, K):
    W = S.normal((N, K), 0.02, 70, N)
    X = S.decode_acts(M, K, seed=71)
    sample = np.unique(np.r_[0, 1, np.arange(5, M, max(1, M // 17)), M - 2, M - 1])
    sampled_gemm_check(cuda_lib, W, X, False, sample)


@pytest.mark.parametrize("M,K", [(8, 4096), (700, 4096)])
def test_act_inputs_ready_then_dependent_reader(cuda_lib, M, K):
    """Independent activation quantisations with TQ_FLAG_INPUTS_READY, then a
    flag-less contraction of the last batch right behind them."""
    tq = cuda_lib
    L = 5
    Xs = [S.decode_acts(M, K, seed=80 + i) for i in range(L)]
    outs = [(torch.empty((M, K), dtype=torch.int8, device="cuda"),
             torch.empty((M,), dtype=torch.float32, device="cuda"),
             torch.empty((M,), dtype=torch.int32, device="cuda")) for _ in range(L)]
    Xd = [dev(X) for X in Xs]
    N = 300
    W = S.normal((N, K), 0.02, 81, N)
    p_ref, g_ref = oracle.quantize_pack(W, per_row=True)
    packed, gamma = dev(p_ref), dev(g_ref)
    torch.cuda.synchronize()
    for x, (xq, sx, rs) in zip(Xd, outs):
        tq.quantize_act_int8_(x, tq.FLAG_INPUTS_READY, 0.05, 40.0, xq, sx, rs)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    tq.ternary_gemm_(outs[-1][0], outs[-1][1], outs[-1][2], packed, gamma, tq.GAMMA_PER_ROW, y)
    for X, (xq, sx, rs) in zip(Xs, outs):
        xq_ref, sx_ref, rs_ref = oracle.act_quant(X)
        assert np.array_equal(host(xq), xq_ref) and np.array_equal(host(sx), sx_ref)
        assert np.array_equal(host(rs), rs_ref)
    xq_ref, sx_ref, _ = oracle.act_quant(Xs[-1])
    assert_y_close(host(y), oracle.dequant(oracle.matmul_addsub(xq_ref, p_ref), g_ref, sx_ref, True))
    assert tq.device_status() == 0


@pytest.mark.parametrize("odd, expect", [(1.25, 1.0), (1.75, 1.0 + 2.0 ** -22)])
@pytest.mark.parametrize("sanitize", [False, True])
def test_pack_per_tensor_midpoint_many_ctas(cuda_lib, odd, expect, sanitize):
    """1024 x 4096 ones and one odd value: the mean is 1 + 2^-24 (ties to 1) or
    1 + 3 * 2^-24 (ties to 1 + 2^-22), so every pack CTA must take the exact
    path and all must agree with the oracle."""
    N, K = 1024, 4096
    W = np.ones((N, K), np.float32)
    W[N // 2, 7] = odd
    W[::3] *= -1.0
    if sanitize:
        W[5, 5], W[6, 6] = np.nan, np.nan  # quenched to 0: the mean drops by 2/(N K)
        W[7, 7] = 1.0
    packed, gamma = cuda_lib.quantize_ternary_pack(dev(W), per_row=False, sanitize=sanitize)
    p_ref, g_ref = oracle.quantize_pack(W, per_row=False, sanitize=sanitize)
    if not sanitize:
        assert g_ref[0] == np.float32(expect)
    assert np.array_equal(host(gamma), g_ref) and np.array_equal(host(packed), p_ref)


# ---------------------------------------------------------------------------
# Packed-code layouts: Hetman-2b section 3 "Format 0" / "Format 1" beside
# Foundry's (the default).  Bytes bit-exact against the oracle's packer;
# contractions (both GEMV shapes and the tcgen05 GEMM) bit-exact against the
# oracle's add/subtract walk in the same layout, with reserved fields mixed in
# (they read as 0).
# ---------------------------------------------------------------------------
LAYOUTS = [1, 2]  # oracle numbering; flag = layout << 7


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("N,K,per_row", [(33, 512, True), (129, 4160, False), (5, 8256, True), (64, 2048, False)])
def test_pack_layouts_match_oracle(cuda_lib, layout, N, K, per_row):
    tq = cuda_lib
    W = S.normal((N, K), 0.02, 90, N)
    p_ref, g_ref = oracle.quantize_pack(W, per_row=per_row, encoding=layout)
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    gamma = torch.empty((N if per_row else 1,), dtype=torch.float32, device="cuda")
    flags = (tq.GAMMA_PER_ROW if per_row else 0) | (layout << 7)
    ws = torch.empty((max(16, tq.pack_workspace_bytes(N, K, flags)),), dtype=torch.uint8, device="cuda")
    tq.quantize_ternary_pack_(dev(W), flags, packed, gamma, ws)
    assert np.array_equal(host(packed), p_ref)
    assert np.array_equal(host(gamma), g_ref)


def _with_reserved(packed, layout, seed):
    """Replace about 5 % of the fields with the layout's reserved code."""
    rng = np.random.default_rng(seed)
    res = 0b10 if layout == 1 else 0b11
    out = packed.copy()
    mask = rng.random(out.shape + (4,)) < 0.05
    for i in range(4):
        m = mask[..., i]
        out[m] = (out[m] & ~np.uint8(3 << (2 * i))) | np.uint8(res << (2 * i))
    return out


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("M,N,K,ready", [(1, 300, 4096, False), (5, 129, 1088, True), (8, 1000, 4096, True),
                                         (12, 64, 8192, False), (64, 256, 1024, False), (300, 384, 1536, False)])
def test_contraction_layouts_match_oracle(cuda_lib, layout, M, N, K, ready):
    tq = cuda_lib
    W = S.normal((N, K), 0.02, 91, N)
    X = S.decode_acts(M, K, seed=92)
    p_lay, g_ref = oracle.quantize_pack(W, per_row=True, encoding=layout)
    p_lay = _with_reserved(p_lay, layout, 93)
    xq_ref, sx_ref, rs_ref = oracle.act_quant(X)
    acc_ref = oracle.matmul_addsub_format(xq_ref, p_lay, layout)
    ins = [dev(a) for a in (xq_ref, sx_ref, rs_ref, p_lay, g_ref)]
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    fl = tq.GAMMA_PER_ROW | (layout << 7) | (tq.FLAG_WEIGHTS_STATIC | tq.FLAG_INPUTS_READY if ready else 0)
    tq.ternary_gemm_(*ins, fl, y, acc)
    assert np.array_equal(host(acc), acc_ref)
    assert_y_close(host(y), oracle.dequant(acc_ref, g_ref, sx_ref, True))
    assert tq.device_status() == 0


@pytest.mark.parametrize("layout", LAYOUTS)
def test_fused_layouts_equal_default_layout(cuda_lib, layout):
    tq = cuda_lib
    M, N, K = 512, 640, 2048
    W = S.normal((N, K), 0.02, 94, N)
    fl = tq.FLAG_FWHT | tq.FLAG_RMSNORM
    x = dev(S.student_t3((M, K), 95, M))
    outs = []
    for lay in (0, layout):
        p_ref, g_ref = oracle.quantize_pack(W, per_row=False, encoding=lay)
        packed, gamma = dev(p_ref), dev(g_ref)
        y = torch.empty((M, N), dtype=torch.float32, device="cuda")
        ws = torch.empty((tq.fused_workspace_bytes(M, K, fl),), dtype=torch.uint8, device="cuda")
        tq.bitlinear_fused_(x, packed, gamma, fl | (lay << 7), y, ws)
        outs.append(host(y))
    assert np.array_equal(outs[0], outs[1])
    assert tq.device_status() == 0


# ---------------------------------------------------------------------------
# Threshold ternarisation (Foundry "Absmean Thresholding": ratio 1; BitRASP
# ternarize_weight: ratio 0.55 per row), bytes and gamma bit-exact.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("ratio", [1.0, 0.55, 0.5, 2.0])
@pytest.mark.parametrize("N,K,per_row", [(17, 512, True), (129, 4160, False), (5, 8256, True), (40, 2048, True),
                                         (300, 1024, False)])
def test_pack_threshold_matches_oracle(cuda_lib, ratio, N, K, per_row):
    tq = cuda_lib
    W = S.normal((N, K), 0.02, 96, N)
    p_ref, g_ref = oracle.quantize_pack_threshold(W, per_row=per_row, ratio=ratio)
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    gamma = torch.empty((N if per_row else 1,), dtype=torch.float32, device="cuda")
    flags = tq.GAMMA_PER_ROW if per_row else 0
    ws = torch.empty((max(16, tq.pack_workspace_bytes(N, K, flags)),), dtype=torch.uint8, device="cuda")
    tq.quantize_ternary_pack_threshold_(dev(W), flags, ratio, packed, gamma, ws)
    assert np.array_equal(host(packed), p_ref)
    assert np.array_equal(host(gamma), g_ref)


def test_pack_threshold_boundaries_and_layout(cuda_lib):
    """Rows whose mean |w| is exactly 1 (so tau = ratio exactly for ratio 1 and
    0.5) holding weights at tau, just above and just below it, in both signs;
    packed in Hetman-2b's Format 1 as well."""
    tq = cuda_lib
    K = 512
    base = np.ones((8, K), np.float32)
    up, dn = np.nextafter(np.float32(1), np.float32(2)), np.nextafter(np.float32(1), np.float32(0))
    h_up, h_dn = np.nextafter(np.float32(0.5), np.float32(1)), np.nextafter(np.float32(0.5), np.float32(0))
    vals = np.array([1.0, -1.0, up, -up, dn, -dn, 0.5, -0.5, h_up, -h_up, h_dn, -h_dn], np.float32)
    base[:, :vals.size] = vals
    base[:, vals.size:2 * vals.size] = 2.0 - np.abs(vals)  # keeps the row's mean |w| at exactly 1
    W = base
    for ratio in (1.0, 0.5):
        for layout in (0, 2):
            p_ref, g_ref = oracle.quantize_pack_threshold(W, per_row=True, ratio=ratio, encoding=layout)
            assert np.all(g_ref == 1.0)
            packed = torch.empty((8, K // 4), dtype=torch.uint8, device="cuda")
            gamma = torch.empty((8,), dtype=torch.float32, device="cuda")
            tq.quantize_ternary_pack_threshold_(dev(W), tq.GAMMA_PER_ROW | (layout << 7), ratio, packed, gamma)
            assert np.array_equal(host(packed), p_ref), (ratio, layout)
            assert np.array_equal(host(gamma), g_ref)


# ---------------------------------------------------------------------------
# NEXT row N2: the FWHT module's quantisation round trip (Hetman-2b section 1,
# FastWalshHadamardTransform.forward) and the contraction's extra epilogues
# (BitLinear bias; BitRASP's integer bias + arithmetic shift).
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("rows,K", [(1, 512), (7, 1536), (300, 4096), (3, 16384)])
def test_fwht_roundtrip_bit_exact(cuda_lib, rows, K):
    tq = cuda_lib
    X = S.student_t3((rows, K), 97, rows)
    X[0, 5] = np.nan
    X[-1, 9] = np.inf
    X[-1, 11] = -np.inf
    y_ref, eta_ref = oracle.fwht_roundtrip(X, 0.05, 40.0)
    x = dev(X)
    y = torch.empty_like(x)
    eta = torch.empty((rows,), dtype=torch.float32, device="cuda")
    tq.fwht_roundtrip_(x, y, 0.05, 40.0, eta)
    assert np.array_equal(host(y), y_ref)
    assert np.array_equal(host(eta), eta_ref)
    tq.fwht_roundtrip_(x, x, 0.05, 40.0)  # in place
    assert np.array_equal(host(x), y_ref)


def test_fwht_roundtrip_gain_clamp_both_ends(cuda_lib):
    tq = cuda_lib
    X = np.zeros((3, 1024), np.float32)
    X[1, 0] = 1000.0  # rotates above eta_max
    X[2] = S.normal((1, 1024), 1e-4, 98, 1)[0]  # eta below eta_min
    for lo, hi in ((0.05, 40.0), (0.5, 2.0)):
        y_ref, eta_ref = oracle.fwht_roundtrip(X, lo, hi)
        x = dev(X)
        y = torch.empty_like(x)
        eta = torch.empty((3,), dtype=torch.float32, device="cuda")
        tq.fwht_roundtrip_(x, y, lo, hi, eta)
        assert np.array_equal(host(y), y_ref) and np.array_equal(host(eta), eta_ref)
        assert host(eta)[1] == np.float32(hi) and host(eta)[0] == np.float32(lo)


@pytest.mark.parametrize("M,N,K,layout", [(1, 300, 4096, 0), (8, 129, 1088, 1), (16, 64, 8192, 0),
                                          (64, 256, 1024, 2), (300, 384, 1536, 0)])
def test_gemm_ex_bias_and_integer_epilogue(cuda_lib, M, N, K, layout):
    tq = cuda_lib
    W = S.normal((N, K), 0.02, 99, N)
    X = S.decode_acts(M, K, seed=100)
    p_ref, g_ref = oracle.quantize_pack(W, per_row=True, encoding=layout)
    xq_ref, sx_ref, rs_ref = oracle.act_quant(X)
    acc_ref = oracle.matmul_addsub_format(xq_ref, p_ref, layout)
    rng = np.random.default_rng(101)
    bias = (rng.standard_normal(N) * 0.3).astype(np.float32)
    abias = rng.integers(-5000, 5000, N).astype(np.int32)
    for shift in (0, 3):
        ins = [dev(a) for a in (xq_ref, sx_ref, rs_ref, p_ref, g_ref)]
        bd, abd = dev(bias), dev(abias)
        y = torch.empty((M, N), dtype=torch.float32, device="cuda")
        acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
        tq.ternary_gemm_ex_(*ins, tq.GAMMA_PER_ROW | (layout << 7), y, acc, bd, abd, shift)
        assert np.array_equal(host(acc), oracle.int_epilogue(acc_ref, abias, shift))
        y_ref = oracle.dequant_bias(acc_ref, g_ref, sx_ref, True, bias)
        y0 = np.abs(oracle.dequant(acc_ref, g_ref, sx_ref, True).astype(np.float64))
        # two fp32 roundings (product, then the sum) against one: within 1e-5 of the
        # terms' magnitude, not of a possibly cancelled sum
        err = np.abs(host(y).astype(np.float64) - y_ref.astype(np.float64))
        assert np.all(err <= REL * (y0 + np.abs(bias)[None, :]) + 1e-30)
    assert tq.device_status() == 0


# ---------------------------------------------------------------------------
# NEXT row N3: Hetman-2b's clamped SwiGLU block of three BitLinear layers,
# every stage against the oracle's own chain (nothing the GPU produced is fed
# to the oracle):
#   * the gate/up projections' input codes and the projections themselves,
#     with the fused layer's rule (codes within 1 LSB on <= 1e-4 of the
#     elements; y within 1e-5, or bounded by the flipped codes);
#   * the clamped activation within the error its fp32 evaluation can carry:
#     SiLU(g) * u as g / (1 + expf(-g)) * u is within 4 ulp of the exact value
#     for the GPU's own g, u (expf <= 2 ulp, three IEEE operations), and the
#     differences of g and u from the oracle's propagate with the condition
#     numbers |1 + g (1 - sigmoid(g))| and 1 (the clamp is 1-Lipschitz);
#   * the down projection's input codes and the block output, again with the
#     fused layer's rule.
# ---------------------------------------------------------------------------
def check_codes_and_y(xq, sx, y, xq_ref, sx_ref, y_ref, gamma_n):
    """The fused layer's bar: codes within 1 LSB on <= 1e-4 of the elements,
    s_x within 1e-5; y within 1e-5 where no code of its token moved, else
    within the flips' bound (each flip moves acc by one)."""
    d = np.abs(xq.astype(np.int32) - xq_ref.astype(np.int32))
    assert d.max() <= 1
    assert (d != 0).sum() <= 1e-4 * d.size, f"{(d != 0).sum()} codes differ"
    rel_sx = np.abs(sx.astype(np.float64) - sx_ref) / sx_ref
    assert rel_sx.max() <= REL
    flips = (d != 0).sum(axis=1)
    if flips.sum() == 0 and np.array_equal(sx, sx_ref):
        assert_y_close(y, y_ref)
    else:
        bound = flips[:, None] * gamma_n[None, :].astype(np.float64) * sx_ref[:, None] * (1 + 1e-5) \
            + REL * np.abs(y_ref) + np.abs(y_ref) * rel_sx[:, None]
        assert np.all(np.abs(y.astype(np.float64) - y_ref) <= bound)
    return int(flips.sum())


@pytest.mark.parametrize("M,D,F,per_row", [(5, 512, 1024, False), (64, 1536, 6144, False), (33, 1024, 2048, True)])
def test_swiglu_mlp(cuda_lib, M, D, F, per_row):
    tq = cuda_lib
    X = S.student_t3((M, D), 110, M)
    Ws = [S.normal(shape, 0.02, 111 + i, shape[0]) for i, shape in enumerate([(F, D), (F, D), (D, F)])]
    packs = [oracle.quantize_pack(W, per_row=per_row) for W in Ws]
    y_ref, act_ref, xq2_ref, yg_ref, yu_ref = oracle.swiglu_mlp(X, packs[0], packs[1], packs[2], per_row)
    _, xq1_ref, sx1_ref, _ = oracle.bitlinear(X, packs[0][0], packs[0][1], per_row)
    sx2_ref = oracle.bitlinear(act_ref, packs[2][0], packs[2][1], per_row)[2]
    fl = tq.FLAG_FWHT | tq.FLAG_RMSNORM | (tq.GAMMA_PER_ROW if per_row else 0)
    dp = [(dev(p), dev(g)) for p, g in packs]
    y = torch.empty((M, D), dtype=torch.float32, device="cuda")
    act = torch.empty((M, F), dtype=torch.float32, device="cuda")
    ws = torch.zeros((tq.swiglu_workspace_bytes(M, D, F, fl),), dtype=torch.uint8, device="cuda")
    tq.swiglu_mlp_(dev(X), dp[0], dp[1], dp[2], fl, y, ws, 10.0, act)
    mid = {k: host(v) for k, v in tq.swiglu_intermediates(ws, M, D, F).items()}

    def gam(i, n):
        g = packs[i][1]
        return g if per_row else np.full(n, g[0], np.float32)

    # gate and up projections (one activation pass feeds both)
    for yk, yr, i in (("y_gate", yg_ref, 0), ("y_up", yu_ref, 1)):
        check_codes_and_y(mid["xq1"], mid["s_x1"], mid[yk], xq1_ref, sx1_ref, yr.astype(np.float64), gam(i, F))
    # the clamped activation, from the GPU's own projections and against the oracle's
    act_h = host(act).astype(np.float64)
    assert np.abs(act_h).max() <= 10.0
    g64, u64 = mid["y_gate"].astype(np.float64), mid["y_up"].astype(np.float64)
    gr, ur = yg_ref.astype(np.float64), yu_ref.astype(np.float64)
    sig = 1.0 / (1.0 + np.exp(-gr))
    unclamped = gr * sig * ur
    eps_g = np.abs(g64 - gr) / np.maximum(np.abs(gr), 1e-300)
    eps_u = np.abs(u64 - ur) / np.maximum(np.abs(ur), 1e-300)
    kappa = np.abs(1.0 + gr * (1.0 - sig))
    bound = 2.0 * np.abs(unclamped) * (kappa * eps_g + eps_u + 4 * 2.0 ** -24) + 1e-30
    assert np.all(np.abs(act_h - act_ref.astype(np.float64)) <= bound)
    # the down projection and the block output
    check_codes_and_y(mid["xq2"], mid["s_x2"], host(y), xq2_ref, sx2_ref, y_ref.astype(np.float64), gam(2, D))
    assert tq.device_status() == 0


# ---------------------------------------------------------------------------
# NEXT row N4: training.  STE and flip bit-exact; the input gradient within
# 1e-5 of sum_n |fp32(dY gamma) q| * |row_scale| (+ |dX_in|): each term keeps
# 22 significant bits on the GPU (per-token power-of-two scale, two fp16
# parts), the accumulation rounds in fp32, and a cancelled sum has no
# relative accuracy in any fp32 order.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N,K,per_row,san,tau", [(1, 64, False, False, 1.0), (37, 448, True, True, 1.0),
                                                  (300, 4096, False, True, 1.5), (1024, 2048, True, False, 0.5)])
def test_ste_backward_bit_exact(cuda_lib, N, K, per_row, san, tau):
    tq = cuda_lib
    W = S.normal((N, K), 0.02, 120, N)
    G = S.normal((N, K), 1.0, 121, N)
    if N > 2:
        W[1, :4] = [np.nan, np.inf, -np.inf, 0.0]
        G[2, :2] = [np.nan, np.inf]
    p, gam = oracle.quantize_pack(np.nan_to_num(W, nan=0.0, posinf=1.0, neginf=-1.0), per_row=per_row)
    fl = (tq.GAMMA_PER_ROW if per_row else 0) | (tq.FLAG_SANITIZE_NONFINITE if san else 0)
    want = oracle.ste_backward(G, W, gam, per_row, tau, san)
    out = torch.empty((N, K), dtype=torch.float32, device="cuda")
    gd, wd, gmd = dev(G), dev(W), dev(gam)
    tq.ste_backward_(gd, wd, gmd, fl, out, tau)
    got = host(out)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32)) or \
        np.array_equal(np.nan_to_num(got, nan=7.0), np.nan_to_num(want, nan=7.0))
    tq.ste_backward_(gd, wd, gmd, fl, gd, tau)  # in place on the gradient
    assert np.array_equal(np.nan_to_num(host(gd), nan=7.0), np.nan_to_num(want, nan=7.0))
    assert tq.device_status() == 0


@pytest.mark.parametrize("layout", [0, 1, 2])
@pytest.mark.parametrize("N,K,temp", [(1, 64, 0.5), (37, 448, 0.05), (300, 4096, 0.2), (2048, 4096, 0.05)])
def test_stochastic_flip_bit_exact(cuda_lib, layout, N, K, temp):
    tq = cuda_lib
    q = np.clip(np.rint(S.normal((N, K), 0.7, 130, N)), -1, 1).astype(np.int8)
    G = S.normal((N, K), 1.0, 131, N)
    if N > 3:
        G[3, :3] = [np.nan, np.inf, 0.0]
    packed = oracle.pack_format(q, layout)
    st0 = tq.seed(1000 + N)
    assert st0 == oracle.seed(1000 + N)
    want, st_want = oracle.stochastic_flip(packed, G, temp, st0, layout)
    pd, gd = dev(packed), dev(G)
    st = tq.ternary_stochastic_flip_(pd, gd, temp, st0, layout << 7)
    assert st == st_want
    got = host(pd)
    assert np.array_equal(got, want)
    # a second call continues the stream where the first one stopped
    want2, st_want2 = oracle.stochastic_flip(want, G, temp, st_want, layout)
    assert tq.ternary_stochastic_flip_(pd, gd, temp, st, layout << 7) == st_want2
    assert np.array_equal(host(pd), want2)
    assert tq.device_status() == 0


def _bwd_check(tq, M, N, K, per_row, use_rs, accumulate, layout, seed, rows=None):
    dY = S.normal((M, N), 1.0, seed, M)
    if M > 3:  # heavy-tailed and wide-range rows: the per-token scale must cope
        dY[1] = S.student_t3((N,), seed, 7)
        dY[2] *= np.float32(1e-30)
        dY[3, ::3] *= np.float32(1e6)
    W = S.normal((N, K), 0.02, seed + 1, N)
    packed, gam = oracle.quantize_pack(W, per_row=per_row, encoding=layout)
    rs = (S.uniform(seed + 2, 0, 0, M).astype(np.float32) * np.float32(0.02)).astype(np.float32) if use_rs else None
    dX0 = S.normal((M, K), 1.0, seed + 3, M) if accumulate else None
    fl = (tq.GAMMA_PER_ROW if per_row else 0) | (tq.FLAG_ACCUMULATE if accumulate else 0) | (layout << 7)
    dXd = dev(dX0) if accumulate else torch.empty((M, K), dtype=torch.float32, device="cuda")
    ws = torch.empty((tq.backward_input_workspace_bytes(M, N),), dtype=torch.uint8, device="cuda")
    tq.ternary_backward_input_(dev(dY), dev(packed), dev(gam), fl, dXd, ws, None if rs is None else dev(rs))
    got = host(dXd)
    sel = np.arange(M) if rows is None else np.asarray(rows)
    want = oracle.backward_input(dY[sel], packed, gam, per_row, K, None if rs is None else rs[sel],
                                 None if dX0 is None else dX0[sel], layout)
    # magnitude of the terms: |g| @ |q| (+ |dX_in|)
    q = np.abs(oracle.unpack_format(packed, K, layout).astype(np.float64))
    g = np.abs((dY[sel] * (gam[None, :] if per_row else gam[0])).astype(np.float32).astype(np.float64))
    mag = (g @ q) * (np.abs(rs[sel].astype(np.float64))[:, None] if use_rs else 1.0)
    if accumulate:
        mag = mag + np.abs(dX0[sel].astype(np.float64))
    err = np.abs(got[sel].astype(np.float64) - want.astype(np.float64))
    assert np.all(err <= REL * mag + 1e-30), f"max err/mag {np.max(err / (mag + 1e-30)):.3e}"
    return err, mag


@pytest.mark.parametrize("M,N,K,per_row,use_rs,acc,layout", [
    (1, 1, 64, False, False, False, 0),        # one token, one output feature
    (5, 17, 64, True, True, False, 0),         # ragged everything, N % 4 != 0
    (300, 99, 192, False, False, True, 1),     # two token tiles, ragged; accumulate
    (257, 1000, 384, True, True, False, 2),    # three feature tiles, ragged token tile
    (512, 2048, 1024, False, True, True, 0),   # 4 x 8 tiles over 148 SMs
    (64, 4096, 256, True, False, False, 0),    # one token tile, long contraction
])
def test_backward_input_matches_oracle(cuda_lib, M, N, K, per_row, use_rs, acc, layout):
    err, mag = _bwd_check(cuda_lib, M, N, K, per_row, use_rs, acc, layout, 140 + M)
    assert cuda_lib.device_status() == 0


def test_backward_input_full_size_sampled_rows(cuda_lib):
    # the training workload: gradient of the prefill layer (2048 tokens,
    # 11008 -> 4096), rows sampled across token tiles and the ragged corners
    rows = [0, 1, 255, 256, 1000, 1791, 2046, 2047]
    err, mag = _bwd_check(cuda_lib, 2048, 11008, 4096, False, False, False, 0, 150, rows)
    # typical error far below the bound: the accumulation is fp32 over 11008 terms
    assert np.median(err / (mag + 1e-30)) < 1e-6
    assert cuda_lib.device_status() == 0


# ---------------------------------------------------------------------------
# Repeated calls are bit-identical (every result is a fixed function of the
# inputs).  Full size, where a pipeline hazard shows up: the packed-weight
# slot of the unpackers was once released before every lane's read of it
# was complete, and a refill could overtake the read.
# ---------------------------------------------------------------------------
def test_gemms_repeat_bit_identical_full_size(cuda_lib):
    tq = cuda_lib
    M, N, K = 2048, 11008, 4096
    W, X = cached("prefill", M, N, K, 0)
    pk, gm = tq.quantize_ternary_pack(dev(W), per_row=False)
    xq, sx, rs = tq.quantize_act_int8(dev(X))
    accs = []
    for _ in range(4):
        _, acc = tq.ternary_gemm(xq, sx, rs, pk, gm, per_row=False, with_acc=True)
        accs.append(host(acc))
    assert all(np.array_equal(a, accs[0]) for a in accs[1:])
    dY = dev(S.normal((M, N), 1.0, 160, 0))
    ws = torch.empty((tq.backward_input_workspace_bytes(M, N),), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(6):
        dX = torch.full((M, K), float("nan"), dtype=torch.float32, device="cuda")
        tq.ternary_backward_input_(dY, pk, gm, 0, dX, ws)
        outs.append(host(dX))
    assert not np.isnan(outs[0]).any()
    assert all(np.array_equal(o, outs[0]) for o in outs[1:])
    assert tq.device_status() == 0
