"""Pins for the CPU oracle: each check ties the oracle to something other than
itself -- a value printed on the pages (tests/golden), a closed form, a
library routine the oracle does not call, exact rational arithmetic, or an
invariant of the mathematics.  Chosen so that a dropped term, a wrong sign,
index or rounding rule in any oracle function fails at least one of them.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg

import oracle
from ternary_bit_linear_b200 import synthetic as S
from tests.conftest import golden_lines

F32_ONE_OVER_SQRT512 = np.frombuffer(bytes.fromhex("f304353d"), np.float32)[0]  # 0x3D3504F3


def f32_round_rational(q: Fraction) -> np.float32:
    """Nearest float32 to a non-negative rational, ties to even.  Written
    independently of the oracle: bracket with float64, walk float32 neighbours,
    compare exactly with Fraction."""
    assert q >= 0
    c = np.float32(float(q))
    lo, hi = c, c
    while Fraction(float(lo)) > q:
        lo = np.nextafter(lo, np.float32(0))
    while Fraction(float(hi)) < q:
        hi = np.nextafter(hi, np.float32(np.inf))
    if lo == hi:
        return lo
    dlo, dhi = q - Fraction(float(lo)), Fraction(float(hi)) - q
    if dlo < dhi:
        return lo
    if dhi < dlo:
        return hi
    bits_lo = np.array([lo], np.float32).view(np.uint32)[0]
    return lo if bits_lo % 2 == 0 else hi


# --------------------------------------------------------------------------
# packing
# --------------------------------------------------------------------------

def test_pack_hand_worked_bytes():
    for ln in golden_lines("pack_bytes.txt"):
        *vals, byte = ln.split()
        q = np.array([[int(v) for v in vals]], np.int8)
        assert oracle.pack(q)[0, 0] == int(byte, 16), ln


def test_pack_all_81_tuples_round_trip_and_no_reserved_code():
    vals = np.array(np.meshgrid(*[[-1, 0, 1]] * 4, indexing="ij")).reshape(4, -1).T.astype(np.int8)
    packed = oracle.pack(vals.reshape(1, -1))  # 81 tuples in one row of 324 values
    assert packed.shape == (1, 81)
    assert len(set(packed[0].tolist())) == 81
    for b in packed[0]:
        assert all(((int(b) >> (2 * i)) & 3) != 3 for i in range(4))
    back, n_res = oracle.unpack(packed, 324)
    assert n_res == 0
    assert np.array_equal(back.reshape(-1, 4), vals)


def test_pack_random_round_trip_64x1536():
    # Hetman-2b section 8 Test 5 shape: N=64, K=1536
    rng = np.random.default_rng(5)
    q = rng.integers(-1, 2, (64, 1536)).astype(np.int8)
    packed = oracle.pack(q)
    assert packed.shape == (64, 384)
    back, n_res = oracle.unpack(packed, 1536)
    assert n_res == 0 and np.array_equal(back, q)


def test_unpack_flags_reserved_code():
    # 0xFF holds four 0b11 fields; 0x7D = 0b01111101 holds (LSB first) 01, 11, 11, 01
    back, n_res = oracle.unpack(np.array([[0xFF, 0x7D]], np.uint8), 8)
    assert n_res == 6
    assert back.tolist() == [[0, 0, 0, 0, 0, 0, 0, 0]]


# Hetman-2b section 3 layouts ("Format 0" = encoding 1, "Format 1" = encoding 2)
FORMATS = {"F0": 1, "F1": 2}


def test_pack_formats_hand_worked_bytes():
    for ln in golden_lines("pack_bytes_formats.txt"):
        fmt, *vals, byte = ln.split()
        q = np.array([[int(v) for v in vals]], np.int8)
        assert oracle.pack_format(q, FORMATS[fmt])[0, 0] == int(byte, 16), ln


def test_pack_formats_test13_round_trip_and_all_tuples():
    # Hetman-2b section 8 Test 13 (Format 1 round trip), and the same for
    # every 4-tuple in both layouts
    t13 = np.array([[-1, 0, 1, -1], [1, -1, 0, 1]], np.int8)
    vals = np.array(np.meshgrid(*[[-1, 0, 1]] * 4, indexing="ij")).reshape(4, -1).T.astype(np.int8)
    for enc in (1, 2):
        assert np.array_equal(oracle.unpack_format(oracle.pack_format(t13, enc), 4, enc), t13)
        packed = oracle.pack_format(vals.reshape(1, -1), enc)
        assert len(set(packed[0].tolist())) == 81
        assert np.array_equal(oracle.unpack_format(packed, 324, enc).reshape(-1, 4), vals)


def test_unpack_formats_every_byte_against_the_code_table():
    # the page's stated codes (reserved field reads as 0), not its formulas
    table = {1: {0b00: 0, 0b01: 1, 0b11: -1, 0b10: 0}, 2: {0b00: 0, 0b01: 1, 0b10: -1, 0b11: 0},
             0: {0b00: -1, 0b01: 0, 0b10: 1, 0b11: 0}}
    allb = np.arange(256, dtype=np.uint8).reshape(1, 256)
    for enc, tab in table.items():
        got = oracle.unpack_format(allb, 1024, enc).reshape(256, 4)
        want = np.array([[tab[(b >> (2 * i)) & 3] for i in range(4)] for b in range(256)], np.int8)
        assert np.array_equal(got, want), enc


def test_contraction_in_every_layout_equals_dense():
    rng = np.random.default_rng(11)
    q = rng.integers(-1, 2, (7, 192)).astype(np.int8)
    xq = rng.integers(-127, 128, (5, 192)).astype(np.int8)
    dense = xq.astype(np.int64) @ q.astype(np.int64).T
    for enc in (0, 1, 2):
        acc = oracle.matmul_addsub_format(xq, oracle.pack_format(q, enc), enc)
        assert np.array_equal(acc, dense), enc
    # reserved fields contribute nothing: a row of them gives 0
    res = {1: 0xAA, 2: 0xFF}
    for enc, b in res.items():
        packed = np.full((1, 48), b, np.uint8)
        assert np.all(oracle.matmul_addsub_format(xq, packed, enc) == 0)


def test_quantize_pack_layouts_carry_the_same_codes():
    W = S.normal((9, 256), 0.02, 12, 9)
    p0, g0 = oracle.quantize_pack(W, per_row=True)
    q0, _ = oracle.unpack(p0, 256)
    for enc in (1, 2):
        p, g = oracle.quantize_pack(W, per_row=True, encoding=enc)
        assert np.array_equal(g, g0)
        assert np.array_equal(oracle.unpack_format(p, 256, enc), q0)


def test_threshold_rule_hand_worked_rows():
    for ln in golden_lines("threshold_codes.txt"):
        ratio, ws, codes = [f.strip() for f in ln.split("|")]
        w = np.array([[float(v) for v in ws.split()]], np.float32)
        p, g = oracle.quantize_pack_threshold(w, per_row=True, ratio=float(ratio))
        q, n_res = oracle.unpack(p, 4)
        assert n_res == 0
        assert q[0].tolist() == [int(c) for c in codes.split()], ln


def test_threshold_rule_one_half_matches_round_rule_off_ties():
    # ratio 0.5: w > gamma/2 is the round rule's |w/gamma| > 0.5 except where the
    # fp32 quotient lands exactly on 0.5 (the round rule then gives 0, as strict > does,
    # unless the quotient rounded up onto 0.5 from below or down from above)
    W = S.normal((64, 512), 0.02, 21, 64)
    for per_row in (True, False):
        p_round, g = oracle.quantize_pack(W, per_row=per_row)
        q_round, _ = oracle.unpack(p_round, 512)
        p_thr, g2 = oracle.quantize_pack_threshold(W, per_row=per_row, ratio=0.5)
        q_thr, _ = oracle.unpack(p_thr, 512)
        assert np.array_equal(g, g2)
        gg = np.broadcast_to(g[:, None] if per_row else g, W.shape).astype(np.float32)
        tie = np.abs(W / gg) == np.float32(0.5)
        assert np.array_equal(q_round[~tie], q_thr[~tie])


def test_threshold_rule_boundaries_are_strict():
    # a row whose mean is exactly 1: w = 1 is not above tau = 1, the next float is
    w = np.array([[1.0, 1.0, 1.0, 1.0, 0.5, 1.5, 1.0, 1.0]], np.float32)  # mean |w| = 1
    q = oracle.ternary_codes_threshold(w, np.array([1.0], np.float32), True, 1.0)
    assert q[0].tolist() == [0, 0, 0, 0, 0, 1, 0, 0]
    up = np.nextafter(np.float32(1.0), np.float32(2.0))
    q = oracle.ternary_codes_threshold(np.array([[up, -up, 1.0, -1.0]], np.float32),
                                       np.array([1.0], np.float32), True, 1.0)
    assert q[0].tolist() == [1, -1, 0, 0]


def test_packed_size_and_compression():
    for ln in golden_lines("sizes.txt"):
        N, K, nbytes, f32bytes = map(int, ln.split())
        assert N * K * 4 == f32bytes
        # size of the packed array the oracle produces for an N x K matrix
        q = np.zeros((1, K), np.int8)
        assert oracle.pack(q).nbytes * N == nbytes
        assert f32bytes // nbytes == 16


# --------------------------------------------------------------------------
# gamma = mean |w|
# --------------------------------------------------------------------------

def test_gamma_constant_magnitude_exact():
    rng = np.random.default_rng(1)
    for c in [0.02, 1.0, 3.0e-3, 7.25, np.float32(1.0) / np.float32(3.0)]:
        c = np.float32(c)
        w = (np.where(rng.random(1000) < 0.5, -1, 1) * c).astype(np.float32)
        assert oracle.absmean_gamma(w) == c


def test_gamma_ties_round_to_even():
    one = np.float32(1.0)
    u = np.float32(2.0 ** -23)
    # mean = 1 + 2^-24: halfway between 1 (even) and 1 + 2^-23 (odd) -> 1
    assert oracle.absmean_gamma(np.array([one, one + u], np.float32)) == one
    # mean = 1 + 1.5 * 2^-23: halfway between 1+2^-23 (odd) and 1+2^-22 (even) -> 1+2^-22
    w = np.array([one + u, one + 2 * u], np.float32)
    assert oracle.absmean_gamma(w) == np.float32(1.0 + 2.0 ** -22)
    # just above the tie rounds up
    w = np.array([one, one + u, one + u], np.float32)  # mean = 1 + (2/3) 2^-23
    assert oracle.absmean_gamma(w) == one + u


def test_gamma_matches_exact_rational_mean():
    rng = np.random.default_rng(2)
    for trial in range(40):
        n = int(rng.integers(1, 300))
        scale = 10.0 ** rng.uniform(-5, 3)
        w = (rng.standard_normal(n) * scale).astype(np.float32)
        if trial % 5 == 0:  # mix in very different magnitudes
            w[: n // 2] *= np.float32(1e-20)
        exact = sum(Fraction(abs(float(v))) for v in w) / n
        expect = max(f32_round_rational(exact), np.float32(1e-6))
        assert oracle.absmean_gamma(w) == expect


def test_gamma_order_independent_and_large_n():
    rng = np.random.default_rng(3)
    w = S.normal((1 << 16,), 0.02, 0, 9)
    g = oracle.absmean_gamma(w)
    for _ in range(3):
        assert oracle.absmean_gamma(rng.permutation(w)) == g
    assert abs(float(g) - np.abs(w.astype(np.float64)).mean()) <= 1e-7 * float(g)
    big = np.concatenate([np.full(1 << 20, 0.75, np.float32), np.full(1 << 20, 0.25, np.float32)])
    assert oracle.absmean_gamma(big) == np.float32(0.5)


def test_gamma_eps_floor():
    assert oracle.absmean_gamma(np.zeros(64, np.float32)) == np.float32(1e-6)
    assert oracle.absmean_gamma(np.full(64, 1e-9, np.float32)) == np.float32(1e-6)
    # subnormal path of the exact rounding (eps = 0 exposes it)
    tiny = np.full(3, np.float32(2.0 ** -149), np.float32)
    assert oracle.absmean_gamma(tiny, eps=0.0) == np.float32(2.0 ** -149)
    two_tiny = np.array([2.0 ** -149, 0.0], np.float32)  # mean = 2^-150, tie -> 0 (even)
    assert oracle.absmean_gamma(two_tiny, eps=0.0) == np.float32(0.0)


def test_gamma_per_row_equals_row_wise_per_tensor():
    W = S.normal((16, 256), 0.02, 0, 11)
    _, g_rows = oracle.quantize_pack(W, per_row=True)
    for n in range(16):
        assert g_rows[n] == oracle.absmean_gamma(W[n])
    _, g_t = oracle.quantize_pack(W, per_row=False)
    assert g_t[0] == oracle.absmean_gamma(W.reshape(-1))


# --------------------------------------------------------------------------
# ternary codes
# --------------------------------------------------------------------------

def test_codes_ties_and_clamp():
    g = np.array([1.0], np.float32)
    half_up = np.nextafter(np.float32(0.5), np.float32(1))
    w = np.array([[0.5, -0.5, 1.5, -1.5, 2.5, -2.5, half_up, -half_up, 0.0, 1e30, -1e30, 0.49999997]],
                 np.float32)
    q = oracle.ternary_codes(w, g, per_row=False)
    assert q.tolist() == [[0, 0, 1, -1, 1, -1, 1, -1, 0, 1, -1, 0]]


def test_codes_nonzero_fraction_closed_forms():
    # N(0, s): gamma -> s*sqrt(2/pi); P(|w| > gamma/2) = erfc(sqrt(2/pi)/2 / sqrt(2))
    W = S.normal((512, 512), 0.02, 0, 12)
    p, g = oracle.quantize_pack(W, per_row=False)
    q, _ = oracle.unpack(p, 512)
    expect = math.erfc(math.sqrt(2 / math.pi) * 0.5 / math.sqrt(2))
    assert abs((q != 0).mean() - expect) < 0.005
    assert set(np.unique(q).tolist()) <= {-1, 0, 1}
    # Laplace(0, b): gamma -> b; P(|w| > b/2) = exp(-1/2)
    W = S.laplace((512, 512), 0.02, 0, 13)
    p, g = oracle.quantize_pack(W, per_row=True)
    q, _ = oracle.unpack(p, 512)
    assert abs((q != 0).mean() - math.exp(-0.5)) < 0.005
    # sign agreement: a nonzero code always has the sign of its weight
    assert np.all(q * np.sign(W) >= 0)


def test_codes_per_row_uses_row_gamma():
    W = np.array([[1.0, 0.4, -0.4, 0.0], [100.0, 40.0, -60.0, 0.0]], np.float32)
    g = np.array([1.0, 100.0], np.float32)
    assert oracle.ternary_codes(W, g, per_row=True).tolist() == [[1, 0, 0, 0], [1, 0, -1, 0]]


def test_sanitize_weights_mapping():
    w = np.array([np.nan, np.inf, -np.inf, 0.5], np.float32)
    assert oracle.sanitize_weights(w).tolist() == [0.0, 1.0, -1.0, 0.5]


# --------------------------------------------------------------------------
# activation quantisation
# --------------------------------------------------------------------------

def test_act_quant_hand_case():
    for ln in golden_lines("act_quant_cases.txt"):
        xs, qs = ln.split("|")
        x = np.array([[float(v) for v in xs.split()]], np.float32)
        xq, sx, rs = oracle.act_quant(x)
        assert xq[0].tolist() == [int(v) for v in qs.split()]
        assert sx[0] == np.float32(1.0) / np.float32(127.0)
        assert rs[0] == sum(int(v) for v in qs.split())


def test_act_quant_invariants():
    X = S.decode_acts(8, 4096)
    xq, sx, rs = oracle.act_quant(X)
    assert xq.min() >= -127 and xq.max() <= 127
    amax = np.abs(X).max(axis=1)
    arg = np.abs(X).argmax(axis=1)
    for m in range(8):
        assert abs(int(xq[m, arg[m]])) == 127
        assert sx[m] == np.float32(amax[m]) / np.float32(127.0)
        assert rs[m] == int(xq[m].astype(np.int64).sum())
    # |x_q - x/s_x| <= 1/2 + tiny (round to nearest)
    err = np.abs(xq - X.astype(np.float64) / sx[:, None].astype(np.float64))
    assert err.max() <= 0.5 + 1e-4
    # exact power-of-two scaling leaves every code unchanged
    xq2, sx2, _ = oracle.act_quant(X * np.float32(8.0))
    assert np.array_equal(xq, xq2) and np.array_equal(sx2, sx * np.float32(8.0))


def test_act_quant_zero_token_and_eta_clamp():
    xq, sx, rs = oracle.act_quant(np.zeros((1, 64), np.float32))
    assert not xq.any() and sx[0] == np.float32(1e-6) / np.float32(127) and rs[0] == 0
    # Hetman-2b section 8 Test 4: gain clamp keeps eta within [0.05, 40]
    big = S.normal((2, 512), 500.0, 0, 21)
    _, sx, _ = oracle.act_quant(big, clamp_eta=True)
    assert np.all(sx == np.float32(40.0) / np.float32(127.0))
    tiny = S.normal((2, 512), 1e-5, 0, 22)
    xq, sx, _ = oracle.act_quant(tiny, clamp_eta=True)
    assert np.all(sx == np.float32(0.05) / np.float32(127.0))
    assert np.abs(xq).max() < 5


# --------------------------------------------------------------------------
# contraction and rescale
# --------------------------------------------------------------------------

def test_matmul_forms_agree_and_match_library_matmul():
    rng = np.random.default_rng(7)
    for M, N, K in [(1, 1, 4), (3, 5, 8), (8, 8, 64), (2, 7, 128)]:
        xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
        q = rng.integers(-1, 2, (N, K)).astype(np.int8)
        a_dense = oracle.matmul_dense(xq, q)
        a_addsub = oracle.matmul_addsub(xq, oracle.pack(q))
        a_lib = xq.astype(np.int64) @ q.T.astype(np.int64)
        assert np.array_equal(a_dense, a_lib) and np.array_equal(a_addsub, a_lib)


def test_matmul_special_weights():
    rng = np.random.default_rng(8)
    xq = rng.integers(-127, 128, (4, 256)).astype(np.int8)
    rowsum = xq.astype(np.int64).sum(axis=1)
    for val, expect in [(1, rowsum), (-1, -rowsum), (0, 0 * rowsum)]:
        q = np.full((3, 256), val, np.int8)
        acc = oracle.matmul_addsub(xq, oracle.pack(q))
        assert np.all(acc == expect[:, None])


def test_single_layer_workload_end_to_end_consistency():
    W, X = S.single_layer()
    packed, g = oracle.quantize_pack(W, per_row=False)
    q, _ = oracle.unpack(packed, 512)
    xq, sx, _ = oracle.act_quant(X)
    acc = oracle.matmul_addsub(xq, packed)
    assert np.array_equal(acc, xq.astype(np.int64) @ q.T.astype(np.int64))
    y = oracle.dequant(acc, g, sx, per_row=False)
    # against a dense float64 product of the dequantised operands
    ref = (xq * sx[:, None].astype(np.float64)) @ (q * np.float64(g[0])).T
    assert np.allclose(y, ref, rtol=1e-6, atol=1e-12)  # acc == 0 gives y == 0, ref ~1e-18


def test_dequant_correct_rounding_and_zero():
    rng = np.random.default_rng(9)
    acc = rng.integers(-500000, 500000, (6, 9)).astype(np.int32)
    acc[0, 0] = 0
    g = (rng.random(9) * 0.05 + 1e-3).astype(np.float32)
    sx = (rng.random(6) * 0.1 + 1e-3).astype(np.float32)
    y = oracle.dequant(acc, g, sx, per_row=True)
    assert y[0, 0] == 0.0
    for m in range(6):
        for n in range(9):
            exact = Fraction(int(acc[m, n])) * Fraction(float(g[n])) * Fraction(float(sx[m]))
            r = f32_round_rational(abs(exact))
            assert abs(y[m, n]) == r or abs(y[m, n]) in (np.nextafter(r, np.float32(0)),
                                                          np.nextafter(r, np.float32(np.inf)))
            assert np.sign(y[m, n]) == np.sign(float(exact))


def test_dequant_bias_correct_rounding():
    # [H] section 5 step 6 with the layer bias: acc * gamma * s_x + bias, one rounding
    rng = np.random.default_rng(19)
    acc = rng.integers(-500000, 500000, (5, 7)).astype(np.int32)
    acc[0, 0] = 0
    g = (rng.random(7) * 0.05 + 1e-3).astype(np.float32)
    sx = (rng.random(5) * 0.1 + 1e-3).astype(np.float32)
    b = (rng.standard_normal(7) * 0.5).astype(np.float32)
    y = oracle.dequant_bias(acc, g, sx, True, b)
    assert y[0, 0] == b[0]
    for m in range(5):
        for n in range(7):
            exact = Fraction(int(acc[m, n])) * Fraction(float(g[n])) * Fraction(float(sx[m])) + Fraction(float(b[n]))
            r = f32_round_rational(abs(exact))
            assert abs(y[m, n]) in (r, np.nextafter(r, np.float32(0)), np.nextafter(r, np.float32(np.inf)))
            assert np.sign(y[m, n]) == np.sign(float(exact))
    assert np.array_equal(oracle.dequant_bias(acc, g, sx, True, None), oracle.dequant(acc, g, sx, True))


def test_int_epilogue_hand_worked():
    for ln in golden_lines("int_epilogue.txt"):
        a, b, sh, want = map(int, ln.split())
        out = oracle.int_epilogue(np.array([[a]], np.int32), np.array([b], np.int32), sh)
        assert out[0, 0] == want, ln


def test_swiglu_act_closed_forms_and_clamp():
    # Hetman-2b section 6 SwiGLUClamped: clamp(SiLU(gate) * up, -10, 10).
    # sigmoid(ln 3) = 3/4 exactly; SiLU(v) - SiLU(-v) = v; SiLU(0) = 0.
    ln3 = math.log(3.0)
    a = oracle.swiglu_act(np.array([0.0, ln3], np.float32), np.array([1.0, 1.0], np.float32))
    assert a[0] == 0.0
    assert abs(float(a[1]) - 0.75 * float(np.float32(ln3))) <= 2e-7
    v = S.normal((1, 257), 2.0, 23, 1)[0]
    ones = np.ones_like(v)
    diff = oracle.swiglu_act(v, ones, 1e6).astype(np.float64) - oracle.swiglu_act(-v, ones, 1e6).astype(np.float64)
    assert np.all(np.abs(diff - v.astype(np.float64)) <= 3e-7 * np.maximum(1.0, np.abs(v)))
    # the clamp bounds both signs; it is the last step (large gate, opposite signs)
    big = oracle.swiglu_act(np.array([10.0, 5.0, 50.0], np.float32), np.array([10.0, -5.0, 0.1], np.float32))
    assert big[0] == 10.0 and big[1] == -10.0 and abs(float(big[2]) - 5.0) < 1e-5
    assert np.array_equal(oracle.swiglu_act(np.array([3.0], np.float32), np.array([1.0], np.float32), 1.5),
                          np.array([1.5], np.float32))


def test_swiglu_mlp_is_the_composition():
    # gate and up see the same x; the down projection sees the clamped activation
    M, d, f = 3, 512, 1024
    X = S.student_t3((M, d), 24, M)
    packs = [oracle.quantize_pack(S.normal(shape, 0.02, 25 + i, shape[0]), per_row=False)
             for i, shape in enumerate([(f, d), (f, d), (d, f)])]
    y, act, xq, yg, yu = oracle.swiglu_mlp(X, packs[0], packs[1], packs[2], per_row=False)
    assert np.array_equal(yg, oracle.bitlinear(X, *packs[0], False)[0])
    assert np.array_equal(act, oracle.swiglu_act(yg, yu))
    assert np.abs(act).max() <= 10.0
    assert np.array_equal(y, oracle.bitlinear(act, *packs[2], False)[0])


# --------------------------------------------------------------------------
# FWHT-512
# --------------------------------------------------------------------------

def test_fwht_matches_explicit_sylvester_product():
    H = scipy.linalg.hadamard(512).astype(np.int64)
    assert np.array_equal(H @ H, 512 * np.eye(512, dtype=np.int64))
    X = S.normal((8, 1536), 1.0, 0, 31)
    Y = oracle.fwht512(X)
    ref = (X.astype(np.float64).reshape(8, 3, 512) @ H.T.astype(np.float64)) / math.sqrt(512.0)
    ref = ref.reshape(8, 1536)
    assert np.linalg.norm(Y - ref) <= 1e-6 * np.linalg.norm(ref)
    # unnormalised transform is the integer Hadamard product
    Xi = np.random.default_rng(4).integers(-8, 8, (2, 512)).astype(np.float32)
    assert np.array_equal(oracle.fwht512(Xi, normalize=False).astype(np.int64),
                          Xi.astype(np.int64) @ H.T)


def test_fwht_isometry_involution_and_constant():
    # Hetman-2b section 8 Tests 1 and 2 (randn(8, 512), tolerance 1e-5)
    X = S.normal((8, 512), 1.0, 0, 32)
    Y = oracle.fwht512(X)
    assert np.abs(np.linalg.norm(X, axis=1) - np.linalg.norm(Y, axis=1)).max() < 1e-5
    assert np.abs(oracle.fwht512(Y) - X).max() < 1e-5
    assert F32_ONE_OVER_SQRT512 == np.float32(1.0 / math.sqrt(512.0))
    e0 = np.zeros((1, 512), np.float32)
    e0[0, 0] = 1
    assert np.all(oracle.fwht512(e0) == F32_ONE_OVER_SQRT512)


def test_fwht_spike_attenuation_golden():
    (ln,) = golden_lines("fwht_spike.txt")
    idx, val, peak, tol, max_peak = ln.split()
    x = np.zeros((1, 512), np.float32)
    x[0, int(idx)] = float(val)
    y = oracle.fwht512(x)[0]
    assert abs(np.abs(y).max() - float(peak)) < float(tol)
    assert np.abs(y).max() <= float(max_peak)
    c = np.float32(float(val)) * F32_ONE_OVER_SQRT512
    assert np.all(y[:256] == c) and np.all(y[256:] == -c)  # row 256 of H: + then -


def test_fwht_roundtrip_spike_closed_form():
    # Hetman-2b section 1 FastWalshHadamardTransform: a spike of 100 at 256 rotates to
    # +-100/sqrt(512) everywhere, eta = that + 1e-5, every code is +-127 (the value
    # sits 1e-5 below eta), the dequantised +-eta rotates back to a spike of
    # 512 * eta / sqrt(512) = 100 + 1e-5 * sqrt(512) and exact zeros elsewhere
    x = np.zeros((1, 512), np.float32)
    x[0, 256] = 100.0
    y, eta = oracle.fwht_roundtrip(x)
    c = float(F32_ONE_OVER_SQRT512)
    assert abs(float(eta[0]) - (100.0 * c + 1e-5)) < 1e-6
    assert abs(float(y[0, 256]) - (100.0 + 1e-5 * math.sqrt(512))) < 5e-5
    assert np.count_nonzero(y[0]) == 1


def test_fwht_roundtrip_gain_clamp_and_quench():
    # eta below eta_min / above eta_max is clamped; NaN reads as 0, +-inf as +-eta_max
    z, eta = oracle.fwht_roundtrip(np.zeros((1, 512), np.float32))
    assert eta[0] == np.float32(0.05) and not z.any()
    x = np.zeros((1, 512), np.float32)
    x[0, 0] = 1000.0  # rotates to 44.19 > eta_max = 40: codes saturate at 127
    y, eta = oracle.fwht_roundtrip(x)
    assert eta[0] == np.float32(40.0)
    step = np.float32(40.0) / np.float32(127.0)
    assert abs(float(y[0, 0]) - 512 * float(np.float32(127.0) * step) * float(F32_ONE_OVER_SQRT512)) < 1e-3
    xn = np.zeros((1, 512), np.float32)
    xn[0, 3] = np.nan
    xn[0, 7] = np.inf
    xf = np.zeros((1, 512), np.float32)
    xf[0, 7] = 40.0
    assert np.array_equal(oracle.fwht_roundtrip(xn)[0], oracle.fwht_roundtrip(xf)[0])


def test_fwht_roundtrip_error_bound():
    # the rotation is orthonormal, so ||y - x||_2 = ||dequant - x_rot||_2 <= sqrt(K) * step / 2
    X = S.student_t3((6, 1024), 22, 6)
    Y, eta = oracle.fwht_roundtrip(X)
    for r in range(6):
        step = float(eta[r]) / 127.0
        err = float(np.linalg.norm(Y[r].astype(np.float64) - X[r].astype(np.float64)))
        assert err <= math.sqrt(1024) * step / 2 * 1.001 + 1e-5


def test_fwht_blocks_are_independent():
    X = S.normal((2, 1536), 1.0, 0, 33)
    Y = oracle.fwht512(X)
    for b in range(3):
        assert np.array_equal(Y[:, b * 512:(b + 1) * 512], oracle.fwht512(X[:, b * 512:(b + 1) * 512]))


# --------------------------------------------------------------------------
# RMSNorm and the whole layer
# --------------------------------------------------------------------------

def test_rmsnorm_closed_forms():
    c = np.float32(3.0)
    y = oracle.rmsnorm(np.full((1, 64), c, np.float32))
    assert np.allclose(y, c / math.sqrt(9.0 + 1e-6), rtol=1e-7)
    X = S.normal((4, 2048), 1.0, 0, 41)
    g = S.normal((2048,), 1.0, 0, 42)
    Y = oracle.rmsnorm(X, g)
    for m in range(4):
        ms = math.fsum(float(v) * float(v) for v in X[m]) / 2048
        r = 1.0 / math.sqrt(ms + float(np.float32(1e-6)))
        ref = (X[m].astype(np.float64) * r * g.astype(np.float64)).astype(np.float32)
        assert np.abs(Y[m].view(np.int32) - ref.view(np.int32)).max() <= 1
        assert abs(np.mean(Y[m].astype(np.float64) ** 2 / g.astype(np.float64) ** 2) - 1.0) < 1e-5


def test_bitlinear_is_the_composition_of_its_steps():
    W, X = S.fused(M=3, N=64, K=1024)
    packed, g = oracle.quantize_pack(W, per_row=False)
    y, xq, sx, acc = oracle.bitlinear(X, packed, g, per_row=False)
    xr = oracle.fwht512(oracle.rmsnorm(X))
    xq2, sx2, _ = oracle.act_quant(xr)
    assert np.array_equal(xq, xq2) and np.array_equal(sx, sx2)
    acc2 = oracle.matmul_addsub(xq2, packed)
    assert np.array_equal(acc, acc2)
    assert np.array_equal(y, oracle.dequant(acc2, g, sx2, per_row=False))
    # sanitize path: non-finite inputs become finite outputs
    Xb = X.copy()
    Xb[0, 0], Xb[1, 5], Xb[2, 9] = np.nan, np.inf, -np.inf
    yb, _, sxb, _ = oracle.bitlinear(Xb, packed, g, per_row=False, sanitize=True)
    assert np.all(np.isfinite(yb)) and np.all(np.isfinite(sxb))


def test_bitlinear_float_gemm_parity_1536():
    # Hetman-2b section 8 Test 9: the float F.linear path and the integer
    # GEMV agree within 1e-4 at in = out = 1536, batch 1.
    W = S.normal((1536, 1536), 1.0 / math.sqrt(1536), 0, 51)
    X = S.normal((1, 1536), 1.0, 0, 52)
    packed, g = oracle.quantize_pack(W, per_row=False)
    y, xq, sx, acc = oracle.bitlinear(X, packed, g, per_row=False, clamp_eta=True)
    q, _ = oracle.unpack(packed, 1536)
    y_float = (xq.astype(np.float32) @ q.T.astype(np.float32)) * (g[0] / (np.float32(127.0) / (sx * np.float32(127.0))))
    assert np.abs(y_float - y).max() < 1e-4
