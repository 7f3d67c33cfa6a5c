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


def test_manual_threshold_hand_worked_rows():
    """Foundry's manual threshold: codes and packed bytes worked by hand, the
    stored scale equal to the threshold itself, every layout decoding to the
    same codes."""
    for ln in golden_lines("abs_threshold_codes.txt"):
        t, ws, codes, bytes_ = [f.strip() for f in ln.split("|")]
        w = np.array([[float(v) for v in ws.split()]], np.float32)
        p, g = oracle.quantize_pack_abs_threshold(w, float(t))
        assert g.tolist() == [np.float32(float(t))], ln
        assert p[0].tolist() == [int(b, 16) for b in bytes_.split()], ln
        want = [int(c) for c in codes.split()]
        for enc in (1, 2):
            pe, _ = oracle.quantize_pack_abs_threshold(w, float(t), encoding=enc)
            assert oracle.unpack_format(pe, 8, enc)[0].tolist() == want, (ln, enc)


def test_manual_threshold_limits_and_sanitising():
    """t = 0 is the sign (zeros stay 0); t above every |w| gives all zeros; with
    t = the row's mean |w| it is the absmean threshold rule (ratio 1); NaN -> 0
    and +-inf -> +-1 under sanitising."""
    W = S.laplace((16, 256), 0.02, 22, 16)
    p, g = oracle.quantize_pack_abs_threshold(W, 0.0)
    q, _ = oracle.unpack(p, 256)
    assert np.array_equal(q, np.sign(W).astype(np.int8))
    p, _ = oracle.quantize_pack_abs_threshold(W, float(np.abs(W).max()))
    assert np.all(oracle.unpack(p, 256)[0] == 0)
    for n in range(3):
        row = W[n:n + 1]
        gamma = oracle.absmean_gamma(row)
        p_abs, _ = oracle.quantize_pack_abs_threshold(row, float(gamma))
        p_thr, _ = oracle.quantize_pack_threshold(row, per_row=True, ratio=1.0)
        assert np.array_equal(p_abs, p_thr)
    bad = np.array([[np.nan, np.inf, -np.inf, 0.5]], np.float32)
    p, _ = oracle.quantize_pack_abs_threshold(bad, 0.75, sanitize=True)
    assert oracle.unpack(p, 4)[0][0].tolist() == [0, 1, -1, 0]


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


# --------------------------------------------------------------------------
# training: gradient through the layer, STE, stochastic flip
# --------------------------------------------------------------------------

def _codes_by_table(packed, K):
    """Foundry's code table applied byte by byte (independent of the oracle's unpack)."""
    tab = {0b00: -1, 0b01: 0, 0b10: 1}
    N = packed.shape[0]
    q = np.empty((N, K), np.int64)
    for n in range(N):
        for j in range(K // 4):
            b = int(packed[n, j])
            for i in range(4):
                q[n, 4 * j + i] = tab[(b >> (2 * i)) & 3]
    return q


def test_backward_input_adjoint_identity_exact():
    # <dX, x_q> = <dY * gamma, x_q W^T> exactly: small integers, a power-of-two
    # gamma, so every sum is exact.  A transposed operand, a dropped term or a
    # wrong sign breaks it (N != K).
    rng = np.random.default_rng(21)
    M, N, K = 5, 7, 64
    q = rng.integers(-1, 2, (N, K)).astype(np.int8)
    packed = oracle.pack(q)
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    dY = rng.integers(-8, 9, (M, N)).astype(np.float32)
    for per_row, gamma in ((False, np.float32(0.25)), (True, np.float32(2.0) ** rng.integers(-3, 3, N))):
        gamma = np.atleast_1d(gamma).astype(np.float32)
        dX = oracle.backward_input(dY, packed, gamma, per_row, K)
        acc = oracle.matmul_addsub(xq, packed).astype(np.float64)
        g = gamma.astype(np.float64) if per_row else np.full(N, float(gamma[0]))
        lhs = float(np.sum(dX.astype(np.float64) * xq.astype(np.float64)))
        rhs = float(np.sum(dY.astype(np.float64) * g[None, :] * acc))
        assert lhs == rhs


def test_backward_input_closed_forms():
    M, N, K = 3, 5, 64
    dY = np.arange(1, M * N + 1, dtype=np.float32).reshape(M, N) / np.float32(8)
    # all weights +1: every input feature receives the row sum of dY * gamma
    ones = oracle.pack(np.ones((N, K), np.int8))
    dX = oracle.backward_input(dY, ones, np.float32(0.5), False, K)
    assert np.all(dX == (dY.sum(axis=1) * np.float32(0.5))[:, None])
    # one-hot dY picks one weight row, scaled by its gamma
    rng = np.random.default_rng(22)
    q = rng.integers(-1, 2, (N, K)).astype(np.int8)
    gam = np.array([0.5, 0.25, 2.0, 1.0, 4.0], np.float32)
    onehot = np.zeros((1, N), np.float32)
    onehot[0, 3] = 3.0
    dX = oracle.backward_input(onehot, oracle.pack(q), gam, True, K)
    assert np.array_equal(dX[0], (3.0 * 1.0 * q[3]).astype(np.float32))
    # zero gradient gives zero; the accumulate form adds to what is there
    assert np.all(oracle.backward_input(np.zeros((M, N), np.float32), oracle.pack(q), gam, True, K) == 0)
    base = np.full((M, K), 1.5, np.float32)
    acc = oracle.backward_input(dY, ones, np.float32(0.5), False, K, dX_in=base)
    assert np.all(acc == (dY.sum(axis=1) * np.float32(0.5))[:, None] + np.float32(1.5))


def test_backward_input_matches_library_matmul_and_rounds_once():
    rng = np.random.default_rng(23)
    M, N, K = 6, 37, 128
    q = rng.integers(-1, 2, (N, K)).astype(np.int8)
    packed = oracle.pack(q)
    dY = rng.standard_normal((M, N)).astype(np.float32)
    gam = (rng.random(N).astype(np.float32) + np.float32(0.5)).astype(np.float32)
    rs = (rng.random(M).astype(np.float32) * np.float32(0.01)).astype(np.float32)
    dX = oracle.backward_input(dY, packed, gam, True, K, row_scale=rs)
    g = (dY * gam[None, :]).astype(np.float32).astype(np.float64)  # one fp32 product per term
    ref = (g @ _codes_by_table(packed, K).astype(np.float64)) * rs.astype(np.float64)[:, None]
    assert np.array_equal(dX, ref.astype(np.float32))
    # the same codes in Hetman-2b's layouts give the same gradient
    for enc in (1, 2):
        assert np.array_equal(oracle.backward_input(dY, oracle.pack_format(q, enc), gam, True, K,
                                                    row_scale=rs, encoding=enc), dX)


def test_ste_backward_closed_forms():
    one_tenth = np.float32(0.1)
    cases = [  # w, gamma, tau, grad, sanitize -> expected (exact rational, rounded once to fp32 where noted)
        (0.25, 0.5, 1.0, 1.0, False, np.float32(2.0)),       # |w/gamma| = 0.5: inside, grad / gamma
        (0.5, 0.5, 1.0, 1.0, False, np.float32(2.0)),        # |w/gamma| = tau exactly: inside (<=)
        (-0.5, 0.5, 1.0, -1.0, False, np.float32(-2.0)),
        (0.75, 0.5, 1.5, 3.0, False, np.float32(6.0)),       # 1.5 <= tau = 1.5
        (float("nan"), 0.5, 1.0, -1.0, True, np.float32(-2.0)),   # quench nan -> 0: inside
        (3.0, 3.0, 1.0, 1.0, False, f32_round_rational(Fraction(1, 3))),  # 1/3 rounded once
    ]
    for w, gm, tau, gr, san, want in cases:
        got = oracle.ste_backward(np.array([[gr]], np.float32), np.array([[w]], np.float32), np.float32(gm),
                                  False, tau, san)[0, 0]
        assert got == want, (w, gm, tau, gr, san, got, want)
    # outside the band the gradient is damped by the fp32 constant 0.1:
    # fp32(fp32(grad / gamma) * fp32(0.1)), checked with exact rationals
    t = Fraction(float(one_tenth))
    outside = [(0.75, 0.5, 3.0, Fraction(6)), (-0.75, 0.5, 3.0, Fraction(6)),
               (float("inf"), 0.5, 1.0, Fraction(2)),    # sanitised +inf -> 1: |1/0.5| = 2 > 1
               (float("nan"), 0.5, 1.0, Fraction(2))]    # nan kept: |nan| <= tau is false
    for w, gm, gr, quotient in outside:
        san = math.isinf(w)
        got = oracle.ste_backward(np.array([[gr]], np.float32), np.array([[w]], np.float32), np.float32(gm),
                                  False, 1.0, san)[0, 0]
        assert got == f32_round_rational(quotient * t), (w, got)
    # the next float above tau * gamma leaves the band once the quotient rounds above tau
    w = np.nextafter(np.float32(3.0), np.float32(4.0))
    got = oracle.ste_backward(np.ones((1, 1), np.float32), np.array([[w]], np.float32), np.float32(3.0),
                              False, 1.0)[0, 0]
    assert got == f32_round_rational(Fraction(float(f32_round_rational(Fraction(1, 3)))) * t)


def test_ste_backward_per_row_uses_row_gamma():
    rng = np.random.default_rng(24)
    w = rng.standard_normal((4, 64)).astype(np.float32)
    gr = rng.standard_normal((4, 64)).astype(np.float32)
    gam = np.array([0.5, 1.0, 2.0, 0.25], np.float32)
    got = oracle.ste_backward(gr, w, gam, True)
    for n in range(4):
        assert np.array_equal(got[n], oracle.ste_backward(gr[n:n + 1], w[n:n + 1], gam[n], False)[0])


def test_xorshift64_worked_steps():
    # seed 1 worked by hand from the (13, 7, 17) definition:
    #   1 ^ 1<<13 = 0x2001;  ^ >>7 -> 0x2041;  ^ <<17 -> 0x40822041
    #   0x40822041 ^ <<13: 0x81044082000 ^ 0x40822041 = 0x810048A0041
    #   ^ >>7: 0x810048A0041 ^ 0x1020091400 = 0x80024831441
    #   ^ <<17: 0x1000490628820000 ^ 0x80024831441 = 0x100041060C011441
    out, st = oracle.xorshift64(1, 2)
    assert out == [0x40822041, 0x100041060C011441] and st == out[-1]
    assert oracle.seed(1) == 1 and oracle.seed(0) != 0
    assert oracle.xorshift64(0, 3)[0] == [0, 0, 0]  # why seed 0 is mapped away


def _gf2_columns(step):
    return [step(1 << b) for b in range(64)]


def _gf2_apply(cols, v):
    r = 0
    b = 0
    while v:
        if v & 1:
            r ^= cols[b]
        v >>= 1
        b += 1
    return r


def _gf2_mul(a, b):
    return [_gf2_apply(a, c) for c in b]


def _gf2_pow(cols, e):
    result = [1 << b for b in range(64)]
    base = cols
    while e:
        if e & 1:
            result = _gf2_mul(result, base)
        base = _gf2_mul(base, base)
        e >>= 1
    return result


def test_xorshift64_is_linear_with_maximal_period():
    # Treat the oracle's step as a black box.  It must be linear over GF(2),
    # and a generator of maximal period 2^64 - 1 has a transition matrix whose
    # order is exactly 2^64 - 1 = 3 * 5 * 17 * 257 * 641 * 65537 * 6700417.
    step = lambda v: oracle.xorshift64(v, 1)[1]
    rng = np.random.default_rng(25)
    for _ in range(20):
        a, b = (int(x) for x in rng.integers(0, 2 ** 63, 2, dtype=np.uint64))
        assert step(a ^ b) == step(a) ^ step(b)
    cols = _gf2_columns(step)
    ident = [1 << b for b in range(64)]
    order = 2 ** 64 - 1
    primes = [3, 5, 17, 257, 641, 65537, 6700417]
    assert math.prod(primes) == order
    assert _gf2_pow(cols, order) == ident
    for p in primes:
        assert _gf2_pow(cols, order // p) != ident, p


def test_stochastic_flip_deterministic_limits():
    rng = np.random.default_rng(26)
    N, K = 6, 64
    q = rng.integers(-1, 2, (N, K)).astype(np.int8)
    grad = rng.standard_normal((N, K)).astype(np.float32)
    grad[0, :8] = 0.0
    st0 = oracle.seed(7)
    for enc in (0, 1, 2):
        packed = oracle.pack_format(q, enc)
        # temperature 0: nothing moves, yet one draw per weight was taken
        out, st = oracle.stochastic_flip(packed, grad, 0.0, st0, enc)
        assert np.array_equal(out, packed) and st == oracle.xorshift64(st0, N * K)[1]
        # |grad| * T >= 1: every weight with a nonzero gradient steps toward -grad
        out, _ = oracle.stochastic_flip(packed, grad, 1e9, st0, enc)
        want = np.clip(q.astype(np.int64) - np.sign(grad).astype(np.int64), -1, 1)
        assert np.array_equal(oracle.unpack_format(out, K, enc), want.astype(np.int8)), enc
    # a NaN gradient never flips, an infinite one always does
    g2 = np.zeros((1, 64), np.float32)
    g2[0, 0], g2[0, 1] = np.nan, -np.inf
    zero = oracle.pack(np.zeros((1, 64), np.int8))
    out, _ = oracle.stochastic_flip(zero, g2, 0.5, st0)
    codes = oracle.unpack(out, 64)[0][0]
    assert codes[0] == 0 and codes[1] == 1 and np.all(codes[2:] == 0)


def test_stochastic_flip_rate_and_stream_order():
    # p = 0.3 everywhere on zero codes: the flipped fraction is binomial(n, 0.3)
    N, K = 64, 1024
    grad = np.full((N, K), 0.3, np.float32)
    grad[::2] *= -1
    zero = oracle.pack(np.zeros((N, K), np.int8))
    out, st = oracle.stochastic_flip(zero, grad, 1.0, oracle.seed(11))
    codes = oracle.unpack(out, K)[0].astype(np.int64)
    moved = codes != 0
    n = N * K
    assert abs(moved.sum() - 0.3 * n) < 5 * math.sqrt(n * 0.3 * 0.7)
    assert np.all(codes[moved] == -np.sign(grad[moved]))
    # the draw of weight i is the (i+1)-th output: splitting the rows over two
    # calls that carry the state gives the same codes
    a, st_a = oracle.stochastic_flip(zero[:N // 3], grad[:N // 3], 1.0, oracle.seed(11))
    b, st_b = oracle.stochastic_flip(zero[N // 3:], grad[N // 3:], 1.0, st_a)
    assert np.array_equal(np.concatenate([a, b]), out) and st_b == st
    # the comparison uses the top 24 bits of each output as u = (x >> 40) / 2^24
    xs, _ = oracle.xorshift64(oracle.seed(11), 64)
    g1 = np.full((1, 64), 0.5, np.float32)
    out1, _ = oracle.stochastic_flip(oracle.pack(np.zeros((1, 64), np.int8)), g1, 1.0, oracle.seed(11))
    want = np.array([-1 if (x >> 40) < (1 << 23) else 0 for x in xs], np.int8)
    assert np.array_equal(oracle.unpack(out1, 64)[0][0], want)
