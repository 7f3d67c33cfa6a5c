"""CPU-side checks of the C ABI: the library builds, loads and exports every
entry point include/tq.h declares, and argument validation rejects bad calls
with the documented status before touching the device (fake, never
dereferenced pointers; no compute call is made)."""
import ctypes
import os
import re

import pytest

import ternary_bit_linear_b200 as tq
from ternary_bit_linear_b200 import build as tqbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "tq.h")


@pytest.fixture(scope="module")
def lib():
    tqbuild.build()
    return tq.load()


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"TQ_API\s+[\w\s\*]+?\b(tq_\w+)\s*\(", src)


def test_header_declares_the_five_calls_and_helpers():
    names = set(declared_functions())
    for n in ["tq_quantize_ternary_pack", "tq_quantize_act_int8", "tq_fwht512",
              "tq_ternary_gemm", "tq_bitlinear_fused"]:
        assert n in names
    assert names == set(tq.SIGNATURES), "binding and header disagree"


def test_header_flag_values_match_binding():
    src = open(HEADER).read()
    flags = dict((k, int(v)) for k, v in re.findall(r"#define\s+TQ_(\w+)\s+\(1u\s*<<\s*(\d+)\)", src))
    py = {"GAMMA_PER_ROW": tq.GAMMA_PER_ROW, "FLAG_FWHT": tq.FLAG_FWHT, "FLAG_RMSNORM": tq.FLAG_RMSNORM,
          "FLAG_ETA_CLAMP": tq.FLAG_ETA_CLAMP, "FLAG_SANITIZE_NONFINITE": tq.FLAG_SANITIZE_NONFINITE,
          "FLAG_WEIGHTS_STATIC": tq.FLAG_WEIGHTS_STATIC, "FLAG_INPUTS_READY": tq.FLAG_INPUTS_READY,
          "FLAG_ACCUMULATE": tq.FLAG_ACCUMULATE, "FLAG_SHARED_INPUT": tq.FLAG_SHARED_INPUT}
    for name, value in py.items():
        assert name in flags, name
        assert value == 1 << flags[name], name
    assert len(set(py.values())) == len(py)
    enc = dict((k, int(v) << int(sh)) for k, v, sh in re.findall(r"#define\s+TQ_(ENC_\w+)\s+\((\d+)u\s*<<\s*(\d+)\)", src))
    assert enc == {"ENC_FOUNDRY": tq.ENC_FOUNDRY, "ENC_FORMAT0": tq.ENC_FORMAT0, "ENC_FORMAT1": tq.ENC_FORMAT1,
                   "ENC_MASK": tq.ENC_MASK}
    assert all(not (tq.ENC_MASK & v) for v in py.values())


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert lib.tq_version() == 100


def test_status_strings(lib):
    for code in range(8):
        assert lib.tq_status_string(code)
    assert b"unknown" in lib.tq_status_string(99)


def test_workspace_sizes(lib):
    assert lib.tq_pack_workspace_bytes(4096, 4096, tq.GAMMA_PER_ROW) == 0
    n = lib.tq_pack_workspace_bytes(11008, 4096, 0)
    assert n >= 16 + 16 and n < 1 << 20
    assert lib.tq_fused_workspace_bytes(512, 2048, tq.FLAG_FWHT) >= 512 * 2048 + 2 * 512 * 4


FAKE = 0x10000000  # 16-byte aligned, never dereferenced: validation fails first


def P(off=0):
    return ctypes.c_void_p(FAKE + off)


def test_pack_validation(lib):
    f = lib.tq_quantize_ternary_pack
    assert f(None, 4, 64, 1, P(), P(1 << 20), None, 0, None) == 1            # NULL
    assert f(P(), 4, 60, 1, P(1 << 20), P(2 << 20), None, 0, None) == 2      # K % 64
    assert f(P(), 0, 64, 1, P(1 << 20), P(2 << 20), None, 0, None) == 2      # N = 0
    assert f(P(4), 4, 64, 1, P(1 << 20), P(2 << 20), None, 0, None) == 3     # misaligned
    assert f(P(), 4, 64, 1 << 9, P(1 << 20), P(2 << 20), None, 0, None) == 4  # unknown flag
    assert f(P(), 4, 64, 1 | 3 << 7, P(1 << 20), P(2 << 20), None, 0, None) == 4  # reserved layout
    assert f(P(), 4, 64, 1, P(16), P(2 << 20), None, 0, None) == 4           # overlap w/packed
    assert f(P(), 4, 64, 0, P(1 << 20), P(2 << 20), None, 0, None) == 1      # needs workspace
    assert f(P(), 4, 64, 0, P(1 << 20), P(2 << 20), P(3 << 20), 8, None) == 4  # too small


def test_noalloc_validation(lib):
    """tq_quantize_ternary_pack_noalloc: its own limits, checked before any
    device work (the pointers are fake and never touched)."""
    f = lib.tq_quantize_ternary_pack_noalloc
    limit = 2048 * 65536  # per-tensor weights the fixed scratch array covers
    N, K = limit // 65536 + 1, 65536  # one row past the limit
    big = ctypes.c_void_p(1 << 40)
    assert f(big, N, K, 0, ctypes.c_void_p((1 << 40) + (1 << 36)), ctypes.c_void_p((1 << 40) + (1 << 37)),
             None) == 2                                                       # over the limit
    assert f(None, 4, 64, 0, P(1 << 20), P(2 << 20), None) == 1                # NULL
    assert f(P(4), 4, 64, 0, P(1 << 20), P(2 << 20), None) == 3                # misaligned
    assert f(P(), 4, 64, tq.FLAG_INPUTS_READY, P(1 << 20), P(2 << 20), None) == 4  # shared scratch: no overlap
    assert f(P(), 4, 64, 3 << 7, P(1 << 20), P(2 << 20), None) == 4            # reserved layout
    assert f(P(), 4, 60, 0, P(1 << 20), P(2 << 20), None) == 2                 # K % 64


def test_grouped_validation(lib):
    """tq_bitlinear_grouped: shape, flag, pointer-table and workspace checks
    before any device work (fake device pointers, never touched)."""
    f = lib.tq_bitlinear_grouped
    G, M, N, K = 3, 4, 64, 256
    arr = ctypes.c_void_p * G
    pk = arr(*[FAKE + (8 << 20) + i * (1 << 20) for i in range(G)])
    gm = arr(*[FAKE + (16 << 20) + i * 4096 for i in range(G)])
    ws_need = lib.tq_grouped_workspace_bytes(G, M, K, 0)
    assert ws_need >= G * M * K + 2 * G * M * 4
    assert lib.tq_grouped_workspace_bytes(G, M, K, tq.FLAG_SHARED_INPUT) < ws_need
    x, y, ws = P(), P(1 << 20), P(2 << 20)
    ok = [x, G, ctypes.cast(pk, ctypes.c_void_p), ctypes.cast(gm, ctypes.c_void_p), 0, M, N, K, y, ws, ws_need, None]

    def call(**kw):
        a = list(ok)
        names = ["x", "G", "packed", "gamma", "flags", "M", "N", "K", "y", "ws", "wsb", "stream"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return f(*a)
    assert call(x=None) == 1
    assert call(packed=None) == 1
    assert call(G=0) == 2 and call(G=65) == 2           # 1 <= G <= 64
    assert call(M=17) == 2 and call(M=0) == 2           # the small-M range
    assert call(K=8256) == 2 and call(K=100) == 2       # K <= 8192, K % 64 == 0
    assert call(flags=1 << 11) == 4                     # unknown flag
    assert call(flags=3 << 7) == 4                      # reserved layout
    assert call(wsb=ws_need - 1) == 4                   # workspace too small
    assert call(x=P(4)) == 3                            # misaligned
    assert call(y=P(64)) == 4                           # y overlaps x
    bad = arr(*([FAKE + (8 << 20)] * (G - 1) + [0]))
    assert call(packed=ctypes.cast(bad, ctypes.c_void_p)) == 1  # a NULL entry
    odd = arr(*([FAKE + (8 << 20)] * (G - 1) + [FAKE + (9 << 20) + 4]))
    assert call(packed=ctypes.cast(odd, ctypes.c_void_p)) == 3  # a misaligned entry


def test_pack_abs_threshold_validation(lib):
    f = lib.tq_quantize_ternary_pack_abs_threshold
    ok = [P(), 4, 64, 0, 0.05, P(1 << 20), P(2 << 20), None]
    for bad_t in (-0.01, float("nan"), float("inf")):
        a = list(ok)
        a[4] = bad_t
        assert f(*a) == 4, bad_t
    for flags, code in ((tq.GAMMA_PER_ROW, 4), (1 << 9, 4), (3 << 7, 4)):
        a = list(ok)
        a[3] = flags
        assert f(*a) == code, flags
    a = list(ok)
    a[0] = None
    assert f(*a) == 1
    a = list(ok)
    a[2] = 100
    assert f(*a) == 2
    a = list(ok)
    a[6] = P(4)
    assert f(*a) == 3
    a = list(ok)
    a[5] = P(16)  # packed overlaps w
    assert f(*a) == 4


def test_selftest_wait_validation(lib):
    f = lib.tq_selftest_wait_timeout
    assert f(999, 0, None) == 4            # below 1 us
    assert f(10 ** 9 + 1, 0, None) == 4    # above 1 s
    assert f(10 ** 6, 2, None) == 4       # sleeping must be 0 or 1


def test_pack_threshold_validation(lib):
    f = lib.tq_quantize_ternary_pack_threshold
    ok = [P(), 4, 64, 1, 0.55, P(1 << 20), P(2 << 20), None, 0, None]
    for bad_ratio in (0.0, -1.0, 65.0, float("nan"), float("inf")):
        args = list(ok)
        args[4] = bad_ratio
        assert f(*args) == 4, bad_ratio
    args = list(ok)
    args[0] = None
    assert f(*args) == 1
    args = list(ok)
    args[3] = 1 << 9
    assert f(*args) == 4


def test_act_and_fwht_validation(lib):
    f = lib.tq_quantize_act_int8
    assert f(P(), 2, 64, 0, 0.05, 40.0, P(1 << 20), P(2 << 20), None, None) == 1
    assert f(P(), 2, 96, 0, 0.05, 40.0, P(1 << 20), P(2 << 20), P(3 << 20), None) == 2
    assert f(P(), 2, 64, tq.FLAG_ETA_CLAMP, 0.0, 40.0, P(1 << 20), P(2 << 20), P(3 << 20), None) == 4
    assert f(P(), 2, 64, 0, 0.05, 40.0, P(112), P(2 << 20), P(3 << 20), None) == 4  # overlap
    g = lib.tq_fwht512
    assert g(P(), P(1 << 20), 2, 1000, 1, None) == 2
    assert g(P(), P(16), 2, 512, 1, None) == 4  # partial overlap (in place is allowed)


def test_gemm_and_fused_validation(lib):
    f = lib.tq_ternary_gemm
    args = [P(), P(1 << 20), P(2 << 20), P(3 << 20), P(4 << 20), 0, 8, 8, 64, P(5 << 20), None, None]
    bad = list(args)
    bad[5] = 4
    assert f(*bad) == 4
    bad[5] = 3 << 7  # reserved layout
    assert f(*bad) == 4
    bad = list(args)
    bad[8] = 32
    assert f(*bad) == 2
    bad = list(args)
    bad[9] = P(16)  # y overlaps x_q
    assert f(*bad) == 4
    bad = list(args)
    bad[2] = None
    assert f(*bad) == 1
    h = lib.tq_bitlinear_fused
    fused = [P(), None, 1e-6, 0.05, 40.0, tq.FLAG_FWHT, P(1 << 20), P(2 << 20), 4, 8, 640,
             P(3 << 20), None, None, P(4 << 20), 1 << 20, None]
    assert h(*fused) == 2  # FWHT needs K % 512 == 0
    fused[10] = 512
    fused[15] = 16
    assert h(*fused) == 4  # workspace too small
    fused[15] = 1 << 20
    fused[5] = tq.FLAG_FWHT | 3 << 7
    assert h(*fused) == 4  # reserved layout


def test_training_validation(lib):
    f = lib.tq_ternary_backward_input
    ws = lib.tq_backward_input_workspace_bytes(4, 40)
    assert ws >= 2 * 4 * 64 * 2 + 4 * 4 and lib.tq_backward_input_workspace_bytes(0, 8) == 0
    ok = [P(), P(1 << 20), P(2 << 20), None, 0, 4, 40, 128, P(3 << 20), P(4 << 20), ws, None]
    bad = list(ok); bad[0] = None
    assert f(*bad) == 1
    bad = list(ok); bad[7] = 96
    assert f(*bad) == 2                                   # K % 64
    bad = list(ok); bad[4] = 1 << 10
    assert f(*bad) == 4                                   # unknown flag
    bad = list(ok); bad[4] = 3 << 7
    assert f(*bad) == 4                                   # reserved layout
    bad = list(ok); bad[10] = ws - 16
    assert f(*bad) == 4                                   # workspace too small
    bad = list(ok); bad[8] = P(16)
    assert f(*bad) == 4                                   # dX overlaps dY
    bad = list(ok); bad[3] = P((5 << 20) + 4)
    assert f(*bad) == 3                                   # misaligned row_scale
    g = lib.tq_ste_backward
    ok = [P(), P(1 << 20), P(2 << 20), 4, 64, 1.0, 0, P(3 << 20), None]
    bad = list(ok); bad[5] = float("nan")
    assert g(*bad) == 4
    bad = list(ok); bad[5] = -1.0
    assert g(*bad) == 4
    bad = list(ok); bad[6] = tq.FLAG_FWHT
    assert g(*bad) == 4
    bad = list(ok); bad[7] = P(64)
    assert g(*bad) == 4                                   # partial overlap with grad
    bad = list(ok); bad[4] = 60
    assert g(*bad) == 2
    h = lib.tq_ternary_stochastic_flip
    st = ctypes.c_uint64(5)
    ok = [P(), P(1 << 20), 4, 64, 0.5, ctypes.byref(st), 0, None]
    bad = list(ok); bad[5] = None
    assert h(*bad) == 1
    for t in (float("nan"), -0.5, float("inf")):
        bad = list(ok); bad[4] = t
        assert h(*bad) == 4, t
    bad = list(ok); bad[1] = P(32)
    assert h(*bad) == 4                                   # grad overlaps packed
    bad = list(ok); bad[6] = tq.GAMMA_PER_ROW
    assert h(*bad) == 4
    assert st.value == 5                                  # a refused call leaves the state alone
    s = ctypes.c_uint64(0)
    lib.tq_seed(ctypes.byref(s), 0)
    assert s.value == 0x9E3779B97F4A7C15
    lib.tq_seed(ctypes.byref(s), 12345)
    assert s.value == 12345


def test_xorshift_jump_tables_are_generated_and_jump_the_oracle_stream():
    import importlib.util
    import oracle
    here = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "ternary_bit_linear_b200", "csrc")
    spec = importlib.util.spec_from_file_location("gen_xorshift_jump", os.path.join(here, "gen_xorshift_jump.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    assert open(os.path.join(here, "tq_xorshift_jump.h")).read() == gen.header()
    chunk, warp, lane = gen.tables()
    x = 0x0123456789ABCDEF
    seq, _ = oracle.xorshift64(x, gen.CHUNK)
    assert gen.apply(chunk[0], x) == seq[-1]
    assert gen.apply(warp[3], x) == seq[3 * gen.WARP_RUN - 1]
    for l in (1, 7, 31):
        assert gen.apply([lane[b][l] for b in range(64)], x) == seq[gen.RUN * l - 1]
    # two chunks = chunk[1]
    seq2, _ = oracle.xorshift64(seq[-1], gen.CHUNK)
    assert gen.apply(chunk[1], x) == seq2[-1]
