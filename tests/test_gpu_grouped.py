"""GPU parity of tq_bitlinear_grouped (G same-shape layers in one activation
pass and one persistent GEMV launch) against the CPU oracle, layer by layer:
x_q, s_x and rowsum bit-exact (read back from the workspace, whose layout the
header states), y within 1e-5 of the oracle's correctly rounded rescale of
the exact int32 accumulator.  Each layer's oracle result is
act_quant -> matmul_addsub -> dequant on that layer's own inputs."""
import numpy as np
import pytest

import oracle
from ternary_bit_linear_b200 import synthetic as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

REL = 1e-5


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run_grouped(tq, X, packs, flags):
    """X: [G, M, K] (or [M, K] shared); packs: list of (packed, gamma) numpy."""
    G = len(packs)
    M, K = X.shape[-2], X.shape[-1]
    N = packs[0][0].shape[0]
    pd = [dev(p) for p, _ in packs]
    gd = [dev(g) for _, g in packs]
    y = torch.full((G, M, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros((tq.grouped_workspace_bytes(G, M, K, flags),), dtype=torch.uint8, device="cuda")
    tq.bitlinear_grouped_(dev(X), pd, gd, flags, y, ws)
    torch.cuda.synchronize()
    mid = tq.grouped_intermediates(ws, G, M, K, flags)
    return y.cpu().numpy(), {k: v.cpu().numpy() for k, v in mid.items()}


def check(tq, X, packs, per_row, flags, enc=0):
    G = len(packs)
    y, mid = run_grouped(tq, X, packs, flags)
    shared = bool(flags & tq.FLAG_SHARED_INPUT)
    for g in range(G):
        Xg = X if shared else X[g]
        xq_ref, sx_ref, rs_ref = oracle.act_quant(Xg)
        gx = 0 if shared else g
        assert np.array_equal(mid["xq"][gx], xq_ref), g
        assert np.array_equal(mid["s_x"][gx], sx_ref) and np.array_equal(mid["rowsum"][gx], rs_ref), g
        acc = oracle.matmul_addsub_format(xq_ref, packs[g][0], enc)
        y_ref = oracle.dequant(acc, packs[g][1], sx_ref, per_row).astype(np.float64)
        yg = y[g].astype(np.float64)
        zero = y_ref == 0
        assert np.all(yg[zero] == 0), g
        rel = np.abs(yg[~zero] - y_ref[~zero]) / np.abs(y_ref[~zero])
        assert rel.size == 0 or rel.max() <= REL, (g, rel.max())


def make_packs(G, N, K, per_row, seed, enc=0):
    return [oracle.quantize_pack(S.normal((N, K), 0.02, seed, 1000 * g + N), per_row=per_row, encoding=enc)
            for g in range(G)]


@pytest.mark.parametrize("G,M,N,K", [(1, 1, 64, 64), (3, 5, 100, 512), (8, 8, 4096, 4096), (2, 16, 129, 1024),
                                     (5, 3, 1000, 2048), (4, 1, 300, 8192), (64, 2, 48, 256), (2, 9, 4097, 4096)])
@pytest.mark.parametrize("per_row", [True, False])
def test_grouped_matches_oracle(cuda_lib, G, M, N, K, per_row):
    tq = cuda_lib
    packs = make_packs(G, N, K, per_row, 200)
    X = np.stack([S.decode_acts(M, K, seed=g) for g in range(G)])
    fl = (tq.GAMMA_PER_ROW if per_row else 0)
    check(tq, X, packs, per_row, fl)
    check(tq, X, packs, per_row, fl | tq.FLAG_WEIGHTS_STATIC | tq.FLAG_INPUTS_READY)
    assert tq.device_status() == 0


@pytest.mark.parametrize("G,M,N,K", [(3, 4, 512, 4096), (6, 16, 200, 2048)])
def test_grouped_shared_input(cuda_lib, G, M, N, K):
    tq = cuda_lib
    packs = make_packs(G, N, K, True, 201)
    X = S.decode_acts(M, K, seed=7)
    check(tq, X, packs, True, tq.GAMMA_PER_ROW | tq.FLAG_SHARED_INPUT)
    assert tq.device_status() == 0


@pytest.mark.parametrize("enc", [1, 2])
def test_grouped_layouts(cuda_lib, enc):
    tq = cuda_lib
    G, M, N, K = 4, 6, 300, 1024
    packs = make_packs(G, N, K, True, 202, enc)
    X = np.stack([S.decode_acts(M, K, seed=10 + g) for g in range(G)])
    check(tq, X, packs, True, tq.GAMMA_PER_ROW | (enc << 7), enc)
    assert tq.device_status() == 0


def test_grouped_one_x_buffer_plan(cuda_lib):
    """M = 16 at K = 8192: the x_q of one problem is 128 KiB, so the plan
    keeps a single x buffer and every problem switch waits for all warps."""
    tq = cuda_lib
    G, M, N, K = 3, 16, 2400, 8192
    packs = make_packs(G, N, K, False, 203)
    X = np.stack([S.decode_acts(M, K, seed=20 + g) for g in range(G)])
    check(tq, X, packs, False, tq.FLAG_WEIGHTS_STATIC)
    assert tq.device_status() == 0


def test_grouped_full_size_decode(cuda_lib):
    """The decode configuration, 8 layers of 4096 x 4096 per call, M = 1 and 8,
    checked on every output against the oracle."""
    tq = cuda_lib
    N = K = 4096
    W = S.decode_weights(N, K, seed=0)
    p, g = oracle.quantize_pack(W, per_row=True)
    packs = [(p, g)] * 8
    for M in (1, 8):
        X = np.stack([S.decode_acts(M, K, seed=s) for s in range(8)])
        check(tq, X, packs, True, tq.GAMMA_PER_ROW | tq.FLAG_WEIGHTS_STATIC | tq.FLAG_INPUTS_READY)
    assert tq.device_status() == 0


def test_grouped_repeat_bit_identical(cuda_lib):
    """Repeated calls give identical bits (no race between the ring's slots,
    the x buffers and the partial-sum buffers)."""
    tq = cuda_lib
    G, M, N, K = 16, 8, 2048, 4096
    packs = make_packs(G, N, K, True, 204)
    X = np.stack([S.decode_acts(M, K, seed=30 + g) for g in range(G)])
    fl = tq.GAMMA_PER_ROW | tq.FLAG_WEIGHTS_STATIC | tq.FLAG_INPUTS_READY
    first, _ = run_grouped(tq, X, packs, fl)
    for _ in range(6):
        again, _ = run_grouped(tq, X, packs, fl)
        assert np.array_equal(first.view(np.uint32), again.view(np.uint32))
    assert tq.device_status() == 0
