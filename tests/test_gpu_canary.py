"""No kernel writes outside its outputs: every output buffer of a call sits
between guard regions filled with a known byte pattern, on ragged shapes (token,
feature and contraction tails, per-row and per-tensor gamma, both small-M and
tcgen05 paths, the grouped call, the training kernels), and the guards must
be untouched afterwards.  The interiors must equal the same call made on plain
buffers."""
import numpy as np
import pytest

from ternary_bit_linear_b200 import synthetic as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


class Guarded:
    """A contiguous CUDA tensor of `shape` inside GUARD bytes of pattern on
    either side (the interior starts 16-byte aligned)."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.n = n
        self.raw = torch.full((2 * GUARD + n,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(shape)

    def intact(self):
        torch.cuda.synchronize()
        head = self.raw[:GUARD].cpu().numpy()
        tail = self.raw[GUARD + self.n:].cpu().numpy()
        return bool(np.all(head == PATTERN) and np.all(tail == PATTERN))


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("N,K,per_row", [(17, 192, True), (17, 192, False), (3, 8256, True), (5, 8256, False)])
def test_pack_canaries(cuda_lib, N, K, per_row):
    tq = cuda_lib
    W = dev(S.normal((N, K), 0.02, 150, N))
    fl = tq.GAMMA_PER_ROW if per_row else 0
    p, g = Guarded((N, K // 4), torch.uint8), Guarded((N if per_row else 1,), torch.float32)
    ws = torch.empty((max(16, tq.pack_workspace_bytes(N, K, fl)),), dtype=torch.uint8, device="cuda")
    tq.quantize_ternary_pack_(W, fl, p.t, g.t, ws)
    p_ref, g_ref = tq.quantize_ternary_pack(W, per_row=per_row)
    assert p.intact() and g.intact()
    assert torch.equal(p.t, p_ref) and torch.equal(g.t, g_ref)
    g2 = Guarded((1,), torch.float32)
    p2 = Guarded((N, K // 4), torch.uint8)
    tq.quantize_ternary_pack_abs_threshold_(W, 0, 0.01, p2.t, g2.t)
    assert p2.intact() and g2.intact()


@pytest.mark.parametrize("M,K", [(3, 320), (1, 64), (700, 448)])
def test_act_quant_canaries(cuda_lib, M, K):
    tq = cuda_lib
    X = dev(S.decode_acts(M, K, seed=151))
    xq, sx, rs = Guarded((M, K), torch.int8), Guarded((M,), torch.float32), Guarded((M,), torch.int32)
    tq.quantize_act_int8_(X, 0, 0.05, 40.0, xq.t, sx.t, rs.t)
    assert xq.intact() and sx.intact() and rs.intact()
    xr, sr, rr = tq.quantize_act_int8(X)
    assert torch.equal(xq.t, xr) and torch.equal(sx.t, sr) and torch.equal(rs.t, rr)


@pytest.mark.parametrize("M,N,K,ready", [(5, 33, 192, False), (5, 33, 192, True), (13, 17, 576, False),
                                         (130, 200, 320, False), (257, 129, 4160, False)])
def test_contraction_canaries(cuda_lib, M, N, K, ready):
    tq = cuda_lib
    W = dev(S.normal((N, K), 0.02, 152, N))
    X = dev(S.decode_acts(M, K, seed=153))
    packed, gamma = tq.quantize_ternary_pack(W, per_row=True)
    xq, sx, rs = tq.quantize_act_int8(X)
    fl = tq.GAMMA_PER_ROW | ((tq.FLAG_WEIGHTS_STATIC | tq.FLAG_INPUTS_READY) if ready else 0)
    y, acc = Guarded((M, N), torch.float32), Guarded((M, N), torch.int32)
    tq.ternary_gemm_(xq, sx, rs, packed, gamma, fl, y.t, acc.t)
    assert tq.device_status() == 0
    assert y.intact() and acc.intact()
    y_ref, acc_ref = tq.ternary_gemm(xq, sx, rs, packed, gamma, per_row=True, with_acc=True)
    assert torch.equal(acc.t, acc_ref) and torch.equal(y.t, y_ref)


@pytest.mark.parametrize("M,N,K", [(7, 45, 1024), (129, 70, 512)])
def test_fused_canaries(cuda_lib, M, N, K):
    tq = cuda_lib
    W = dev(S.normal((N, K), 0.02, 154, N))
    X = dev(S.student_t3((M, K), 155, M))
    packed, gamma = tq.quantize_ternary_pack(W, per_row=False)
    fl = tq.FLAG_FWHT | tq.FLAG_RMSNORM
    y, xq, sx = Guarded((M, N), torch.float32), Guarded((M, K), torch.int8), Guarded((M,), torch.float32)
    ws = torch.empty((tq.fused_workspace_bytes(M, K, fl),), dtype=torch.uint8, device="cuda")
    tq.bitlinear_fused_(X, packed, gamma, fl, y.t, ws, xq_out=xq.t, s_x_out=sx.t)
    assert y.intact() and xq.intact() and sx.intact()
    y_ref, xq_ref, sx_ref = tq.bitlinear_fused(X, packed, gamma, per_row=False, return_xq=True)
    assert torch.equal(y.t, y_ref) and torch.equal(xq.t, xq_ref) and torch.equal(sx.t, sx_ref)


@pytest.mark.parametrize("G,M,N,K", [(3, 5, 37, 192), (2, 12, 20, 4160)])
def test_grouped_canaries(cuda_lib, G, M, N, K):
    tq = cuda_lib
    packs = [tq.quantize_ternary_pack(dev(S.normal((N, K), 0.02, 156, g)), per_row=True) for g in range(G)]
    X = dev(np.stack([S.decode_acts(M, K, seed=157 + g) for g in range(G)]))
    fl = tq.GAMMA_PER_ROW
    y = Guarded((G, M, N), torch.float32)
    wsz = tq.grouped_workspace_bytes(G, M, K, fl)
    ws = Guarded((wsz,), torch.uint8)
    tq.bitlinear_grouped_(X, [p for p, _ in packs], [g for _, g in packs], fl, y.t, ws.t)
    assert tq.device_status() == 0
    assert y.intact() and ws.intact()
    for g in range(G):
        xq, sx, rs = tq.quantize_act_int8(X[g].contiguous())
        y_ref = tq.ternary_gemm(xq, sx, rs, packs[g][0], packs[g][1], per_row=True)
        assert torch.equal(y.t[g], y_ref), g


def test_training_and_fwht_canaries(cuda_lib):
    tq = cuda_lib
    M, N, K = 9, 33, 192
    W = dev(S.normal((N, K), 0.02, 158, 1))
    packed, gamma = tq.quantize_ternary_pack(W, per_row=False)
    dY = dev(S.normal((M, N), 1.0, 159, 1))
    dX = Guarded((M, K), torch.float32)
    ws = torch.empty((tq.backward_input_workspace_bytes(M, N),), dtype=torch.uint8, device="cuda")
    tq.ternary_backward_input_(dY, packed, gamma, 0, dX.t, ws)
    assert dX.intact()
    G = dev(S.normal((N, K), 1.0, 160, 1))
    out = Guarded((N, K), torch.float32)
    tq.ste_backward_(G, W, gamma, 0, out.t)
    assert out.intact()
    x = dev(S.student_t3((3, 1024), 161, 3))
    yf = Guarded((3, 1024), torch.float32)
    tq.fwht512_(x, yf.t)
    assert yf.intact()
    pk = Guarded((N, K // 4), torch.uint8)
    pk.t.copy_(packed)
    tq.ternary_stochastic_flip_(pk.t, G, 0.05, tq.seed(3))
    assert pk.intact()
    assert tq.device_status() == 0
