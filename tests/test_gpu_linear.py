"""GPU parity of the INT8-weight linear-layer products against the CPU oracle,
through the C ABI.

Bars:
  * W~ = bf16(fp32(q) * s): bit-exact (an integer code times a scale, one float32
    product, one rounding to bf16, the same on both sides).
  * Y = X W~^T, dX = D_y W~, G = D_y^T X: element-wise
    |gpu - exact| <= 2^-8 |exact| + K 2^-21 S, with S the sum of |a||b| over the
    K terms: the bf16 products are exact in float32, the float32 accumulation of
    K terms errs by at most about K 2^-23 S (2^-21 allows for an accumulator
    that is not round-to-nearest at every addition), and the final rounding to
    bf16 by at most 2^-9 of the value.
  * Integer inputs small enough for every partial sum and result to be exact in
    float32 and bf16: bit-exact (checks the operand layouts and transposes).
"""
import numpy as np
import pytest
import torch

import oracle as O
import quantized_rank_gradient_b200 as qg
from gpu_layer import stream

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda(cuda_ok):
    torch.cuda.synchronize()
    yield
    torch.cuda.synchronize()


def _bf16_dev(bits, ld=None):
    """Device bf16 matrix from uint16 bits, rows padded to `ld` elements."""
    r, c = bits.shape
    ld = ld or c
    buf = np.zeros((r, ld), np.uint16)
    buf[:, :c] = bits
    return torch.from_numpy(buf.view(np.int16)).cuda(), ld


def _empty_bf16(r, c, ld=None):
    ld = ld or c
    return torch.full((max(r, 1), ld), 0x7FC0, dtype=torch.int16, device="cuda"), ld  # NaN fill


def _read_bf16(t, r, c):
    return O.bf16_from_bits(t.cpu().numpy().view(np.uint16)[:r, :c])


def _within_bar(got, A, B, exact):
    """|got - exact| <= 2^-8 |exact| + K 2^-21 (|A| |B|), A (R x K), B (K x C)."""
    K = A.shape[1]
    S = np.abs(np.asarray(A, np.float64)) @ np.abs(np.asarray(B, np.float64))
    err = np.abs(got.astype(np.float64) - exact)
    tol = 2.0 ** -8 * np.abs(exact) + K * 2.0 ** -21 * S
    bad = err > tol
    assert not bad.any(), (int(bad.sum()), float((err - tol).max()))


def _weights(m, n, seed, ldw=None):
    rng = np.random.default_rng(seed)
    Wq = rng.integers(-127, 128, size=(m, n)).astype(np.int8)
    ng = -(-(m * n) // 256)
    sW = (rng.uniform(0.5, 1.5, size=ng) * 4.7e-3).astype(np.float32)
    ldw = ldw or -(-n // 16) * 16
    Wpad = np.zeros((m, ldw), np.int8)
    Wpad[:, :n] = Wq
    return Wq, sW, torch.from_numpy(Wpad).cuda(), ldw, torch.from_numpy(sW).cuda()


def _dequant_dev(dW, ldw, dsW, m, n, ldt=None):
    ldt = ldt or -(-n // 8) * 8
    Wt = torch.zeros((m, ldt), dtype=torch.int16, device="cuda")
    qg.check(qg.qg_linear_dequant_weight(dW.data_ptr(), ldw, dsW.data_ptr(), m, n, Wt.data_ptr(), ldt, stream()))
    return Wt, ldt


def _acts(r, c, seed):
    x = np.random.default_rng(seed).standard_normal((r, c)).astype(np.float32)
    return O.bf16_bits(x)


# ---------------------------------------------------------------- W~

@pytest.mark.parametrize("m,n", [(5, 300), (256, 256), (520, 200), (4096, 11008)])
def test_dequant_weight_bit_exact(m, n):
    Wq, sW, dW, ldw, dsW = _weights(m, n, seed=m + n, ldw=-(-n // 16) * 16 + 16)
    Wt, ldt = _dequant_dev(dW, ldw, dsW, m, n, ldt=-(-n // 8) * 8 + 8)
    got = Wt.cpu().numpy().view(np.uint16)[:, :n]
    np.testing.assert_array_equal(got, O.bf16_bits(O.dequant_weight_bf16(Wq, sW)))


# ---------------------------------------------------------------- the three products

SHAPES = [(300, 520, 200), (256, 256, 256), (37, 64, 72), (1000, 1376, 512)]


@pytest.mark.parametrize("T,m,n", SHAPES)
def test_forward_parity(T, m, n):
    Wq, sW, dW, ldw, dsW = _weights(m, n, seed=3 * T + m)
    Wt_dev, ldt = _dequant_dev(dW, ldw, dsW, m, n)
    Wt = O.dequant_weight_bf16(Wq, sW)
    Xb = _acts(T, n, seed=T)
    dX, ldx = _bf16_dev(Xb, ld=n + 8)
    Y, ldy = _empty_bf16(T, m, ld=m + 8)
    qg.check(qg.qg_linear_forward(dX.data_ptr(), ldx, Wt_dev.data_ptr(), ldt, T, m, n, Y.data_ptr(), ldy, stream()))
    X = O.bf16_from_bits(Xb)
    _within_bar(_read_bf16(Y, T, m), X, Wt.T, O.linear_forward(X, Wt))


@pytest.mark.parametrize("T,m,n", SHAPES)
def test_backward_data_parity(T, m, n):
    Wq, sW, dW, ldw, dsW = _weights(m, n, seed=5 * T + n)
    Wt_dev, ldt = _dequant_dev(dW, ldw, dsW, m, n)
    Wt = O.dequant_weight_bf16(Wq, sW)
    Db = _acts(T, m, seed=T + 1)
    dD, ldd = _bf16_dev(Db, ld=m + 16)
    dX, lddx = _empty_bf16(T, n)
    qg.check(qg.qg_linear_backward_data(dD.data_ptr(), ldd, Wt_dev.data_ptr(), ldt, T, m, n, dX.data_ptr(), lddx,
                                        stream()))
    D = O.bf16_from_bits(Db)
    _within_bar(_read_bf16(dX, T, n), D, Wt, O.linear_backward_data(D, Wt))


@pytest.mark.parametrize("T,m,n", SHAPES)
def test_backward_weight_parity(T, m, n):
    Db, Xb = _acts(T, m, seed=T + 2), _acts(T, n, seed=T + 3)
    dD, ldd = _bf16_dev(Db)
    dX, ldx = _bf16_dev(Xb, ld=n + 8)
    G, ldg = _empty_bf16(m, n, ld=n + 24)
    qg.check(qg.qg_linear_backward_weight(dD.data_ptr(), ldd, dX.data_ptr(), ldx, T, m, n, G.data_ptr(), ldg,
                                          stream()))
    D, X = O.bf16_from_bits(Db), O.bf16_from_bits(Xb)
    _within_bar(_read_bf16(G, m, n), D.T, X, O.linear_backward_weight(D, X))


def test_products_bit_exact_on_small_integers():
    # entries in {-1, 0, 1} and K <= 256: every partial sum and result is an
    # integer of magnitude <= 256, exact in float32 and in bf16
    rng = np.random.default_rng(21)
    T, m, n = 200, 248, 136
    Wq = rng.integers(-1, 2, size=(m, n)).astype(np.int8)
    sW = np.ones(-(-(m * n) // 256), np.float32)
    X = rng.integers(-1, 2, size=(T, n)).astype(np.float32)
    D = rng.integers(-1, 2, size=(T, m)).astype(np.float32)
    ldw = -(-n // 16) * 16
    Wpad = np.zeros((m, ldw), np.int8)
    Wpad[:, :n] = Wq
    dW, dsW = torch.from_numpy(Wpad).cuda(), torch.from_numpy(sW).cuda()
    Wt_dev, ldt = _dequant_dev(dW, ldw, dsW, m, n)
    dXa, ldx = _bf16_dev(O.bf16_bits(X))
    dDa, ldd = _bf16_dev(O.bf16_bits(D))
    Y, ldy = _empty_bf16(T, m)
    dX, lddx = _empty_bf16(T, n)
    G, ldg = _empty_bf16(m, n)
    s = stream()
    qg.check(qg.qg_linear_forward(dXa.data_ptr(), ldx, Wt_dev.data_ptr(), ldt, T, m, n, Y.data_ptr(), ldy, s))
    qg.check(qg.qg_linear_backward_data(dDa.data_ptr(), ldd, Wt_dev.data_ptr(), ldt, T, m, n, dX.data_ptr(), lddx, s))
    qg.check(qg.qg_linear_backward_weight(dDa.data_ptr(), ldd, dXa.data_ptr(), ldx, T, m, n, G.data_ptr(), ldg, s))
    Wi = Wq.astype(np.int64)
    np.testing.assert_array_equal(_read_bf16(Y, T, m), (X.astype(np.int64) @ Wi.T).astype(np.float32))
    np.testing.assert_array_equal(_read_bf16(dX, T, n), (D.astype(np.int64) @ Wi).astype(np.float32))
    np.testing.assert_array_equal(_read_bf16(G, m, n), (D.astype(np.int64).T @ X.astype(np.int64)).astype(np.float32))


def test_zero_tokens_gives_zero_gradient_and_no_output():
    m, n = 64, 128
    G, ldg = _empty_bf16(m, n)
    Y, ldy = _empty_bf16(4, m)
    X, ldx = _bf16_dev(np.zeros((4, n), np.uint16))
    D, ldd = _bf16_dev(np.zeros((4, m), np.uint16))
    Wt, ldt = _bf16_dev(np.zeros((m, n), np.uint16))
    s = stream()
    qg.check(qg.qg_linear_backward_weight(D.data_ptr(), ldd, X.data_ptr(), ldx, 0, m, n, G.data_ptr(), ldg, s))
    qg.check(qg.qg_linear_forward(X.data_ptr(), ldx, Wt.data_ptr(), ldt, 0, m, n, Y.data_ptr(), ldy, s))
    assert not G.cpu().numpy().view(np.uint16).any()
    assert (Y.cpu().numpy().view(np.uint16) == 0x7FC0).all()  # untouched


# ---------------------------------------------------------------- full LLaMA-7B sizes, sampled outputs

@pytest.mark.parametrize("m,n", [(4096, 11008), (11008, 4096)])
def test_full_size_sampled(m, n):
    # the bench's layer shapes at T = 8192 tokens; 64 outputs of each product
    # checked one by one against their exact dot products
    T = 8192
    Wq, sW, dW, ldw, dsW = _weights(m, n, seed=m)
    Wt_dev, ldt = _dequant_dev(dW, ldw, dsW, m, n)
    Xb, Db = _acts(T, n, seed=1), _acts(T, m, seed=2)
    dX_in, ldx = _bf16_dev(Xb)
    dD_in, ldd = _bf16_dev(Db)
    Y, ldy = _empty_bf16(T, m)
    dX, lddx = _empty_bf16(T, n)
    G, ldg = _empty_bf16(m, n)
    s = stream()
    qg.check(qg.qg_linear_forward(dX_in.data_ptr(), ldx, Wt_dev.data_ptr(), ldt, T, m, n, Y.data_ptr(), ldy, s))
    qg.check(qg.qg_linear_backward_data(dD_in.data_ptr(), ldd, Wt_dev.data_ptr(), ldt, T, m, n, dX.data_ptr(),
                                        lddx, s))
    qg.check(qg.qg_linear_backward_weight(dD_in.data_ptr(), ldd, dX_in.data_ptr(), ldx, T, m, n, G.data_ptr(), ldg,
                                          s))
    torch.cuda.synchronize()
    X, D = O.bf16_from_bits(Xb), O.bf16_from_bits(Db)
    Wt = O.dequant_weight_bf16(Wq, sW)
    rng = np.random.default_rng(9)
    Yh, dXh, Gh = (t.cpu().numpy().view(np.uint16) for t in (Y, dX, G))
    for _ in range(64):
        t, i, j = int(rng.integers(T)), int(rng.integers(m)), int(rng.integers(n))
        for got, a, b in ((Yh[t, i], X[t, :], Wt[i, :]), (dXh[t, j], D[t, :], Wt[:, j]), (Gh[i, j], D[:, i], X[:, j])):
            a64, b64 = a.astype(np.float64), b.astype(np.float64)
            exact = float(a64 @ b64)
            S = float(np.abs(a64) @ np.abs(b64))
            g = float(O.bf16_from_bits(np.array([got], np.uint16))[0])
            assert abs(g - exact) <= 2.0 ** -8 * abs(exact) + a.size * 2.0 ** -21 * S, (t, i, j, g, exact)


# ---------------------------------------------------------------- Y = X W~^T for a few tokens, INT8 W read once

def _weights_junk_pad(m, n, seed, ldw):
    """INT8 codes with random bytes in the row padding (columns n..ldw), which
    the fused forward must not let into Y."""
    Wq, sW, _, _, dsW = _weights(m, n, seed, ldw=ldw)
    Wpad = np.random.default_rng(seed + 1).integers(-128, 128, size=(m, ldw)).astype(np.int8)
    Wpad[:, :n] = Wq
    return Wq, sW, torch.from_numpy(Wpad).cuda(), dsW


def _forward_int8(dXa, ldx, dW, ldw, dsW, T, m, n, ld_extra=8):
    Y, ldy = _empty_bf16(T, m, ld=-(-m // 8) * 8 + ld_extra)
    qg.check(qg.qg_linear_forward_int8(dXa.data_ptr(), ldx, dW.data_ptr(), ldw, dsW.data_ptr(), T, m, n,
                                       Y.data_ptr(), ldy, stream()))
    return Y


# (m, n, ldw): ragged rows and columns, scale groups straddling 16-column
# chunks (n % 256 != 0), one column slice per row block (m large: each CTA
# streams many stages through its ring) and eight (m small: a cluster of 8)
FUSED_SHAPES = [(37, 64, 64), (300, 700, 720), (640, 1365, 1376), (129, 4096, 4096), (20000, 2600, 2608)]


@pytest.mark.parametrize("T", [1, 3, 8, 9, 16, 17, 32, 33, 64])
@pytest.mark.parametrize("m,n,ldw", FUSED_SHAPES)
def test_forward_int8_parity(T, m, n, ldw):
    Wq, sW, dW, dsW = _weights_junk_pad(m, n, seed=7 * T + m, ldw=ldw)
    Xb = _acts(T, n, seed=T + n)
    dXa, ldx = _bf16_dev(Xb, ld=-(-n // 8) * 8 + 8)
    Y = _forward_int8(dXa, ldx, dW, ldw, dsW, T, m, n)
    Wt = O.dequant_weight_bf16(Wq, sW)
    X = O.bf16_from_bits(Xb)
    _within_bar(_read_bf16(Y, T, m), X, Wt.T, O.linear_forward(X, Wt))
    # nothing written past T rows or m columns
    Yh = Y.cpu().numpy().view(np.uint16)
    assert (Yh[:T, m:] == 0x7FC0).all() and (Yh[T:] == 0x7FC0).all()


@pytest.mark.parametrize("m,n", [(4096, 11008), (11008, 4096)])
@pytest.mark.parametrize("T", [1, 16, 64])
def test_forward_int8_full_size(T, m, n):
    # the 7B stack's MLP shapes at decode sizes, every output against the oracle
    Wq, sW, dW, ldw, dsW = _weights(m, n, seed=m + T)
    Xb = _acts(T, n, seed=T)
    dXa, ldx = _bf16_dev(Xb)
    Y = _forward_int8(dXa, ldx, dW, ldw, dsW, T, m, n, ld_extra=0)
    Wt = O.dequant_weight_bf16(Wq, sW)
    X = O.bf16_from_bits(Xb)
    _within_bar(_read_bf16(Y, T, m), X, Wt.T, O.linear_forward(X, Wt))


@pytest.mark.parametrize("T", [16, 64])
def test_forward_int8_bit_exact_on_small_integers(T):
    # codes in {-1, 0, 1} (one in 32 nonzero), power-of-two scales and X in
    # {-1, 0, 1}: every partial sum, the sum over the cluster's slices and the
    # result are integers times 2^-3 of magnitude < 256 * 2^-3, exact in
    # float32 and in bf16, so the split-K reduction and the operand layouts are
    # checked bit for bit
    rng = np.random.default_rng(33 + T)
    m, n = 300, 4000
    Wq = (rng.integers(-1, 2, size=(m, n)) * (rng.integers(0, 32, size=(m, n)) == 0)).astype(np.int8)
    sW = np.full(-(-(m * n) // 256), 0.125, np.float32)
    X = rng.integers(-1, 2, size=(T, n)).astype(np.float32)
    exact = X.astype(np.int64) @ Wq.astype(np.int64).T
    assert np.abs(exact).max() < 256
    ldw = -(-n // 16) * 16
    Wpad = np.zeros((m, ldw), np.int8)
    Wpad[:, :n] = Wq
    dW, dsW = torch.from_numpy(Wpad).cuda(), torch.from_numpy(sW).cuda()
    dXa, ldx = _bf16_dev(O.bf16_bits(X))
    Y = _forward_int8(dXa, ldx, dW, ldw, dsW, T, m, n)
    np.testing.assert_array_equal(_read_bf16(Y, T, m), (exact * 0.125).astype(np.float32))


def test_forward_int8_deterministic_and_agrees_with_two_step_path():
    # the same bits on every call (the slices' partial sums are added in a
    # fixed order); the dequantize-then-GEMM path meets the same bar on the
    # same inputs
    T, m, n = 8, 4096, 4096
    Wq, sW, dW, ldw, dsW = _weights(m, n, seed=5)
    Xb = _acts(T, n, seed=6)
    dXa, ldx = _bf16_dev(Xb)
    Y1 = _forward_int8(dXa, ldx, dW, ldw, dsW, T, m, n)
    Y2 = _forward_int8(dXa, ldx, dW, ldw, dsW, T, m, n)
    assert torch.equal(Y1, Y2)
    Wt_dev, ldt = _dequant_dev(dW, ldw, dsW, m, n)
    Y3, ldy = _empty_bf16(T, m)
    qg.check(qg.qg_linear_forward(dXa.data_ptr(), ldx, Wt_dev.data_ptr(), ldt, T, m, n, Y3.data_ptr(), ldy, stream()))
    X, Wt = O.bf16_from_bits(Xb), O.dequant_weight_bf16(Wq, sW)
    exact = O.linear_forward(X, Wt)
    for Y in (Y1, Y3):
        _within_bar(_read_bf16(Y, T, m), X, Wt.T, exact)


def test_forward_int8_edges():
    m, n = 64, 128
    Wq, sW, dW, ldw, dsW = _weights(m, n, seed=1)
    X, ldx = _bf16_dev(np.zeros((65, n), np.uint16))
    Y, ldy = _empty_bf16(65, m)
    s = stream()
    # T = 0: nothing written
    qg.check(qg.qg_linear_forward_int8(X.data_ptr(), ldx, dW.data_ptr(), ldw, dsW.data_ptr(), 0, m, n, Y.data_ptr(),
                                       ldy, s))
    torch.cuda.synchronize()
    assert (Y.cpu().numpy().view(np.uint16) == 0x7FC0).all()
    # more than 64 tokens, a weight stride that is not a multiple of 16, a
    # misaligned X: refused before any launch
    assert qg.qg_linear_forward_int8(X.data_ptr(), ldx, dW.data_ptr(), ldw, dsW.data_ptr(), 65, m, n,
                                     Y.data_ptr(), ldy, s) == qg.QG_ESHAPE
    assert qg.qg_linear_forward_int8(X.data_ptr(), ldx, dW.data_ptr(), 136, dsW.data_ptr(), 4, m, n,
                                     Y.data_ptr(), ldy, s) == qg.QG_ESHAPE
    assert qg.qg_linear_forward_int8(X.data_ptr() + 2, ldx, dW.data_ptr(), ldw, dsW.data_ptr(), 4, m, n,
                                     Y.data_ptr(), ldy, s) == qg.QG_EALIGN
    # zero activations give zero outputs
    qg.check(qg.qg_linear_forward_int8(X.data_ptr(), ldx, dW.data_ptr(), ldw, dsW.data_ptr(), 64, m, n,
                                       Y.data_ptr(), ldy, s))
    torch.cuda.synchronize()
    assert (_read_bf16(Y, 64, m) == 0).all()
