"""Integer and bit-level forms the kernels rely on, emulated on the CPU against
the oracle: the decision form of the stochastic-rounding epilogue, and the
code-to-float forms of the INT8 weight and INT4 projection conversions.

The a4+a5 kernel decides each weight without integer conversions: for
|X| < 2^22 the bits of fadd.rn(X, 1.5 * 2^23) are 0x4B400000 + rint(X) (the
sum lies in [2^23, 2^24), where the float32 step is 1, and 1.5 * 2^23 is even,
so ties go to the even integer as rint's do); adding (draw - 0x4B400000) and
q * 2^16 as 32-bit integers leaves rint(X) + draw + q * 2^16, whose upper 16
bits, read as a signed lane and clamped to [-127, 127], are the new code.  This
test carries out exactly those steps with numpy integers and a float32 sum
rounded to nearest (exact float64 sum, then the nearest float32, ties to even),
and requires the oracle's codes for the same q, X and draws.  An upward- or
downward-rounded sum fails it.  It checks the algebra the kernel relies on; the kernel itself is
checked against the oracle by the GPU parity tests.
"""
import numpy as np

import oracle as O

MAGIC = np.float64(1.5 * 2 ** 23)
MAGIC_BITS = np.uint32(0x4B400000)


def _fadd_rn_f32(x32, c):
    exact = x32.astype(np.float64) + c            # exact: both terms are float32 values
    return exact.astype(np.float32)               # nearest float32, ties to even


def _kernel_codes(q, X, d):
    tb = _fadd_rn_f32(X, MAGIC).view(np.uint32)
    dq = (d.astype(np.uint32) - MAGIC_BITS).astype(np.uint32)              # draw - 0x4B400000 (mod 2^32)
    q16 = (q.astype(np.int32) << 16).view(np.uint32)                        # q * 2^16, sign-extended
    s = (tb.astype(np.uint64) + dq + q16).astype(np.uint32)                  # mod 2^32
    hi = (s >> np.uint32(16)).astype(np.uint16).view(np.int16).astype(np.int32)
    return np.clip(hi, -127, 127)


def test_fast_decision_form_equals_the_oracle_rule():
    rng = np.random.default_rng(2024)
    n = 1 << 21
    q = rng.integers(-127, 128, n).astype(np.int8)
    scale = rng.choice([4.0, 300.0, 7.0e4, 4.19e6], n)
    X = (rng.uniform(-1, 1, n) * scale).astype(np.float32)
    X[:64] = np.float32(4194303.75)
    X[64:128] = -np.float32(4194303.75)
    X[128:192] = 0.0
    # ties: half-integers of both parities and signs
    X[256:512] = (rng.integers(-1000, 1000, 256) + 0.5).astype(np.float32)
    d = rng.integers(0, 1 << 16, n).astype(np.uint32)
    d[192:256] = 0xFFFF
    # the oracle's rule with alpha = 1, s = 2^16 (so c' = 1 and U = X), one row
    W = q.reshape(1, n)
    sW = np.full(-(-n // 256), 65536.0, np.float32)
    ref = O.stochastic_round_update(W, sW, X.reshape(1, n), O.Config(m=1, n=n, r=1, alpha=1.0), 1,
                                    u16=d.reshape(1, n))
    np.testing.assert_array_equal(_kernel_codes(q, X, d), ref.ravel().astype(np.int32))


# ---------------------------------------------------------------- code-to-float forms

def _bits_f32(u):
    return np.asarray(u, np.uint32).view(np.float32)


def test_int8_code_to_float_form_equals_the_oracle_dequant():
    # the fused INT8 forward converts a code without the conversion unit: the byte
    # q ^ 0x80 (= q + 128 as an unsigned byte) under the bits of 2^23 is the float
    # 2^23 + q + 128, exact; less 2^23 + 128 (one float32 subtraction, exact) it is q;
    # times the scale in float32, rounded to nearest, then to bf16 (nearest even).
    # Every code against the oracle's W~ = bf16(fp32(q) * s), over many scales.
    rng = np.random.default_rng(7)
    q = np.arange(-128, 128, dtype=np.int32)
    u = (q & 0xFF) ^ 0x80
    f = _bits_f32(np.uint32(0x4B000000) | u.astype(np.uint32))
    qf = (f.astype(np.float64) - np.float64(2 ** 23 + 128)).astype(np.float32)
    assert np.array_equal(qf, q.astype(np.float32))
    scales = np.concatenate([rng.uniform(1e-6, 1.0, 2000), 2.0 ** rng.integers(-30, 10, 64),
                             [np.float32(1.0), np.float32(4.7e-4)]]).astype(np.float32)
    for s in scales:
        prod = (qf.astype(np.float64) * np.float64(s)).astype(np.float32)   # float32 product, nearest
        got = O.bf16_round(prod)
        want = O.dequant_weight_bf16(q.astype(np.int8)[None, :], np.full(1, s, np.float32))[0]
        assert np.array_equal(got, want), float(s)


def test_int4_code_to_float_form_equals_the_oracle():
    # the INT4 projection unpack: nibble ^ 8 (= code + 8) under the bits of
    # 1.5 * 2^23 is the float 1.5 * 2^23 + code + 8, exact; less 1.5 * 2^23 + 8 it
    # is the code, for every nibble
    codes = np.arange(-8, 8, dtype=np.int32)
    v = ((codes & 0xF) ^ 8).astype(np.uint32)
    f = _bits_f32(np.uint32(0x4B400000) | v)
    back = (f.astype(np.float64) - np.float64(1.5 * 2 ** 23 + 8)).astype(np.float32)
    assert np.array_equal(back, codes.astype(np.float32))
    # the even and odd nibbles of a word, spread one to a byte, keep their order
    rng = np.random.default_rng(8)
    w = rng.integers(0, 2 ** 32, 4096, dtype=np.uint64).astype(np.uint32)
    fw = w ^ np.uint32(0x88888888)
    ev, od = fw & np.uint32(0x0F0F0F0F), (fw >> np.uint32(4)) & np.uint32(0x0F0F0F0F)
    for k in range(8):
        nib = (fw >> np.uint32(4 * k)) & np.uint32(0xF)
        src = ev if k % 2 == 0 else od
        assert np.array_equal((src >> np.uint32(8 * (k // 2))) & np.uint32(0xFF), nib)
