"""The integer decision form of the stochastic-rounding epilogue, emulated on
the CPU against the oracle's rounding rule.

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
