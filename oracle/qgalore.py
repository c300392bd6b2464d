"""Plain CPU oracle for the Q-GaLore per-layer optimizer step and subspace refresh.

TEST INFRASTRUCTURE ONLY.  This module is imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the ``cpu_baseline`` / reference arm of
``bench.py``; nothing in the product path may import it.  It shares no code with
the CUDA path: every formula here is written out independently.

What the pages fix, and where (titles of the source pages):

* [QG-abs]  "Q-GaLore: Quantized GaLore with INT4 Projection and Layer-Adaptive
  Low-Rank Gradients", abstract (paper index record): gradients are projected into
  a low-rank subspace found by SVD; projection matrices kept in INT4, weights in
  INT8, stochastic rounding accumulates small updates.
* [QG-sched] AIMech curated page "Q-GaLore (Quantized GaLore with INT4 Projection
  and Layer-Adaptive Low-Rank Gradients)", mechanism "layer-adaptive subspace
  cosine schedule" (paper section 3.1, Eq. (5)):
  CosSim(P_t, P_{t-D}) = (1/r) * sum_i sigma_i(P_t^T P_{t-D}); the layer's
  interval D doubles whenever CosSim > gamma, gamma = 0.4 by default.
* [QG-quant] same page, mechanism "INT4 projection and INT8 stochastic rounding"
  (paper section 3.2): P_t stored in INT4; low-rank first and second moments
  (M^Q, V^Q) in INT8; W^Q_t = W^Q_{t-1} + xi(alpha * P^Q_t * G~_t) with xi an
  unbiased stochastic rounding.

Everything the pages leave open is a stated reading (they are listed, numbered,
in the design notes of this repository); each function below names the reading
it takes.  Floating point: contractions (the two projections, the refresh
products) are carried out in float64 from the exact float32/bf16 operands and
rounded once to float32; element-wise arithmetic that decides an integer (a
quantised code, a rounding decision) is done in IEEE float32, one rounding per
operation, in the order written, exactly as the GPU path must do it.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

F32 = np.float32
U32_MASK = np.uint64(0xFFFFFFFF)

# --------------------------------------------------------------------------
# bf16 rounding (round to nearest, ties to even) — the operand precision of the
# projections.  Pinned against torch's float32 -> bfloat16 conversion.
# --------------------------------------------------------------------------


def bf16_bits(x) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round-to-nearest-even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = ((b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r = np.where(nan, np.uint16(0x7FC0), r)
    return r


def bf16_from_bits(bits) -> np.ndarray:
    """bfloat16 bit patterns -> float32 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def bf16_round(x) -> np.ndarray:
    """float32 -> float32 values representable in bfloat16 (RNE)."""
    return bf16_from_bits(bf16_bits(x))


# --------------------------------------------------------------------------
# Philox counter-based generator (Salmon, Moraes, Dror, Shaw, "Parallel random
# numbers: as easy as 1, 2, 3", SC'11).  The pages only say the rounding is
# stochastic and unbiased; the random stream is a reading (counter-based so
# that any element's draw is computable on its own).
# --------------------------------------------------------------------------

PHILOX4x32 = dict(width=32, mult=(0xD2511F53, 0xCD9E8D57), weyl=(0x9E3779B9, 0xBB67AE85))
PHILOX4x64 = dict(width=64, mult=(0xD2E7470EE14C6C93, 0xCA5A826395121157),
                  weyl=(0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B))


def philox_generic(ctr, key, width, mult, weyl, rounds=10):
    """Philox-4xW on Python integers (slow, any word width).

    One round: the two products mult0*c0 and mult1*c2 are formed at double
    width; the new block is (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0).  The key is
    bumped by the Weyl constants before every round but the first.
    """
    mask = (1 << width) - 1
    c = [int(v) & mask for v in ctr]
    k = [int(v) & mask for v in key]
    for rnd in range(rounds):
        if rnd:
            k = [(k[0] + weyl[0]) & mask, (k[1] + weyl[1]) & mask]
        p0 = mult[0] * c[0]
        p1 = mult[1] * c[2]
        c = [((p1 >> width) ^ c[1] ^ k[0]) & mask, p1 & mask,
             ((p0 >> width) ^ c[3] ^ k[1]) & mask, p0 & mask]
    return c


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox-4x32-10: arrays of counters -> four uint32 arrays."""
    c = np.broadcast_arrays(*(np.asarray(v, dtype=np.uint64) & U32_MASK for v in (c0, c1, c2, c3)))
    c = [np.array(v, dtype=np.uint64) for v in c]
    k0 = np.uint64(int(k0) & 0xFFFFFFFF)
    k1 = np.uint64(int(k1) & 0xFFFFFFFF)
    m0, m1 = (np.uint64(v) for v in PHILOX4x32["mult"])
    w0, w1 = (np.uint64(v) for v in PHILOX4x32["weyl"])
    s32 = np.uint64(32)
    for rnd in range(10):
        if rnd:
            k0 = (k0 + w0) & U32_MASK
            k1 = (k1 + w1) & U32_MASK
        p0 = m0 * c[0]
        p1 = m1 * c[2]
        c = [(p1 >> s32) ^ c[1] ^ k0, p1 & U32_MASK, (p0 >> s32) ^ c[3] ^ k1, p0 & U32_MASK]
    return [v.astype(np.uint32) for v in c]


# --------------------------------------------------------------------------
# Quantizers.  [QG-quant] fixes the widths (INT4 projection, INT8 moments and
# weights); the grids are readings: symmetric absmax; the stored scale is
# absmax / qmax and the codes are clamp(rint(x * (qmax / absmax))) with ties to
# even -- the inverse scale is formed once per group (IEEE float32 division)
# and applied by one multiplication per element; a group whose absmax is below
# 2^-120 (zero, subnormal or so small that qmax / absmax would overflow) gets
# scale 0 and codes 0.
# --------------------------------------------------------------------------

INT4_QMAX = 7
INT8_QMAX = 127
ABSMAX_FLOOR = F32(2.0 ** -120)


def _absmax_grid(absmax, qmax):
    """(scale, inverse scale, live) per group; zero for a group below the floor."""
    absmax = np.asarray(absmax, np.float32)
    live = absmax >= ABSMAX_FLOOR
    s = np.where(live, absmax / F32(qmax), F32(0)).astype(np.float32)
    inv = np.where(live, F32(qmax) / np.where(live, absmax, F32(1)), F32(0)).astype(np.float32)
    return s, inv, live


def quant_int4_groups(P, group=64):
    """INT4 absmax quantization of the flattened row-major array, groups of `group`.

    Returns (codes int8 in [-7, 7] of length P.size, scales float32 of length
    ceil(P.size / group)).  [QG-quant]: P_t is kept in INT4.
    """
    x = np.asarray(P, dtype=np.float32).ravel()
    ng = -(-x.size // group)
    xp = np.zeros(ng * group, dtype=np.float32)
    xp[: x.size] = x
    xg = xp.reshape(ng, group)
    s, inv, live = _absmax_grid(np.max(np.abs(xg), axis=1), INT4_QMAX)
    q = np.clip(np.rint((xg * inv[:, None]).astype(np.float32)), -INT4_QMAX, INT4_QMAX)
    q = np.where(live[:, None], q, 0).astype(np.int8)
    return q.ravel()[: x.size], s


def pack_int4(codes) -> np.ndarray:
    """Two's-complement nibbles, two per byte, the even index in the low nibble."""
    q = np.asarray(codes, dtype=np.int8).ravel()
    if q.size % 2:
        q = np.concatenate([q, np.zeros(1, np.int8)])
    lo = q[0::2].astype(np.uint8) & np.uint8(0xF)
    hi = q[1::2].astype(np.uint8) & np.uint8(0xF)
    return (lo | (hi << np.uint8(4))).astype(np.uint8)


def unpack_int4(packed, count) -> np.ndarray:
    b = np.asarray(packed, dtype=np.uint8)
    nib = np.empty(b.size * 2, dtype=np.int16)
    nib[0::2] = b & 0xF
    nib[1::2] = b >> 4
    nib = np.where(nib >= 8, nib - 16, nib)
    return nib[:count].astype(np.int8)


def dequant_int4_f32(packed, scales, m, r, group=64) -> np.ndarray:
    """P = code * scale in float32 (one rounding), shape (m, r)."""
    q = unpack_int4(packed, m * r).astype(np.float32)
    s = np.asarray(scales, dtype=np.float32)[np.arange(m * r) // group]
    return (q * s).astype(np.float32).reshape(m, r)


def dequant_P_bf16(packed, scales, m, r, group=64) -> np.ndarray:
    """Step a1: P~ = bf16_rn(code * scale): the projection as the tensor cores see it."""
    return bf16_round(dequant_int4_f32(packed, scales, m, r, group))


def quant_rowblock_int8(x, block=256, unsigned=False):
    """INT8 absmax quantization in blocks of `block` consecutive columns of each row.

    The last block of a row is short when n % block != 0 (blocks never cross
    rows).  unsigned=True is used for the second moment (v >= 0): codes in
    [0, 127].  Returns (codes int8 (rows, n), scales float32 (rows, nblocks)).
    """
    x = np.asarray(x, dtype=np.float32)
    rows, n = x.shape
    nb = -(-n // block)
    codes = np.zeros((rows, n), dtype=np.int8)
    scales = np.zeros((rows, nb), dtype=np.float32)
    lo = 0 if unsigned else -INT8_QMAX
    for b in range(nb):
        xs = x[:, b * block: min((b + 1) * block, n)]
        s, inv, live = _absmax_grid(np.max(np.abs(xs), axis=1), INT8_QMAX)
        q = np.clip(np.rint((xs * inv[:, None]).astype(np.float32)), lo, INT8_QMAX)
        codes[:, b * block: min((b + 1) * block, n)] = np.where(live[:, None], q, 0)
        scales[:, b] = s
    return codes, scales


def dequant_rowblock(codes, scales, block=256) -> np.ndarray:
    codes = np.asarray(codes)
    cols = np.arange(codes.shape[1]) // block
    return (codes.astype(np.float32) * np.asarray(scales, np.float32)[:, cols]).astype(np.float32)


# --------------------------------------------------------------------------
# Configuration and host-side constants
# --------------------------------------------------------------------------


@dataclass
class Config:
    m: int
    n: int
    r: int
    w_group: int = 256
    p_group: int = 64
    mom_block: int = 256
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    lr: float = 1e-3
    alpha: float = 0.25
    gamma: float = 0.4
    delta0: int = 200
    oversample: int = 16
    power_iters: int = 2
    seed: int = 0
    layer_id: int = 0
    mom_refresh: int = 0  # moments at a refresh: 0 keep, 1 reset, 2 rotate (see refresh_moments)
    proj_side: int = 0    # 0: P m x r, R = P^T G (the default reading); 1: P n x r, R = G P
    w_rescale: int = 0    # 0: updates saturate at +-127 (default); 1: a group that would leave the grid is re-scaled

    def f32(self, name):
        return F32(getattr(self, name))


def proj_dims(cfg: Config):
    """(rows of P, rows of R, columns of R): (m, r, n) for the left projection,
    (n, m, r) for the right one.  The moments have R's shape."""
    if cfg.proj_side == 0:
        return cfg.m, cfg.r, cfg.n
    if cfg.proj_side == 1:
        return cfg.n, cfg.m, cfg.r
    raise ValueError("proj_side must be 0 or 1")


def adam_constants(cfg: Config, t: int):
    """float32 constants of step t (t counted from 1 per layer), each formed in
    float64 from the float32 hyper-parameters and rounded once to float32:
    (1 - b1), (1 - b2), c1 = -lr / (1 - b1^t), c2 = 1 / sqrt(1 - b2^t)."""
    b1 = float(F32(cfg.beta1))
    b2 = float(F32(cfg.beta2))
    lr = float(F32(cfg.lr))
    return (F32(1.0 - b1), F32(1.0 - b2), F32(-lr / (1.0 - b1 ** t)), F32(1.0 / np.sqrt(1.0 - b2 ** t)))


# --------------------------------------------------------------------------
# The step, a1..a5
# --------------------------------------------------------------------------


def project(P_bf16, G) -> np.ndarray:
    """Step a2: R = P~^T G (r x n), float64 sum of the exact products, rounded to
    float32.  [QG-abs]: the gradient is projected into the low-rank subspace;
    reading: the left factor is projected (P is m x r) unless the right-side
    variant is asked for (project_right)."""
    return (np.asarray(P_bf16, np.float64).T @ np.asarray(G, np.float64)).astype(np.float32)


def project_right(G, P_bf16) -> np.ndarray:
    """Step a2 of the right-side variant: R = G P~ (m x r) for P n x r, float64
    sum of the exact products, rounded to float32."""
    return (np.asarray(G, np.float64) @ np.asarray(P_bf16, np.float64)).astype(np.float32)


def backproject_right(N_bf16, P_bf16) -> np.ndarray:
    """Step a4 of the right-side variant: U = N P~^T (m x n) for N m x r and
    P n x r, in float64 from the exact bf16 operands, rounded to float32."""
    return (np.asarray(N_bf16, np.float64) @ np.asarray(P_bf16, np.float64).T).astype(np.float32)


def adam_moments(R, m0, v0, cfg: Config, t: int):
    """Adam moment update and normalised low-rank step (float32, no fused
    multiply-add).  Readings: bias correction on, epsilon added after the square
    root, no weight decay, the descent sign carried by N:

        m = b1*m0 + (1-b1)*R
        v = b2*v0 + (1-b2)*(R*R)
        N = -lr * m_hat / (sqrt(v_hat) + eps),  m_hat = m/(1-b1^t), v_hat = v/(1-b2^t)

    evaluated as N = (m * c1) / (sqrt(v) * c2 + eps) with the per-step scalars
    c1 = -lr/(1-b1^t) and c2 = 1/sqrt(1-b2^t) (the same quantity; one float32
    rounding per operation, in this order).

    Returns (N float32 before bf16 rounding, m, v).
    """
    om1, om2, c1, c2 = adam_constants(cfg, t)
    R = np.asarray(R, np.float32)
    m = (cfg.f32("beta1") * m0 + om1 * R).astype(np.float32)
    v = (cfg.f32("beta2") * v0 + om2 * (R * R)).astype(np.float32)
    num = (m * c1).astype(np.float32)
    den = ((np.sqrt(v) * c2).astype(np.float32) + cfg.f32("eps")).astype(np.float32)
    return (num / den).astype(np.float32), m, v


def dequant_second_moment(Vq, sV, block=256) -> np.ndarray:
    """v = (code * scale)^2 in float32: V^Q holds the INT8 grid of sqrt(v)."""
    d = dequant_rowblock(Vq, sV, block)
    return (d * d).astype(np.float32)


def lowrank_adam_int8(R, Mq, sM, Vq, sV, cfg: Config, t: int):
    """Step a3: Adam on the INT8 moments.  [QG-quant]: (M^Q, V^Q) are kept in
    INT8.  Readings: per-row blocks of `mom_block` columns, re-quantized with a
    fresh absmax scale every step; the first moment m on a linear grid; the
    second moment through its square root (codes 0..127 of sqrt(v), so that
    v = (code * scale)^2) -- a linear grid on v itself sends the small second
    moments of a block to zero and lets m / sqrt(v) explode; N is formed from
    the float32 moments before they are re-quantized, then rounded to bf16 (the
    operand of step a4).

    Returns (N as bf16 values in float32, Mq', sM', Vq', sV')."""
    m0 = dequant_rowblock(Mq, sM, cfg.mom_block)
    v0 = dequant_second_moment(Vq, sV, cfg.mom_block)
    upd, m, v = adam_moments(R, m0, v0, cfg, t)
    N = bf16_round(upd)
    Mq2, sM2 = quant_rowblock_int8(m, cfg.mom_block, unsigned=False)
    Vq2, sV2 = quant_rowblock_int8(np.sqrt(v).astype(np.float32), cfg.mom_block, unsigned=True)
    return N, Mq2, sM2, Vq2, sV2


def backproject(P_bf16, N_bf16) -> np.ndarray:
    """Step a4: U = P~ N (m x n) in float64 from the exact bf16 operands, rounded
    to float32.  alpha is applied in step a5.  [QG-quant]: alpha * P_t * G~_t."""
    return (np.asarray(P_bf16, np.float64) @ np.asarray(N_bf16, np.float64)).astype(np.float32)


def sr_uniform16(m, n, seed, t, layer_id):
    """The 16-bit uniform draw of every weight element (m x n uint32 in [0, 2^16)).

    Element (i, j) takes the 16-bit half (j mod 2) -- the low half first -- of word
    ((j / 2) mod 4) of Philox-4x32-10(counter = (j / 8, i, t, layer_id), key =
    (seed low 32 bits, seed high 32 bits)): one Philox call serves eight
    consecutive elements of a row, and every row starts a call.
    """
    calls = -(-n // 8)
    row = np.repeat(np.arange(m, dtype=np.uint64), calls)          # call (i, c) for c = j / 8
    call = np.tile(np.arange(calls, dtype=np.uint64), m)
    w = philox4x32_10(call, row, t, layer_id, seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    words = np.stack(w, axis=1).reshape(m, calls, 4)                 # [i, c, k]: word k of call (i, c)
    halves = np.stack([words & np.uint32(0xFFFF), words >> np.uint32(16)], axis=3)  # [i, c, k, h]
    # element j = 8 c + 2 k + h: word k = (j / 2) mod 4, half h = j mod 2
    return halves.reshape(m, calls * 8)[:, :n].astype(np.uint32)


def stochastic_round_update(Wq, sW, U, cfg: Config, t: int, u16=None):
    """Step a5: W^Q <- W^Q + xi(alpha * U), in code units of the fixed weight grid.

    [QG-quant] asks only that xi be an unbiased stochastic rounding; the form is
    a reading.  The weight scale is one float32 per 256 consecutive elements of
    the row-major m x n array (logical index), fixed after initialisation (the
    re-scaling variant, stochastic_round_rescale, lets it grow instead).  The
    update is carried in fixed point with 16 fraction bits:
      c'_g = (alpha / s_g) * 2^16   (IEEE float32 division, exact scaling; a zero
                                     scale gives c'_g = 0 and freezes its group)
      X    = U * c'_g               (float32: the update in units of 2^-16 code)
      K    = rint(X)                (nearest integer, ties to even)
      r    = floor((K + d) / 2^16)  (d = the element's 16-bit uniform draw)
      W'   = clamp(W + r, -127, 127);  a NaN X keeps the old code.
    Adding a uniform 16-bit integer and dropping the 16 fraction bits rounds
    K / 2^16 up with probability equal to its fractional part, so
    E[r] = K / 2^16 exactly (Hermite's identity: the sum of floor((K + d) / 2^16)
    over all 2^16 draws is K).  K / 2^16 is X / 2^16 rounded to the nearest
    point of the 2^-16 draw grid, so it is within 2^-17 code of the update, and
    rint(-X) = -rint(X) makes that residue odd in X: an update and its negation
    move the weight by exactly opposite amounts on average, so no sign of update
    drifts.  |X| is clipped to 2^30 before the rounding, which changes no clamped
    result (|r| >= 2^14 saturates either way)."""
    m, n = Wq.shape
    e = np.arange(m * n, dtype=np.int64).reshape(m, n)
    sW = np.asarray(sW, np.float32)
    c = np.where(sW > 0, F32(cfg.alpha) / np.where(sW > 0, sW, F32(1)), F32(0)).astype(np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        cp = (c * F32(65536.0)).astype(np.float32)
        X = (np.asarray(U, np.float32) * cp[e // cfg.w_group]).astype(np.float32)
        nan = np.isnan(X)
        K = np.rint(np.clip(np.where(nan, F32(0), X), F32(-2.0 ** 30), F32(2.0 ** 30))).astype(np.int64)
    if u16 is None:
        u16 = sr_uniform16(m, n, cfg.seed, t, cfg.layer_id)
    r = (K + np.asarray(u16, np.int64)) >> 16          # floor division by 2^16
    out = np.clip(Wq.astype(np.int64) + r, -INT8_QMAX, INT8_QMAX)
    return np.where(nan, Wq, out).astype(np.int8)


W_RESCALE_LIMIT = INT8_QMAX * 65536  # 127 in units of 2^-16 code


def stochastic_round_rescale(Wq, sW, U, cfg: Config, t: int, u16=None):
    """Step a5 of the re-scaling variant: a weight group whose updated values
    would leave the INT8 grid gets a larger scale instead of saturating.

    [QG-quant] keeps W in INT8 and updates it by unbiased stochastic rounding;
    it does not say what happens at the ends of the grid.  Saturating (the
    default, stochastic_round_update) is biased there; this variant is the
    plainest reading that keeps the rounding unbiased: make the grid fit.

    With X and K = rint(X) as in stochastic_round_update, each element's value
    in units of 2^-16 code is the integer T = q * 2^16 + K (T = q * 2^16 where X
    is NaN).  Per group g of 256 consecutive elements, A = max |T|:
      A <= 127 * 2^16: the codes are those of stochastic_round_update (no
                       element can reach the clamp) and the scale is kept;
      otherwise:       rho = (127 * 2^16) / A and s'_g = s_g / rho (IEEE float32
                       divisions); Z = fl(T) * rho (float32, fl the nearest
                       float), K' = rint(Z) (ties to even), and the code is
                       clamp(floor((K' + d) / 2^16), -127, 127) with the same
                       draw d.  E[code' s'] = T 2^-16 s up to the nearest-point
                       rounding of Z: still unbiased, and odd in T.
    Returns (codes, scales)."""
    m, n = Wq.shape
    e = np.arange(m * n, dtype=np.int64).reshape(m, n)
    sW = np.asarray(sW, np.float32)
    c = np.where(sW > 0, F32(cfg.alpha) / np.where(sW > 0, sW, F32(1)), F32(0)).astype(np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        cp = (c * F32(65536.0)).astype(np.float32)
        X = (np.asarray(U, np.float32) * cp[e // cfg.w_group]).astype(np.float32)
        nan = np.isnan(X)
        K = np.rint(np.clip(np.where(nan, F32(0), X), F32(-2.0 ** 30), F32(2.0 ** 30))).astype(np.int64)
    if u16 is None:
        u16 = sr_uniform16(m, n, cfg.seed, t, cfg.layer_id)
    d = np.asarray(u16, np.int64)
    T = Wq.astype(np.int64) * 65536 + np.where(nan, 0, K)
    g = e.ravel() // cfg.w_group
    flatT, flatd = T.ravel(), d.ravel()
    A = np.zeros(len(sW), np.int64)
    np.maximum.at(A, g, np.abs(flatT))                  # per group max |T|
    grow = (A > W_RESCALE_LIMIT) & (sW > 0)
    rho = np.ones(len(sW), np.float32)
    rho[grow] = F32(W_RESCALE_LIMIT) / A[grow].astype(np.float32)
    s_new = sW.copy()
    s_new[grow] = (sW[grow] / rho[grow]).astype(np.float32)
    Z = (flatT.astype(np.float32) * rho[g]).astype(np.float32)
    Kp = np.where(grow[g], np.rint(Z).astype(np.int64), flatT)
    out = np.clip((Kp + flatd) >> 16, -INT8_QMAX, INT8_QMAX)
    return out.reshape(m, n).astype(np.int8), s_new


@dataclass
class LayerState:
    """Everything one weight matrix carries between steps."""
    cfg: Config
    Wq: np.ndarray            # m x n int8
    sW: np.ndarray            # ceil(m*n/256) float32, fixed
    Pq: np.ndarray | None = None      # packed INT4 (ceil(m*r/2) uint8)
    sP: np.ndarray | None = None      # ceil(m*r/64) float32
    Pq_prev: np.ndarray | None = None
    sP_prev: np.ndarray | None = None
    Mq: np.ndarray = None     # r x n int8
    sM: np.ndarray = None     # r x ceil(n/256) float32
    Vq: np.ndarray = None
    sV: np.ndarray = None
    t: int = 0
    delta: int = 0
    t_next: int = 0
    n_refresh: int = 0
    cossim_trace: list = field(default_factory=list)

    @staticmethod
    def create(cfg: Config, Wq, sW):
        _, rows, cols = proj_dims(cfg)
        nb = -(-cols // cfg.mom_block)
        return LayerState(cfg=cfg, Wq=np.array(Wq, np.int8), sW=np.array(sW, np.float32),
                          Mq=np.zeros((rows, cols), np.int8), sM=np.zeros((rows, nb), np.float32),
                          Vq=np.zeros((rows, cols), np.int8), sV=np.zeros((rows, nb), np.float32),
                          delta=cfg.delta0)


def step(st: LayerState, G) -> dict:
    """One optimizer step a1..a5 on one weight matrix (mutates `st`).

    Returns the intermediates (P~, R, N, U) for inspection."""
    cfg = st.cfg
    st.t += 1
    p_rows, _, _ = proj_dims(cfg)
    Pb = dequant_P_bf16(st.Pq, st.sP, p_rows, cfg.r, cfg.p_group)
    R = project(Pb, G) if cfg.proj_side == 0 else project_right(G, Pb)
    N, st.Mq, st.sM, st.Vq, st.sV = lowrank_adam_int8(R, st.Mq, st.sM, st.Vq, st.sV, cfg, st.t)
    U = backproject(Pb, N) if cfg.proj_side == 0 else backproject_right(N, Pb)
    if cfg.w_rescale:
        st.Wq, st.sW = stochastic_round_rescale(st.Wq, st.sW, U, cfg, st.t)
    else:
        st.Wq = stochastic_round_update(st.Wq, st.sW, U, cfg, st.t)
    return dict(P=Pb, R=R, N=N, U=U)


# --------------------------------------------------------------------------
# Subspace refresh (a6) and the layer-adaptive schedule (a7)
# --------------------------------------------------------------------------

OMEGA_KEY_SALT = 0x52454652


def refresh_width(cfg: Config) -> int:
    """k = r + oversampling, capped by min(m, n)."""
    return min(cfg.r + cfg.oversample, cfg.m, cfg.n)


def rademacher_omega(n, k, seed, refresh_idx, layer_id) -> np.ndarray:
    """Test matrix Omega (n x k) of +-1.  Entry e = j*k + c takes bit (e mod 32)
    of word ((e / 32) mod 4) of Philox-4x32-10(counter = (e / 128, refresh_idx,
    layer_id, 0), key = (seed_lo ^ 0x52454652, seed_hi)); a set bit gives -1."""
    assert n * k < (1 << 39)
    e = np.arange(n * k, dtype=np.uint64)
    w = philox4x32_10(e >> np.uint64(7), refresh_idx, layer_id, 0,
                      (seed & 0xFFFFFFFF) ^ OMEGA_KEY_SALT, (seed >> 32) & 0xFFFFFFFF)
    words = np.stack(w, 0)[((e >> np.uint64(5)) & np.uint64(3)).astype(np.int64), np.arange(n * k)]
    bit = (words >> (e & np.uint64(31)).astype(np.uint32)) & np.uint32(1)
    return np.where(bit == 1, -1.0, 1.0).reshape(n, k)


def canonical_signs(P) -> np.ndarray:
    """Make the entry of largest magnitude of every column positive (the first
    such row on ties): fixes the sign freedom of singular vectors."""
    P = np.array(P, dtype=np.float64)
    idx = np.argmax(np.abs(P), axis=0)
    sgn = np.where(P[idx, np.arange(P.shape[1])] < 0, -1.0, 1.0)
    return P * sgn[None, :]


def _orth(Y):
    """Orthonormal basis of the column span (Householder QR, a library step)."""
    Q, _ = np.linalg.qr(Y, mode="reduced")
    return Q


def randomized_topr(G, r, k, power_iters, Omega) -> tuple[np.ndarray, np.ndarray]:
    """Randomized subspace iteration for the top-r left singular vectors of G
    (Halko, Martinsson, Tropp 2011: range finder with power iterations, then
    Rayleigh-Ritz), in float64:

        Q = orth(G Omega);  repeat q times: Z = orth(G^T Q); Q = orth(G Z)
        B = Q^T G;  S = B B^T = V diag(lambda) V^T (descending)
        P = Q V[:, :r], columns sign-canonical.

    The span of each orth() is independent of the basis it returns, and so is
    P: any orthonormalisation (QR, Cholesky-QR) gives the same P in exact
    arithmetic.  Returns (P m x r, sigma = sqrt(lambda[:r]))."""
    G = np.asarray(G, np.float64)
    Q = _orth(G @ Omega)
    for _ in range(power_iters):
        Z = _orth(G.T @ Q)
        Q = _orth(G @ Z)
    B = Q.T @ G
    lam, V = np.linalg.eigh(B @ B.T)
    order = np.argsort(-lam, kind="stable")
    lam, V = lam[order], V[:, order]
    P = canonical_signs(Q @ V[:, :r])
    return P, np.sqrt(np.maximum(lam[:r], 0.0))


def exact_topr(G, r) -> tuple[np.ndarray, np.ndarray]:
    """Top-r left singular vectors by a full SVD (LAPACK), sign-canonical."""
    U, s, _ = np.linalg.svd(np.asarray(G, np.float64), full_matrices=False)
    return canonical_signs(U[:, :r]), s[:r]


def cossim(Pa, Pb) -> float:
    """[QG-sched] Eq. (5): CosSim(Pa, Pb) = (1/r) * sum_i sigma_i(Pa^T Pb)."""
    Pa = np.asarray(Pa, np.float64)
    Pb = np.asarray(Pb, np.float64)
    s = np.linalg.svd(Pa.T @ Pb, compute_uv=False)
    return float(s.sum() / Pa.shape[1])


def schedule_after_refresh(t, delta, cs, gamma):
    """[QG-sched]: after a refresh at step t with CosSim `cs` against the previous
    projection (None at the first refresh), the interval doubles iff cs > gamma
    (strict); the next refresh is due at t + delta.  Returns (delta, t_next)."""
    if cs is not None and cs > gamma:
        delta = 2 * delta
    return delta, t + delta


def refresh_due(st: LayerState, force=False) -> bool:
    return bool(force) or st.t == st.t_next


def refresh(st: LayerState, G, force=False) -> dict | None:
    """Subspace refresh of one layer, if due: randomized top-r SVD of G, INT4
    quantization of the new P, CosSim against the previous INT4 P (both
    dequantized to float32), the doubling rule.  Reading: the moments are kept
    as they are across a refresh.  Returns None when not due."""
    if not refresh_due(st, force):
        return None
    cfg = st.cfg
    k = refresh_width(cfg)
    # the right-side variant takes the top-r left singular vectors of G^T
    Geff = np.asarray(G) if cfg.proj_side == 0 else np.asarray(G).T
    p_rows = Geff.shape[0]
    Omega = rademacher_omega(Geff.shape[1], k, cfg.seed, st.n_refresh, cfg.layer_id)
    P, sigma = randomized_topr(Geff, cfg.r, k, cfg.power_iters, Omega)
    codes, sP = quant_int4_groups(P.astype(np.float32), cfg.p_group)
    Pq = pack_int4(codes)
    cs = None
    if st.Pq is not None:
        Pa = dequant_int4_f32(Pq, sP, p_rows, cfg.r, cfg.p_group)
        Pb = dequant_int4_f32(st.Pq, st.sP, p_rows, cfg.r, cfg.p_group)
        cs = cossim(Pa, Pb)
        refresh_moments(st, Pa, Pb)
        st.Pq_prev, st.sP_prev = st.Pq, st.sP
    st.Pq, st.sP = Pq, sP
    st.delta, st.t_next = schedule_after_refresh(st.t, st.delta, cs, cfg.gamma)
    st.n_refresh += 1
    st.cossim_trace.append((st.t, cs))
    return dict(P=P, sigma=sigma, cossim=cs, Omega=Omega)


def refresh_moments(st: LayerState, Pa, Pb):
    """The low-rank moments at a refresh that replaces the projection Pb (the
    dequantized previous P, m x r) by Pa (the dequantized new one).  The moments
    live in P's coordinates (R = P^T G, r x n), and the pages do not say what
    happens to them when P changes.  cfg.mom_refresh selects a reading:
      0  keep them as they are (the default);
      1  reset them to zero;
      2  rotate them into the new basis: with C = Pa^T Pb (r x r), m' = C m, the
         first moment mapped as a vector is; v' = (C o C) v, the second moment
         mapped as the variance of independent coordinates is (C o C the
         element-wise square).  C, and both products, in float64 from the
         float32 operands; the results rounded to float32 and re-quantized on the
         step's grids (linear for m, square root for v).  For the right-side
         projection the r coordinates run along the columns of the moments
         (m x r): m' = m C^T and v' = v (C o C)^T."""
    cfg = st.cfg
    if cfg.mom_refresh == 0:
        return
    if cfg.mom_refresh == 1:
        st.Mq = np.zeros_like(st.Mq)
        st.Vq = np.zeros_like(st.Vq)
        st.sM = np.zeros_like(st.sM)
        st.sV = np.zeros_like(st.sV)
        return
    if cfg.mom_refresh != 2:
        raise ValueError("mom_refresh must be 0, 1 or 2")
    C = np.asarray(Pa, np.float64).T @ np.asarray(Pb, np.float64)
    m0 = dequant_rowblock(st.Mq, st.sM, cfg.mom_block).astype(np.float64)
    v0 = dequant_second_moment(st.Vq, st.sV, cfg.mom_block).astype(np.float64)
    if cfg.proj_side == 0:
        m1 = (C @ m0).astype(np.float32)
        v1 = ((C * C) @ v0).astype(np.float32)
    else:
        m1 = (m0 @ C.T).astype(np.float32)
        v1 = (v0 @ (C * C).T).astype(np.float32)
    st.Mq, st.sM = quant_rowblock_int8(m1, cfg.mom_block, unsigned=False)
    st.Vq, st.sV = quant_rowblock_int8(np.sqrt(v1).astype(np.float32), cfg.mom_block, unsigned=True)


def set_projection(st: LayerState, P):
    """Quantize and install a given float projection (m x r) as P^Q."""
    codes, sP = quant_int4_groups(np.asarray(P, np.float32), st.cfg.p_group)
    st.Pq, st.sP = pack_int4(codes), sP


# --------------------------------------------------------------------------
# Linear layers around the optimizer: simulated weight-only INT8 quantization.
# [QG-lim] AIMech Q-GaLore page, limitation "simulated weight-quantization
# throughput" (paper section 3.2 and section 4.4, Fig. 4): activations stay in
# 16-bit floating point and the INT8 weights are dequantized for the forward and
# backward matrix products.  [QG-thm] same page, Theorem 3.1 (paper section
# 3.1, Eqs. (3)-(4)): for a linear layer y = W x the weight gradient is
# G = (1/B) D_y X^T.
# Readings: W~ = bf16_rn(fp32(q) * s_g), one float32 product rounded to bf16,
# with g = floor((i n + j) / 256) the group of the optimizer's own W grid; the
# three products are the exact sums (float64 here), which the GPU rounds once to
# bf16 after a float32 accumulation; the 1/B of G is folded into D_y, so G is
# the bf16 gradient the optimizer step takes.
# --------------------------------------------------------------------------


def dequant_weight_bf16(Wq, sW, group=256) -> np.ndarray:
    """W~ (m x n float32 holding bf16 values) from INT8 codes and the flattened
    group scales: each element is float32(q) times its group's scale, rounded
    once to float32 and then to bf16 (round to nearest even)."""
    Wq = np.asarray(Wq)
    m, n = Wq.shape
    g = (np.arange(m, dtype=np.int64)[:, None] * n + np.arange(n, dtype=np.int64)[None, :]) // group
    prod = Wq.astype(np.float32) * np.asarray(sW, np.float32)[g]
    return bf16_round(prod.astype(np.float32))


def linear_forward(X, Wt) -> np.ndarray:
    """Y = X W~^T (T x m) for activations X (T x n) and the dequantized weight
    W~ (m x n), exact in float64."""
    return np.asarray(X, np.float64) @ np.asarray(Wt, np.float64).T


def linear_backward_data(dY, Wt) -> np.ndarray:
    """dX = D_y W~ (T x n) for the output gradient D_y (T x m), exact in float64."""
    return np.asarray(dY, np.float64) @ np.asarray(Wt, np.float64)


def linear_backward_weight(dY, X) -> np.ndarray:
    """G = D_y^T X (m x n), the weight gradient of y = W x over the T rows of the
    batch, exact in float64."""
    return np.asarray(dY, np.float64).T @ np.asarray(X, np.float64)
