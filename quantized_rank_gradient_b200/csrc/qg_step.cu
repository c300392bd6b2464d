// The optimizer step a1..a5 on sm_100a.
//
//   a1  dequant_projection_kernel : INT4 P^Q -> P~ (bf16, m x r) in scratch
//   a2+a3  gemm_tc_kernel<AdamEpi, A MN-major, B MN-major>:
//          R = P~^T G in TMEM; the epilogue runs Adam on the INT8 moments,
//          re-quantizes them and writes N (bf16, r x n) to scratch.  R never
//          leaves the SM.
//   a4+a5  gemm_tc_kernel<StochRoundEpi, A K-major, B MN-major>:
//          U = P~ N in TMEM; the epilogue adds alpha*U/s_W to the INT8 weights
//          with Philox-keyed stochastic rounding.  U never leaves the SM.
//
// Arithmetic follows the Q-GaLore step as described on the AIMech Q-GaLore
// page (mechanism "INT4 projection and INT8 stochastic rounding", paper
// section 3.2) with the readings documented in the repository's design notes;
// every float32 operation that decides a code uses an explicitly rounded
// intrinsic so that no multiply-add is contracted.
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>
#include <mutex>

#include "qg_exact.cuh"
#include "qg_gemm.cuh"
#include "qg_internal.h"
#include "qg_philox.cuh"
#include "qg_refresh.h"

#ifndef QG_SR_REVERSE
#define QG_SR_REVERSE 1
#endif
#include "../../include/qgalore.h"

namespace qg {

static_assert(kErrTimeout == kStatusTimeout && kErrNonFinite == kStatusNonFinite, "status bits");

// Groups / blocks whose absmax is below this are quantized as zero (127 / absmax
// would overflow float32).
constexpr float kAbsmaxFloor = 7.52316384526264e-37f;  // 2^-120

// ------------------------------------------------------------------ helpers

QG_DEV uint32_t word_of(const uint4& v, int k) { return k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w; }

QG_DEV uint16_t bf16_bits_rn(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

QG_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Conversions between small integers and float32 done with integer/FP-add
// arithmetic (exact for |value| < 2^22) instead of the conversion pipe.
// 12582912 = 1.5 * 2^23: a float in [2^23, 2^24) has an integer ulp of 1.
constexpr float kMagic = 12582912.0f;
constexpr uint32_t kMagicBits = 0x4B400000u;

// Byte k (0..3) of w as a signed int8, converted to float exactly (k is a
// constant after unrolling, so the selector is an immediate).
QG_DEV float sbyte_f32(uint32_t w, int k) {
  const uint32_t sel = k | ((k | 8) << 4) | ((k | 8) << 8) | ((k | 8) << 12);  // sign-extend byte k
  const uint32_t sx = prmt(w, 0u, sel);
  return __fsub_rn(__uint_as_float(kMagicBits + sx), kMagic);
}

// 16-bit draw h (0: low half, 1: high half) of w as u = u16 * 2^-16, exact.
QG_DEV float draw_u(uint32_t w, int h) {
  const uint32_t m = h ? ((w >> 9) & 0x007FFF80u) : ((w << 7) & 0x007FFF80u);
  return __fsub_rn(__uint_as_float(0x3F800000u | m), 1.0f);
}

// x (integer-valued or not, already clamped to [-127, 127]) rounded to the
// nearest integer, ties to even, returned in the low byte.
QG_DEV uint32_t round_to_byte(float x) { return __float_as_uint(__fadd_rn(x, kMagic)); }

// max(m, |x|) propagating NaN: a NaN x makes the result NaN.
QG_DEV float max_nan_abs(float m, float x) {
  float r;
  asm("{\n\t.reg .f32 t;\n\tabs.f32 t, %2;\n\tmax.NaN.f32 %0, %1, t;\n\t}" : "=f"(r) : "f"(m), "f"(x));
  return r;
}

// Both signed 16-bit lanes of x clamped to [-127, 127].
QG_DEV uint32_t clamp127_s16x2(uint32_t x) {
  uint32_t r;
  asm("max.s16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(0xFF81FF81u));
  asm("min.s16x2 %0, %1, %2;" : "=r"(r) : "r"(r), "r"(0x007F007Fu));
  return r;
}

// max(m, v) propagating NaN.
QG_DEV float max_nan(float m, float v) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(m), "f"(v));
  return r;
}

// 16-byte granule g (0..15) of row `row` of a 128 x 256 int8 side tile, staged by
// TMA as two 128 x 128 boxes with the 128-byte swizzle (granule j of a 128-byte
// row r is stored at position j ^ (r mod 8)).
QG_DEV uint4 side_granule(const uint8_t* side, int row, int g) {
  return *reinterpret_cast<const uint4*>(side + (g >> 3) * 16384 + row * 128 + (((g & 7) ^ (row & 7)) << 4));
}

// Low bytes of four words packed into one word.
QG_DEV uint32_t pack4(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  return prmt(prmt(b0, b1, 0x0040u), prmt(b2, b3, 0x0040u), 0x5410u);
}

// ------------------------------------------------------------------ a2 + a3 epilogue

struct AdamEpi {
  // side operands: the tile's M^Q codes (bytes [0, 32K)) and V^Q codes ([32K, 64K))
  static constexpr int kSideBytes = 65536;
  static constexpr int kSideBufs = 1;
  static constexpr bool kExchange = true;  // block maxima combined across the two warpgroups

  static QG_DEV void issue_side(const CUtensorMap* tmS, int mb, int nb, uint8_t* dst, uint64_t* bar) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      tma_load_2d(dst + k * 32768, &tmS[k], bar, nb * BN, mb * BM);
      tma_load_2d(dst + k * 32768 + 16384, &tmS[k], bar, nb * BN + 128, mb * BM);
    }
  }

  struct Args {
    int8_t* Mq;
    int8_t* Vq;
    float* sM;
    float* sV;
    uint16_t* Nout;
    int64_t ld_mom;
    int64_t ldN;
    int32_t nblk;
    float beta1, beta2, om1, om2, c1, c2, eps;
  };

  // m = b1*m0 + (1-b1)*R ; v = b2*v0 + (1-b2)*(R*R), one rounding per operation.
  // M^Q holds m on a linear grid; V^Q holds sqrt(v), so v0 = (code*scale)^2.
  static QG_DEV void moments(float R, float mc, float vc, float sm, float sv, const Args& a, float& mm,
                             float& vv) {
    const float m0 = __fmul_rn(mc, sm);
    const float d0 = __fmul_rn(vc, sv);
    const float v0 = __fmul_rn(d0, d0);
    mm = __fadd_rn(__fmul_rn(a.beta1, m0), __fmul_rn(a.om1, R));
    vv = __fadd_rn(__fmul_rn(a.beta2, v0), __fmul_rn(a.om2, __fmul_rn(R, R)));
  }

  // the pair kernel drains every tile with four epilogue warpgroups, 64 columns each
  static constexpr int kPairGroups = 4;
  // Ring stages of K = 64 (32 KiB per CTA): four fit beside the 64 KiB side
  // tiles.  Measured on the 7B stack: three stages made the launch 12 % slower;
  // nine stages of K = 32 (more bytes in flight, but two MMAs per stage) 25 %
  // slower.
  static constexpr int kPairBKMN = 64;
  static constexpr int kPairMaxStages = 6;

  // Pass 1 on one 16-column sub-chunk (moment codes in qm, qv): the new moments
  // and the running block maxima of |m| and of v (max over the block of sqrt(v)
  // is sqrt of the max of v, the correctly rounded square root being monotone).
  // The maxima propagate NaN, so a non-finite moment shows in them.  It also
  // keeps the smallest |m| and v (zeros included), which decide whether pass 2
  // may use the branch-free square root and division.  kFull: all 16 columns are
  // inside the matrix.
  template <bool kFull>
  static QG_DEV void pass1_sub(const Args& a, const uint32_t (&v)[16], const uint4& qm, const uint4& qv, float sm,
                               float sv, int valid, float& amax_m, float& amax_vv, float& mmin, float& vmin) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float R = __uint_as_float(v[e]);
      float mm, vv;
      moments(R, sbyte_f32(word_of(qm, e >> 2), e & 3), sbyte_f32(word_of(qv, e >> 2), e & 3), sm, sv, a, mm, vv);
      if (kFull || e < valid) {
        amax_m = max_nan_abs(amax_m, mm);
        amax_vv = max_nan(amax_vv, vv);
        mmin = fminf(mmin, fabsf(mm));
        vmin = fminf(vmin, vv);
      }
    }
  }

  // True when every square root and division of this thread's pass 2 has its
  // operands and quotient inside the ranges where sqrt_exact and div_exact equal
  // the IEEE operations: v in [2^-100, 2^100], the denominator sqrt(v) c2 + eps
  // in [eps, dmax] within [2^-100, 2^100], the numerator m c1 in [2^-90, 2^90],
  // and every quotient in [2^-100, 2^100].  A zero m or v sends the row to the
  // intrinsics, as does anything non-finite.
  static QG_DEV bool exact_fast_ok(const Args& a, float amax_m, float amax_vv, float mmin, float vmin) {
    const float c1a = fabsf(a.c1);
    bool ok = amax_m <= 3.4028234663852886e38f && amax_vv <= kSafeHi && vmin >= kSafeLo && a.eps >= kSafeLo &&
              a.c2 > 0.f;
    const float dmax = __fadd_rn(__fmul_rn(__fsqrt_rn(amax_vv), a.c2), a.eps);
    const float nmax = __fmul_rn(amax_m, c1a);
    const float nmin = __fmul_rn(mmin, c1a);
    ok = ok && dmax <= kSafeHi && nmax <= kSafeDivHi && nmax <= __fmul_rn(kSafeHi, a.eps);
    ok = ok && nmin >= kSafeDivLo && nmin >= __fmul_rn(kSafeLo, dmax);
    return ok;
  }

  // Pass 2 on one 16-column sub-chunk: the same moments; N = -lr m_hat /
  // (sqrt(v_hat) + eps) = (m c1) / (sqrt(v) c2 + eps) -> bf16; codes of m and
  // sqrt(v) on the block's new grids.  |m| * (127 / absmax) and sqrt(v) *
  // (127 / absmax_v) stay within 127 (1 + 2^-24), so their nearest integers need
  // no clamp; a zero block has inverse scale 0 and gets codes 0.
  // kExact selects sqrt_exact / div_exact, equal to the IEEE operations on the
  // ranges exact_fast_ok checks, over the intrinsics.
  template <bool kExact>
  static QG_DEV void pass2_sub(const Args& a, const uint32_t (&v)[16], const uint4& qm, const uint4& qv, float sm,
                               float sv, float inv_m, float inv_v, uint16_t* nptr, int8_t* mptr, int8_t* vptr) {
    uint32_t om[4], ov[4], packed[8], bm[4], bv[4];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float R = __uint_as_float(v[e]);
      float mm, vv;
      moments(R, sbyte_f32(word_of(qm, e >> 2), e & 3), sbyte_f32(word_of(qv, e >> 2), e & 3), sm, sv, a, mm, vv);
      const float rv = kExact ? sqrt_exact(vv) : __fsqrt_rn(vv);
      const float num = __fmul_rn(mm, a.c1), den = __fadd_rn(__fmul_rn(rv, a.c2), a.eps);
      const float upd = kExact ? div_exact(num, den) : __fdiv_rn(num, den);
      const uint32_t b = bf16_bits_rn(upd);
      if (e & 1)
        packed[e >> 1] |= b << 16;
      else
        packed[e >> 1] = b;
      bm[e & 3] = round_to_byte(__fmul_rn(mm, inv_m));
      bv[e & 3] = round_to_byte(__fmul_rn(rv, inv_v));
      if ((e & 3) == 3) {
        om[e >> 2] = pack4(bm[0], bm[1], bm[2], bm[3]);
        ov[e >> 2] = pack4(bv[0], bv[1], bv[2], bv[3]);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(nptr);
    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    *reinterpret_cast<uint4*>(mptr) = make_uint4(om[0], om[1], om[2], om[3]);
    *reinterpret_cast<uint4*>(vptr) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
  }

  // One thread owns row `row` of its warpgroup's slice (BN / groups columns) of
  // the 128 x 256 tile; the tile's 256 columns are exactly one moment block, so
  // the block maxima of all slices are combined through the exchange before the
  // codes are formed.  The tile's codes are staged in shared memory; 16-column
  // sub-chunks keep the thread's registers within the four-warpgroup budget.
  static QG_DEV void apply(const Args& a, int M, int N, int mb, int nb, int row, uint32_t taddr,
                           const EpiPair& ep, const uint8_t* side) {
    const int arow = mb * BM + row;
    const bool row_ok = arow < M;
    const int j0 = nb * BN;
    const int ncols = min(BN, N - j0);
    const int nsub = BN / 16 / ep.groups;
    const int s0 = ep.group * nsub;
    const int s1 = min(s0 + nsub, (ncols + 15) >> 4);
    float sm = 0.f, sv = 0.f;
    int8_t* mrow = nullptr;
    int8_t* vrow = nullptr;
    uint16_t* nrow = nullptr;
    if (row_ok) {
      sm = a.sM[static_cast<int64_t>(arow) * a.nblk + nb];
      sv = a.sV[static_cast<int64_t>(arow) * a.nblk + nb];
      mrow = a.Mq + static_cast<int64_t>(arow) * a.ld_mom + j0;
      vrow = a.Vq + static_cast<int64_t>(arow) * a.ld_mom + j0;
      nrow = a.Nout + static_cast<int64_t>(arow) * a.ldN + j0;
    }
    float amax_m = 0.f, amax_vv = 0.f, mmin = __int_as_float(0x7f800000), vmin = __int_as_float(0x7f800000);

    // The loop control of both passes is warp-uniform (s0, s1 depend on the
    // tile only); the lane-varying row predicate guards the arithmetic alone and
    // is re-read per sub-chunk (lane_pred).
    auto p1 = [&](const uint32_t (&v)[16], int s, const uint4& qm, const uint4& qv) {
      if (!lane_pred(row_ok)) return;
      const int valid = ncols - s * 16;
      if (valid >= 16)
        pass1_sub<true>(a, v, qm, qv, sm, sv, valid, amax_m, amax_vv, mmin, vmin);
      else
        pass1_sub<false>(a, v, qm, qv, sm, sv, valid, amax_m, amax_vv, mmin, vmin);
    };
    // Each sub-chunk's moment codes are read from shared memory while its
    // accumulators are on their way from tensor memory.
    __syncwarp();
#pragma unroll 1
    for (int s = s0; s < s1; ++s) {
      uint32_t v[16];
      tmem_ld_32x32b_x16(taddr + s * 16, v);
      const uint4 qm = side_granule(side, row, s), qv = side_granule(side + 32768, row, s);
      tmem_ld_wait(v);
      p1(v, s, qm, qv);
    }

    // a non-finite gradient reaches the maxima (they propagate NaN and Inf)
    const bool bad = !(amax_m <= 3.4028234663852886e38f) || !(amax_vv <= 3.4028234663852886e38f);
    const bool exact = exact_fast_ok(a, amax_m, amax_vv, mmin, vmin);

    // block maxima over all slices (the other groups' warps own the same rows);
    // the combination propagates NaN like the maxima themselves
    const int lane = row & 31;
    ep.xchg[ep.group * BM + lane] = make_float2(amax_m, amax_vv);
    __threadfence_block();
    __syncwarp();
    if (lane == 0) mbar_arrive(ep.xbar);
    if (mbar_wait(ep.xbar, ep.xphase, ep.abort, ep.status)) {
      for (int g = 0; g < ep.groups; ++g) {
        if (g == ep.group) continue;
        const float2 o = ep.xchg[g * BM + lane];
        amax_m = max_nan(amax_m, o.x);
        amax_vv = max_nan(amax_vv, o.y);
      }
    }
    const float amax_v = __fsqrt_rn(amax_vv);

    // new block scales absmax / 127 and inverse scales 127 / absmax (IEEE
    // divisions, once per block); a block whose absmax is below 2^-120 is a zero
    // block (scale 0, codes 0)
    const bool live_m = amax_m >= kAbsmaxFloor, live_v = amax_v >= kAbsmaxFloor;
    const float s_m = live_m ? __fdiv_rn(amax_m, 127.0f) : 0.f;
    const float s_v = live_v ? __fdiv_rn(amax_v, 127.0f) : 0.f;
    const float inv_m = live_m ? __fdiv_rn(127.0f, amax_m) : 0.f;
    const float inv_v = live_v ? __fdiv_rn(127.0f, amax_v) : 0.f;

    // both predicates vary across the lanes of a warp (exact depends on the
    // row's maxima), so both are re-read per sub-chunk
    auto p2 = [&](const uint32_t (&v)[16], int s, const uint4& qm, const uint4& qv) {
      if (!lane_pred(row_ok)) return;
      if (lane_pred(exact))
        pass2_sub<true>(a, v, qm, qv, sm, sv, inv_m, inv_v, nrow + s * 16, mrow + s * 16, vrow + s * 16);
      else
        pass2_sub<false>(a, v, qm, qv, sm, sv, inv_m, inv_v, nrow + s * 16, mrow + s * 16, vrow + s * 16);
    };
    __syncwarp();
#pragma unroll 1
    for (int s = s0; s < s1; ++s) {
      uint32_t v[16];
      tmem_ld_32x32b_x16(taddr + s * 16, v);
      const uint4 qm = side_granule(side, row, s), qv = side_granule(side + 32768, row, s);
      tmem_ld_wait(v);
      p2(v, s, qm, qv);
    }
    if (row_ok && ep.group == 0) {
      a.sM[static_cast<int64_t>(arow) * a.nblk + nb] = s_m;
      a.sV[static_cast<int64_t>(arow) * a.nblk + nb] = s_v;
    }
    if (bad && ep.status) atomicOr(ep.status, kErrNonFinite);
  }
};

// ------------------------------------------------------------------ a4 + a5 epilogue

struct StochRoundEpi {
  // side operand: the tile's W codes (128 rows x 256 columns), double-buffered
  static constexpr int kSideBytes = 32768;
  static constexpr int kSideBufs = 2;
  static constexpr bool kExchange = false;

  static QG_DEV void issue_side(const CUtensorMap* tmS, int mb, int nb, uint8_t* dst, uint64_t* bar) {
    tma_load_2d(dst, &tmS[0], bar, nb * BN, mb * BM);
    tma_load_2d(dst + 16384, &tmS[0], bar, nb * BN + 128, mb * BM);
  }

  struct Args {
    int8_t* W;
    float* sW;           // written only by the re-scaling variant
    int64_t ldw;
    float alpha;
    uint32_t t, layer_id;
    PhiloxKey key;
    int32_t aligned256;  // n % 256 == 0: a tile row is exactly one weight group
  };

  // the pair kernel drains every tile with two epilogue warpgroups, 128 columns
  // each (measured on the 7B stack, three warpgroups, and four with 16-column
  // sub-chunks, ran no faster)
  static constexpr int kPairGroups = 2;
  // A is K-major (stages of K = 64); four stages measured 2-7 % faster than
  // five on the 7B stack
  static constexpr int kPairBKMN = 64;
  static constexpr int kPairMaxStages = 4;

  // The 16-bit draws of columns jc .. jc+31 of row irow (jc a multiple of 32):
  // column j's draw is half (j mod 2) of word ((j / 2) mod 4) of
  // Philox-4x32-10(counter = (j / 8, irow, t, layer_id), key = seed), so column
  // jc + i takes half (i & 1) of d[i >> 1].  Every row starts a Philox call.
  static QG_DEV void draws(const Args& a, const PhiloxRoundKeys& rk, int irow, int jc, uint32_t (&d)[16]) {
    const uint32_t cb = static_cast<uint32_t>(jc) >> 3;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t o[4];
      philox4x32_10(cb + k, static_cast<uint32_t>(irow), a.t, a.layer_id, rk, o);
      d[4 * k] = o[0];
      d[4 * k + 1] = o[1];
      d[4 * k + 2] = o[2];
      d[4 * k + 3] = o[3];
    }
  }

  // c'_g = (alpha / s_g) * 2^16: the update factor in units of 2^-16 code; a
  // scale that is not positive freezes its group.
  static QG_DEV float update_factor(float alpha, float s) {
    return s > 0.f ? __fmul_rn(__fdiv_rn(alpha, s), 65536.0f) : 0.f;
  }

  // One 32-column chunk: W codes in (wa, wb), U from TMEM, draws d; the new codes
  // in out[8].  With X = U c' (the update in units of 2^-16 code) and
  // K = rint(X) (nearest, ties to even), the new code is
  // clamp(q + floor((K + draw) / 2^16), -127, 127), and a NaN X keeps q.
  //
  // Fast form, valid while |X| < 2^22: fadd.rn(X, 1.5 * 2^23) has the bits
  // 0x4B400000 + K (the sum lies in [2^23, 2^24), where the float32 step is 1,
  // and 1.5 * 2^23 is even, so ties go to the even K); adding the draw less
  // 0x4B400000 and q * 2^16 leaves K + draw + q * 2^16, whose bits [16, 32) are
  // q + r with r = floor((K + draw) / 2^16) (|q + r| <= 191).  Two such sums
  // give one pair of 16-bit lanes, clamped to [-127, 127] by one max and one
  // min on both lanes; the low bytes of four lanes are the four new codes.
  // When |X| reaches 2^22, or X is NaN, the chunk is redone in the general form.
  template <bool kOneFactor>
  static QG_DEV void sr_chunk(const uint32_t (&U)[32], const uint4& wa, const uint4& wb, const uint32_t (&d)[16],
                              float cp0, float cp1, int split, uint32_t (&out)[8]) {
    float mx = 0.f;
    uint32_t sum[2], lanes[2];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float cp = (kOneFactor || k < split) ? cp0 : cp1;
      const float X = __fmul_rn(__uint_as_float(U[k]), cp);
      mx = max_nan_abs(mx, X);
      const uint32_t tb = __float_as_uint(__fadd_rn(X, kMagic));
      const uint32_t dq = prmt(d[k >> 1], 0xB4C00000u, (k & 1) ? 0x7632u : 0x7610u);
      const uint32_t wsel = 0x44u | (static_cast<uint32_t>(k & 3) << 8) | (static_cast<uint32_t>((k & 3) | 8) << 12);
      const uint32_t q16 = prmt(word_of(k < 16 ? wa : wb, (k >> 2) & 3), 0u, wsel);
      sum[k & 1] = tb + dq + q16;
      if (k & 1) lanes[(k >> 1) & 1] = clamp127_s16x2(prmt(sum[0], sum[1], 0x7632u));
      if ((k & 3) == 3) out[k >> 2] = prmt(lanes[0], lanes[1], 0x6420u);
    }
    if (!(mx < 4194304.0f)) {
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float cp = (kOneFactor || k < split) ? cp0 : cp1;
        const float X = __fmul_rn(__uint_as_float(U[k]), cp);
        const uint4& w = k < 16 ? wa : wb;
        const int q = static_cast<int8_t>((word_of(w, (k >> 2) & 3) >> (8 * (k & 3))) & 0xFFu);
        int v = q, K = 0;
        if (X == X) {
          K = __float2int_rn(fminf(fmaxf(X, -1073741824.0f), 1073741824.0f));
          const int draw = static_cast<int>((d[k >> 1] >> (16 * (k & 1))) & 0xFFFFu);
          v = min(max(q + ((K + draw) >> 16), -127), 127);
        }
        const uint32_t sh = 8 * (k & 3);
        out[k >> 2] = (out[k >> 2] & ~(0xFFu << sh)) | ((static_cast<uint32_t>(v) & 0xFFu) << sh);
      }
    }
  }

  // This warpgroup's slice of the tile's columns, 32-column chunks; W codes
  // come from the staged side tile, the new codes go straight to global memory.
  template <bool kOneGroup>
  static QG_DEV void apply_impl(const Args& a, int M, int N, int mb, int nb, int row, uint32_t taddr,
                                const EpiPair& ep, const uint8_t* side) {
    const int irow = mb * BM + row;
    const bool row_ok = irow < M;
    const int j0 = nb * BN;
    const int ncols = min(BN, N - j0);
    // group g of G takes the 32-column chunks [8 g / G, 8 (g + 1) / G) of the tile
    const int c0 = ep.group * (BN / 32) / ep.groups;
    const int c1 = min((ep.group + 1) * (BN / 32) / ep.groups, (ncols + 31) >> 5);
    float cp_row = 0.f;
    if (kOneGroup && row_ok) cp_row = update_factor(a.alpha, a.sW[(static_cast<int64_t>(irow) * N + j0) >> 8]);
    int8_t* wrow = a.W + static_cast<int64_t>(irow) * a.ldw + j0;
    const PhiloxRoundKeys rk = philox_round_keys(a.key);
    // The chunk's tensor-memory load is in flight while its Philox draws are
    // formed (pure ALU work, computed for every lane: a row past the matrix's
    // edge draws for nothing).  The loop control is warp-uniform; the
    // lane-varying row predicate guards the rounding and the stores alone and
    // is re-read per chunk (lane_pred).
    __syncwarp();
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
      uint32_t U[32];
      tmem_ld_32x32b_x32(taddr + c * 32, U);
      const int jc = c * 32;
      uint32_t d[16];
      draws(a, rk, irow, j0 + jc, d);
      tmem_ld_wait(U);
      if (!lane_pred(row_ok)) continue;
      const int valid = min(32, ncols - jc);
      const int64_t e0 = static_cast<int64_t>(irow) * N + j0 + jc;
      float cp0 = cp_row, cp1 = cp_row;
      int split = 32;
      if (!kOneGroup) {
        const int64_t g0 = e0 >> 8, g1 = (e0 + valid - 1) >> 8;
        cp0 = update_factor(a.alpha, a.sW[g0]);
        cp1 = g1 != g0 ? update_factor(a.alpha, a.sW[g1]) : cp0;
        split = g1 != g0 ? static_cast<int>((g1 << 8) - e0) : 32;
      }
      const uint4 wa = side_granule(side, row, 2 * c), wb = side_granule(side, row, 2 * c + 1);
      uint32_t out[8];
      sr_chunk<kOneGroup>(U, wa, wb, d, cp0, cp1, split, out);
      if (valid == 32) {
        *reinterpret_cast<uint4*>(wrow + jc) = make_uint4(out[0], out[1], out[2], out[3]);
        *reinterpret_cast<uint4*>(wrow + jc + 16) = make_uint4(out[4], out[5], out[6], out[7]);
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (k < valid) wrow[jc + k] = static_cast<int8_t>((out[k >> 2] >> (8 * (k & 3))) & 0xFFu);
      }
    }
  }

  static QG_DEV void apply(const Args& a, int M, int N, int mb, int nb, int row, uint32_t taddr,
                           const EpiPair& ep, const uint8_t* side) {
    if (a.aligned256)
      apply_impl<true>(a, M, N, mb, nb, row, taddr, ep, side);
    else
      apply_impl<false>(a, M, N, mb, nb, row, taddr, ep, side);
  }
};

// ------------------------------------------------------------------ a4 + a5, re-scaling variant

// A weight group that the update would carry off the INT8 grid gets a larger
// scale instead of saturating.  With X = U c' and K = rint(X) as above, every
// element's value in units of 2^-16 code is the integer T = q 2^16 + K
// (T = q 2^16 where X is NaN); per group, A = max |T|.
//   A <= 127 2^16: the codes are those of the saturating form (no element can
//                  reach the clamp) and the scale stays;
//   otherwise:     rho = (127 2^16) / A and s' = s / rho (IEEE float32
//                  divisions), and every code of the group becomes
//                  clamp(floor((rint(fl(T) rho) + draw) / 2^16), -127, 127)
//                  with the same draw, fl(T) the nearest float32.
// The expected value of code' s' stays q s + alpha U (up to the 2^-16 draw
// grid and float32 rounding).  Needs n % 256 == 0, so that a group is one row
// of a 256-column tile.  A first pass takes the row slice's exact max |T|, the
// two warpgroups combine their maxima through the exchange slots, and a
// second pass rounds every element once, on the grid its group ends up with.
struct StochRoundRescaleEpi : StochRoundEpi {
  static constexpr bool kExchange = true;
  static constexpr int kPairGroups = 2;  // 128 columns per warpgroup, the exchange pairs the two halves of a row
  static constexpr int kLimit = 127 * 65536;

  static QG_DEV void rescaled_chunk(const uint32_t (&U)[32], const uint4& wa, const uint4& wb,
                                    const uint32_t (&d)[16], float cp, float rho, uint32_t (&out)[8]) {
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float X = __fmul_rn(__uint_as_float(U[k]), cp);
      const uint4& w = k < 16 ? wa : wb;
      const int q = static_cast<int8_t>((word_of(w, (k >> 2) & 3) >> (8 * (k & 3))) & 0xFFu);
      const int K = X == X ? __float2int_rn(fminf(fmaxf(X, -1073741824.0f), 1073741824.0f)) : 0;
      const float Z = __fmul_rn(__int2float_rn(q * 65536 + K), rho);
      const int draw = static_cast<int>((d[k >> 1] >> (16 * (k & 1))) & 0xFFFFu);
      const int v = min(max((__float2int_rn(Z) + draw) >> 16, -127), 127);
      const uint32_t sh = 8 * (k & 3);
      if ((k & 3) == 0) out[k >> 2] = 0u;
      out[k >> 2] |= (static_cast<uint32_t>(v) & 0xFFu) << sh;
    }
  }

  static QG_DEV void store_chunk(int8_t* dst, const uint32_t (&out)[8]) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
    *reinterpret_cast<uint4*>(dst + 16) = make_uint4(out[4], out[5], out[6], out[7]);
  }

  // max |T| over one 32-column chunk, T = q 2^16 + K with K = rint(X) (0 where
  // X is NaN), the values in units of 2^-16 code; no draws.  Fast form while
  // |X| < 2^22: the bits of fadd.rn(X, 1.5 2^23) less 0x4B400000 are K; a chunk
  // with a larger or NaN X is redone with the conversion (X clipped to 2^30, as
  // the rounding does).  |T| < 2^31.
  static QG_DEV uint32_t chunk_tmax(const uint32_t (&U)[32], const uint4& wa, const uint4& wb, float cp) {
    float mx = 0.f;
    uint32_t amax = 0u;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float X = __fmul_rn(__uint_as_float(U[k]), cp);
      mx = max_nan_abs(mx, X);
      const uint32_t tb = __float_as_uint(__fadd_rn(X, kMagic));
      const uint32_t wsel = 0x44u | (static_cast<uint32_t>(k & 3) << 8) | (static_cast<uint32_t>((k & 3) | 8) << 12);
      const uint32_t q16 = prmt(word_of(k < 16 ? wa : wb, (k >> 2) & 3), 0u, wsel);
      const int T = static_cast<int>(tb + q16 - kMagicBits);
      amax = max(amax, static_cast<uint32_t>(abs(T)));
    }
    if (!(mx < 4194304.0f)) {
      amax = 0u;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float X = __fmul_rn(__uint_as_float(U[k]), cp);
        const uint4& w = k < 16 ? wa : wb;
        const int q = static_cast<int8_t>((word_of(w, (k >> 2) & 3) >> (8 * (k & 3))) & 0xFFu);
        const int K = X == X ? __float2int_rn(fminf(fmaxf(X, -1073741824.0f), 1073741824.0f)) : 0;
        amax = max(amax, static_cast<uint32_t>(abs(q * 65536 + K)));
      }
    }
    return amax;
  }

  // Two passes over the row slice.  Pass 1 takes the exact max |T| (no draws,
  // no stores); the two warpgroups combine their maxima through the exchange
  // slots; pass 2 rounds every element once, on the grown grid where the group
  // grows and on the saturating form's otherwise.  Loop control is
  // warp-uniform; the lane-varying predicates (row inside the matrix, group
  // grows) are re-read per chunk (lane_pred) and guard no tensor-memory load.
  static QG_DEV void apply(const Args& a, int M, int N, int mb, int nb, int row, uint32_t taddr,
                           const EpiPair& ep, const uint8_t* side) {
    const int irow = mb * BM + row;
    const bool row_ok = irow < M;
    const int j0 = nb * BN;  // N % 256 == 0: every tile is 256 columns wide
    const int nchunk = BN / 32 / ep.groups;
    const int c0 = ep.group * nchunk;
    const int64_t g = row_ok ? (static_cast<int64_t>(irow) * N + j0) >> 8 : 0;
    const float s = row_ok ? a.sW[g] : 0.f;
    const float cp = update_factor(a.alpha, s);
    int8_t* wrow = a.W + static_cast<int64_t>(irow) * a.ldw + j0;
    uint32_t amax = 0u;
    __syncwarp();
#pragma unroll 1
    for (int c = c0; c < c0 + nchunk; ++c) {
      uint32_t U[32];
      tmem_ld_32x32b_x32(taddr + c * 32, U);
      const uint4 wa = side_granule(side, row, 2 * c), wb = side_granule(side, row, 2 * c + 1);
      tmem_ld_wait(U);
      if (!lane_pred(row_ok)) continue;
      amax = max(amax, chunk_tmax(U, wa, wb, cp));
    }

    // the group's maximum over both column slices (the other group's warps own
    // the same rows); the slots carry the integer's bits
    const int lane = row & 31;
    ep.xchg[ep.group * BM + lane] = make_float2(__uint_as_float(amax), 0.f);
    __threadfence_block();
    __syncwarp();
    if (lane == 0) mbar_arrive(ep.xbar);
    if (mbar_wait(ep.xbar, ep.xphase, ep.abort, ep.status)) {
      for (int o = 0; o < ep.groups; ++o)
        if (o != ep.group) amax = max(amax, __float_as_uint(ep.xchg[o * BM + lane].x));
    }
    const bool grow = row_ok && s > 0.f && amax > static_cast<uint32_t>(kLimit);
    const float rho = grow ? __fdiv_rn(static_cast<float>(kLimit), __uint2float_rn(amax)) : 1.f;
    const PhiloxRoundKeys rk = philox_round_keys(a.key);
    __syncwarp();
#pragma unroll 1
    for (int c = c0; c < c0 + nchunk; ++c) {
      uint32_t U[32];
      tmem_ld_32x32b_x32(taddr + c * 32, U);
      uint32_t d[16];
      draws(a, rk, irow, j0 + c * 32, d);
      tmem_ld_wait(U);
      if (!lane_pred(row_ok)) continue;
      const uint4 wa = side_granule(side, row, 2 * c), wb = side_granule(side, row, 2 * c + 1);
      uint32_t out[8];
      if (lane_pred(grow))
        rescaled_chunk(U, wa, wb, d, cp, rho, out);
      else
        sr_chunk<true>(U, wa, wb, d, cp, cp, 32, out);
      store_chunk(wrow + c * 32, out);
    }
    if (grow && ep.group == 0) a.sW[g] = __fdiv_rn(s, rho);
  }
};

// ------------------------------------------------------------------ plain fp32 store

struct StoreF32Epi {
  static constexpr int kSideBytes = 0;
  static constexpr int kSideBufs = 1;
  static constexpr bool kExchange = false;
  static QG_DEV void issue_side(const CUtensorMap*, int, int, uint8_t*, uint64_t*) {}

  struct Args {
    float* D;
    int64_t ldd;
    int32_t accumulate;  // D += A B instead of D = A B
  };
  static QG_DEV void apply(const Args& a, int M, int N, int mb, int nb, int row, uint32_t taddr,
                           const EpiPair& ep, const uint8_t*) {
    const int grow = mb * BM + row;
    const bool ok = grow < M;
    const int j0 = nb * BN;
    const int ncols = min(BN, N - j0);
    const int nchunk = BN / 32 / ep.groups;
    const int c0 = ep.group * nchunk;
    const int c1 = min(c0 + nchunk, (ncols + 31) >> 5);
    __syncwarp();
    for (int c = c0; c < c1; ++c) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(taddr + c * 32, v);
      tmem_ld_wait(v);
      if (!lane_pred(ok)) continue;
      float* d = a.D + static_cast<int64_t>(grow) * a.ldd + j0 + c * 32;
      const int valid = ncols - c * 32;
      if (a.accumulate) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e < valid) d[e] = __fadd_rn(d[e], __uint_as_float(v[e]));
      } else if (valid >= 32) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          reinterpret_cast<float4*>(d)[q] =
              make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                          __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e < valid) d[e] = __uint_as_float(v[e]);
      }
    }
  }
};

// kernel parameters up to 32764 bytes (CUDA 12.1 and later on sm_70 and newer)
static_assert(sizeof(GemmParams<AdamEpi>) <= 32764, "kernel parameter block");
static_assert(sizeof(GemmParams<StochRoundEpi>) <= 32764, "kernel parameter block");
static_assert(sizeof(GemmParams<StochRoundRescaleEpi>) <= 32764, "kernel parameter block");
static_assert(sizeof(GemmParams<StoreF32Epi>) <= 32764, "kernel parameter block");

// ------------------------------------------------------------------ a1 and test kernels

// Eight INT4 codes (one 32-bit word, element 2i in the low nibble of byte i) ->
// eight bf16 of P~ = bf16_rn(code * scale), one 16-byte store.  One thread per
// word, kDqUnits words per thread a block apart, so that every warp-wide load
// covers 128 contiguous bytes and every store 512; the loads of a thread's
// words are issued together.  Each block works on one projection (found once
// per block from the prefix sums of the blocks per projection), with 32-bit
// indices inside it.  Every projection has m*r % 32 == 0 (r % 32 == 0), so a
// word stays inside one 64-element scale group (word i uses scale i / 8).  One
// launch covers up to kMaxProblems projections.  Nibbles become floats by
// exact integer/FP-add arithmetic (no conversion-pipe instructions), and pairs
// are rounded to bf16 together.  kVec: every code array 4-byte and every output
// 16-byte aligned.
constexpr int kDqThreads = 256;
constexpr int kDqUnits = 4;
constexpr int kDqBlockUnits = kDqThreads * kDqUnits;

struct DequantBatch {
  const uint8_t* Pq[kMaxProblems];
  const float* sP[kMaxProblems];
  uint16_t* out[kMaxProblems];
  int32_t units[kMaxProblems];              // m*r / 8 per projection
  int32_t block_begin[kMaxProblems + 1];    // prefix sums of the blocks per projection
  int32_t n;
};

QG_DEV uint4 dequant_word(uint32_t w, float s) {
  // nibble x ^ 8 is code + 8 in [0, 15]; the even and the odd nibbles are
  // spread one to a byte, and each byte placed below the bits of 1.5 * 2^23
  // (0x4B4000vv) is the float 1.5 * 2^23 + code + 8, exact; less that offset it
  // is the code, times the group's scale (round to nearest), two weights per
  // packed f32x2 instruction, then rounded to bf16 in pairs
  const uint32_t f = w ^ 0x88888888u;
  const uint32_t ev = f & 0x0F0F0F0Fu, od = (f >> 4) & 0x0F0F0F0Fu;  // elements 2h and 2h + 1 in byte h
  uint64_t sc;
  asm("mov.b64 %0, {%1, %1};" : "=l"(sc) : "f"(s));
  uint64_t off;
  asm("mov.b64 %0, {%1, %1};" : "=l"(off) : "r"(0x4B400008u));  // 1.5 * 2^23 + 8
  uint32_t out[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    uint64_t v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "r"(__byte_perm(ev, 0x4B400000u, 0x7640u | h)),
        "r"(__byte_perm(od, 0x4B400000u, 0x7640u | h)));
    asm("sub.rn.f32x2 %0, %0, %1;" : "+l"(v) : "l"(off));
    asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(v) : "l"(sc));
    uint32_t lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out[h]) : "r"(hi), "r"(lo));  // element 2h in the low half
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

template <bool kVec>
__global__ void __launch_bounds__(kDqThreads) dequant_projection_kernel(const __grid_constant__ DequantBatch b) {
  int p = 0;
  while (p + 1 < b.n && static_cast<int>(blockIdx.x) >= b.block_begin[p + 1]) ++p;
  const int units = b.units[p];
  const int first = (static_cast<int>(blockIdx.x) - b.block_begin[p]) * kDqBlockUnits + static_cast<int>(threadIdx.x);
  const uint8_t* src = b.Pq[p];
  const float* sp = b.sP[p];
  uint16_t* dst = b.out[p];
  uint32_t w[kDqUnits];
  float s[kDqUnits];
#pragma unroll
  for (int u = 0; u < kDqUnits; ++u) {
    const int i = first + u * kDqThreads;
    if (i >= units) continue;
    if (kVec) {
      w[u] = reinterpret_cast<const uint32_t*>(src)[i];
    } else {
      const uint8_t* q = src + 4 * static_cast<int64_t>(i);
      w[u] = static_cast<uint32_t>(q[0]) | (static_cast<uint32_t>(q[1]) << 8) | (static_cast<uint32_t>(q[2]) << 16) |
             (static_cast<uint32_t>(q[3]) << 24);
    }
    s[u] = sp[i >> 3];
  }
#pragma unroll
  for (int u = 0; u < kDqUnits; ++u) {
    const int i = first + u * kDqThreads;
    if (i >= units) continue;
    const uint4 v = dequant_word(w[u], s[u]);
    if (kVec) {
      reinterpret_cast<uint4*>(dst)[i] = v;
    } else {
      uint16_t* d = dst + 8 * static_cast<int64_t>(i);
      const uint32_t o[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        d[2 * h] = static_cast<uint16_t>(o[h] & 0xFFFFu);
        d[2 * h + 1] = static_cast<uint16_t>(o[h] >> 16);
      }
    }
  }
}

__global__ void philox_kernel(const uint32_t* c0, const uint32_t* c1, const uint32_t* c2, const uint32_t* c3,
                              int64_t count, PhiloxKey key, uint32_t* out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= count) return;
  uint32_t o[4];
  philox4x32_10(c0[i], c1[i], c2[i], c3[i], key, o);
  reinterpret_cast<uint4*>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
}

// ------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

static bool encode_map(void* map, CUtensorMapDataType dtype, uint32_t esize, const void* base, uint64_t inner,
                       uint64_t outer, uint64_t ld_elems, uint32_t box_inner, uint32_t box_outer) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {ld_elems * esize};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(reinterpret_cast<CUtensorMap*>(map), dtype, 2,
                              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_map_bf16(void* map, const void* base, uint64_t inner, uint64_t outer, uint64_t ld_elems,
                     uint32_t box_inner, uint32_t box_outer) {
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, inner, outer, ld_elems, box_inner, box_outer);
}

// int8 side tiles: boxes of 128 rows x 128 bytes, 128-byte swizzle
static bool encode_map_i8_side(void* map, const void* base, uint64_t inner, uint64_t outer, uint64_t ld_bytes) {
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, inner, outer, ld_bytes, 128, 128);
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

int64_t step_ldN(int32_t n) { return (static_cast<int64_t>(n) + 31) / 32 * 32; }

static size_t round256(size_t x) { return (x + 255) / 256 * 256; }

size_t step_scratch_bytes(int32_t m, int32_t n, int32_t r, int32_t side) {
  // P~ (rows of P x r), then N (R's shape: r x n, or m x r for the right side)
  const int32_t p_rows = side ? n : m, rows = side ? m : r, cols = side ? r : n;
  return round256(static_cast<size_t>(p_rows) * r * 2) + round256(static_cast<size_t>(rows) * step_ldN(cols) * 2);
}

template <class Epi, bool kAMN, bool kBMN>
static cudaError_t launch_gemm(const GemmParams<Epi>& p, cudaStream_t stream, int kind, double flops,
                               double bytes) {
  auto kern = gemm_tc_kernel<Epi, kAMN, kBMN>;
  static bool attr_set = false;  // per instantiation
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kGemmSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if (p.total_tiles == 0) return cudaSuccess;
  const int grid = std::min(p.total_tiles, sm_count());
  const int tok = profile_begin(stream, kind, flops, bytes);
  kern<<<grid, kGemmThreads, kGemmSmemBytes, stream>>>(p);
  profile_end(stream, tok);
  return cudaGetLastError();
}

// The same GEMMs on CTA pairs (256 x 256 tiles, cta_group::2).
template <class Epi, bool kAMN, bool kBMN = true>
static cudaError_t launch_gemm_pair(const GemmParams<Epi>& p, cudaStream_t stream, int kind, double flops,
                                    double bytes) {
  auto kern = gemm_tc_pair_kernel<Epi, kAMN, kBMN>;
  using L = typename PairCfg<Epi, kAMN, kBMN>::L;
  constexpr size_t kSmem = L::kSmemBytes;
  static bool attr_set = false;  // per instantiation
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int pair_tiles = 0;
  for (int i = 0; i < p.nprob; ++i) pair_tiles += ((p.prob[i].M + 255) / 256) * p.prob[i].tiles_n;
  if (pair_tiles == 0) return cudaSuccess;
  const int clusters = std::min(pair_tiles, std::max(1, sm_count() / 2));
  const int tok = profile_begin(stream, kind, flops, bytes);
  kern<<<2 * clusters, L::kThreads, kSmem, stream>>>(p);
  profile_end(stream, tok);
  return cudaGetLastError();
}

template <class Epi>
static void add_problem(GemmParams<Epi>& p, int M, int N, int K) {
  GemmProblem<Epi>& pr = p.prob[p.nprob];
  pr.M = M;
  pr.N = N;
  pr.K = K;
  pr.tiles_m = (M + BM - 1) / BM;
  pr.tiles_n = (N + BN - 1) / BN;
  pr.tile_begin = p.total_tiles;
  p.total_tiles += pr.tiles_m * pr.tiles_n;
  p.nprob += 1;
}

// Fills the per-projection unit counts' block prefix sums and launches.
static cudaError_t launch_dequant_batch(DequantBatch& b, cudaStream_t stream) {
  b.block_begin[0] = 0;
  double total = 0.0;
  for (int i = 0; i < b.n; ++i) {
    b.block_begin[i + 1] = b.block_begin[i] + (b.units[i] + kDqBlockUnits - 1) / kDqBlockUnits;
    total += b.units[i] * 8.0;
  }
  const int blocks = b.block_begin[b.n];
  if (blocks == 0) return cudaSuccess;
  const double bytes = total / 2.0 + total / 64.0 * 4.0 + total * 2.0;
  bool vec = true;
  for (int i = 0; i < b.n; ++i)
    vec = vec && (reinterpret_cast<uintptr_t>(b.Pq[i]) % 4 == 0) && (reinterpret_cast<uintptr_t>(b.out[i]) % 16 == 0);
  const int tok = profile_begin(stream, QG_KERNEL_DEQUANT, 0.0, bytes);
  if (vec)
    dequant_projection_kernel<true><<<static_cast<unsigned>(blocks), kDqThreads, 0, stream>>>(b);
  else
    dequant_projection_kernel<false><<<static_cast<unsigned>(blocks), kDqThreads, 0, stream>>>(b);
  profile_end(stream, tok);
  return cudaGetLastError();
}

cudaError_t launch_dequant_projection(const uint8_t* Pq, const float* sP, int64_t total, uint16_t* out,
                                      cudaStream_t stream) {
  if (total / 8 > INT32_MAX) return cudaErrorInvalidValue;
  DequantBatch b;
  memset(&b, 0, sizeof(b));
  b.Pq[0] = Pq;
  b.sP[0] = sP;
  b.out[0] = out;
  b.units[0] = static_cast<int32_t>(total / 8);
  b.n = 1;
  return launch_dequant_batch(b, stream);
}

cudaError_t launch_philox(const uint32_t* c0, const uint32_t* c1, const uint32_t* c2, const uint32_t* c3,
                          int64_t count, uint32_t k0, uint32_t k1, uint32_t* out, cudaStream_t stream) {
  if (count == 0) return cudaSuccess;
  const int threads = 256;
  philox_kernel<<<static_cast<unsigned>((count + threads - 1) / threads), threads, 0, stream>>>(
      c0, c1, c2, c3, count, PhiloxKey{k0, k1}, out);
  return cudaGetLastError();
}

static cudaError_t launch_dequant_for(const StepProblem* probs, int cnt, cudaStream_t stream) {
  DequantBatch db;
  memset(&db, 0, sizeof(db));
  for (int i = 0; i < cnt; ++i) {
    const StepProblem& s = probs[i];
    db.Pq[i] = s.Pq;
    db.sP[i] = s.sP;
    db.out[i] = s.Pbf;
    db.units[i] = static_cast<int32_t>(static_cast<int64_t>(s.side ? s.n : s.m) * s.r / 8);
  }
  db.n = cnt;
  return launch_dequant_batch(db, stream);
}

// a4+a5 for `cnt` problems of one projection side, all with the epilogue Epi
// (the saturating or the re-scaling stochastic rounding): one grid.
template <class Epi, bool kRight>
static cudaError_t launch_backproject(const StepProblem* probs, const int* idx, int cnt, cudaStream_t stream) {
  GemmParams<Epi> p2;
  memset(&p2, 0, sizeof(p2));
  double fl2 = 0, by2 = 0;
  // The batch's matrices in reverse order: the last N written by a2+a3 (and
  // its P~, read last there) is the likeliest still in L2.
  for (int jj = 0; jj < cnt; ++jj) {
#if QG_SR_REVERSE
    const int ii = cnt - 1 - jj;
#else
    const int ii = jj;
#endif
    const StepProblem& s = probs[idx[ii]];
    const double m = s.m, n = s.n, r = s.r;
    fl2 += 2 * m * n * r;
    // W read + written, W scales, P~, N
    by2 += 2 * m * n + 4 * std::ceil(m * n / 256.0) + 2 * (kRight ? n : m) * r + 2 * (kRight ? m : r) * (kRight ? r : n);
    GemmProblem<Epi>& pr = p2.prob[p2.nprob];
    if (kRight) {
      // A = N (M = m, K = r), K-major: box {64 (r), 128 (m)}
      if (!encode_map_bf16(&pr.tmA, s.Nbuf, s.r, s.m, s.ldN, 64, 128)) return cudaErrorInvalidValue;
      // B = P~^T (K = r, N = n), K-major over P~ (n x r): box {64 (r), 128 (n)}
      if (!encode_map_bf16(&pr.tmB, s.Pbf, s.r, s.n, s.r, 64, 128)) return cudaErrorInvalidValue;
    } else {
      // A = P~ (M = m, K = r), K-major: box {64 (r), 128 (m)}
      if (!encode_map_bf16(&pr.tmA, s.Pbf, s.r, s.m, s.r, 64, 128)) return cudaErrorInvalidValue;
      // B = N (K = r, N = n), MN-major: box {64 (n), 64 (r)}
      if (!encode_map_bf16(&pr.tmB, s.Nbuf, s.n, s.r, s.ldN, 64, 64)) return cudaErrorInvalidValue;
    }
    // side operand: W^Q (m x n int8, leading dimension ldw)
    if (!encode_map_i8_side(&pr.tmS[0], s.W, s.n, s.m, s.ldw)) return cudaErrorInvalidValue;
    pr.status = s.status;
    pr.epi = typename Epi::Args{s.W, s.sW, s.ldw, s.alpha, s.t, s.layer_id,
                                PhiloxKey{static_cast<uint32_t>(s.seed), static_cast<uint32_t>(s.seed >> 32)},
                                (s.n % 256) == 0 ? 1 : 0};
    add_problem(p2, s.m, s.n, s.r);
  }
  return launch_gemm_pair<Epi, false, !kRight>(p2, stream, QG_KERNEL_BACKPROJECT_SR, fl2, by2);
}

// a2+a3 and a4+a5 for the problems of one projection side (kRight: P n x r,
// R = G P, U = N P^T; otherwise P m x r, R = P^T G, U = P N): one grid each.
template <bool kRight>
static cudaError_t launch_gemms_side(const StepProblem* probs, const int* idx, int cnt, cudaStream_t stream) {
  cudaError_t e;
  GemmParams<AdamEpi> p1;
  memset(&p1, 0, sizeof(p1));
  double fl1 = 0, by1 = 0;
  for (int ii = 0; ii < cnt; ++ii) {
    const StepProblem& s = probs[idx[ii]];
    const double m = s.m, n = s.n, r = s.r;
    const double p_rows = kRight ? n : m, rows = kRight ? m : r, cols = kRight ? r : n;
    fl1 += 2 * m * n * r;
    // a2+a3: G, P~, moments read + written, their scales, N written
    by1 += 2 * m * n + 2 * p_rows * r + 4 * rows * cols + 16.0 * rows * s.nblk + 2 * rows * cols;
    GemmProblem<AdamEpi>& pr = p1.prob[p1.nprob];
    if (kRight) {
      // A = G (M = m, K = n), K-major: box {64 (n), 128 (m)}
      if (!encode_map_bf16(&pr.tmA, s.G, s.n, s.m, s.ldg, 64, 128)) return cudaErrorInvalidValue;
      // B = P~ (K = n, N = r), MN-major: box {64 (r), 64 (n)}
      if (!encode_map_bf16(&pr.tmB, s.Pbf, s.r, s.n, s.r, 64, 64)) return cudaErrorInvalidValue;
      // side operands: M^Q and V^Q (m x r int8)
      if (!encode_map_i8_side(&pr.tmS[0], s.Mq, s.r, s.m, s.ld_mom)) return cudaErrorInvalidValue;
      if (!encode_map_i8_side(&pr.tmS[1], s.Vq, s.r, s.m, s.ld_mom)) return cudaErrorInvalidValue;
    } else {
      // both operands MN-major: boxes of kPairBKMN rows of K
      constexpr uint32_t kBKb = AdamEpi::kPairBKMN;
      // A = P~^T (M = r, K = m), MN-major over P~ (m x r): box {64 (r), kBK (m)}
      if (!encode_map_bf16(&pr.tmA, s.Pbf, s.r, s.m, s.r, 64, kBKb)) return cudaErrorInvalidValue;
      // B = G (K = m, N = n), MN-major: box {64 (n), kBK (m)}
      if (!encode_map_bf16(&pr.tmB, s.G, s.n, s.m, s.ldg, 64, kBKb)) return cudaErrorInvalidValue;
      // side operands: M^Q and V^Q (r x n int8, leading dimension ld_mom)
      if (!encode_map_i8_side(&pr.tmS[0], s.Mq, s.n, s.r, s.ld_mom)) return cudaErrorInvalidValue;
      if (!encode_map_i8_side(&pr.tmS[1], s.Vq, s.n, s.r, s.ld_mom)) return cudaErrorInvalidValue;
    }
    pr.status = s.status;
    pr.epi = AdamEpi::Args{s.Mq, s.Vq, s.sM, s.sV, s.Nbuf, s.ld_mom, s.ldN, s.nblk,
                           s.beta1, s.beta2, s.om1, s.om2, s.c1, s.c2, s.eps};
    if (kRight)
      add_problem(p1, s.m, s.r, s.n);
    else
      add_problem(p1, s.r, s.n, s.m);
  }
  e = launch_gemm_pair<AdamEpi, !kRight>(p1, stream, QG_KERNEL_PROJECT_ADAM, fl1, by1);
  if (e != cudaSuccess) return e;
  // a4+a5: the saturating problems in one grid, the re-scaling ones in another
  int sat[kMaxProblems], grow[kMaxProblems], ns = 0, ng = 0;
  for (int ii = 0; ii < cnt; ++ii) {
    if (probs[idx[ii]].w_rescale)
      grow[ng++] = idx[ii];
    else
      sat[ns++] = idx[ii];
  }
  if (ns > 0 && (e = launch_backproject<StochRoundEpi, kRight>(probs, sat, ns, stream)) != cudaSuccess) return e;
  if (ng > 0) e = launch_backproject<StochRoundRescaleEpi, kRight>(probs, grow, ng, stream);
  return e;
}

// The batch's left-side problems, then its right-side ones.
static cudaError_t launch_gemms_for(const StepProblem* probs, int cnt, cudaStream_t stream) {
  int left[kMaxProblems], right[kMaxProblems], nl = 0, nr = 0;
  for (int i = 0; i < cnt; ++i) {
    if (probs[i].side)
      right[nr++] = i;
    else
      left[nl++] = i;
  }
  cudaError_t e = cudaSuccess;
  if (nl > 0 && (e = launch_gemms_side<false>(probs, left, nl, stream)) != cudaSuccess) return e;
  if (nr > 0) e = launch_gemms_side<true>(probs, right, nr, stream);
  return e;
}

cudaError_t launch_step(const StepProblem* probs, int count, cudaStream_t stream) {
  for (int base = 0; base < count; base += kMaxProblems) {
    const int cnt = std::min(kMaxProblems, count - base);
    cudaError_t e = launch_dequant_for(probs + base, cnt, stream);
    if (e != cudaSuccess) return e;
    e = launch_gemms_for(probs + base, cnt, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_gemm_f32(const void* A, int64_t lda, bool a_trans, const void* B, int64_t ldb, bool b_trans,
                            float* D, int64_t ldd, int M, int N, int K, cudaStream_t stream, bool accumulate) {
  GemmParams<StoreF32Epi> p;
  memset(&p, 0, sizeof(p));
  GemmProblem<StoreF32Epi>& pr = p.prob[0];
  // A: a_trans = 0 -> given M x K row-major (K-major operand, box {64, 128});
  //    a_trans = 1 -> given K x M row-major (MN-major operand, box {64, 64}).
  const bool okA = a_trans ? encode_map_bf16(&pr.tmA, A, M, K, lda, 64, 64)
                           : encode_map_bf16(&pr.tmA, A, K, M, lda, 64, 128);
  // B: b_trans = 0 -> given K x N row-major (MN-major, box {64, 64});
  //    b_trans = 1 -> given N x K row-major (K-major, box {64, 256}).
  const bool okB = b_trans ? encode_map_bf16(&pr.tmB, B, K, N, ldb, 64, 256)
                           : encode_map_bf16(&pr.tmB, B, N, K, ldb, 64, 64);
  if (!okA || !okB) return cudaErrorInvalidValue;
  pr.status = nullptr;
  pr.epi = StoreF32Epi::Args{D, ldd, accumulate ? 1 : 0};
  add_problem(p, M, N, K);
  const double fl = 2.0 * M * N * K, by = 2.0 * M * K + 2.0 * K * N + 4.0 * M * N;
  if (a_trans && b_trans) return launch_gemm<StoreF32Epi, true, false>(p, stream, QG_KERNEL_OTHER, fl, by);
  if (a_trans) return launch_gemm<StoreF32Epi, true, true>(p, stream, QG_KERNEL_OTHER, fl, by);
  if (b_trans) return launch_gemm<StoreF32Epi, false, false>(p, stream, QG_KERNEL_OTHER, fl, by);
  return launch_gemm<StoreF32Epi, false, true>(p, stream, QG_KERNEL_OTHER, fl, by);
}

}  // namespace qg
