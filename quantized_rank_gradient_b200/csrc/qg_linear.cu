// Linear layers with INT8 weights on sm_100a: the forward and backward matrix
// products around the optimizer step (AIMech Q-GaLore page, limitation
// "simulated weight-quantization throughput", paper section 3.2 and section
// 4.4, Fig. 4: activations stay in 16-bit floating point and the INT8 weights
// are dequantized for the forward and backward products; same page, Theorem
// 3.1, paper section 3.1: the weight gradient of y = W x is G = (1/B) D_y X^T).
//
//   W~ = bf16(fp32(q) * s_W[(i n + j) / 256])          dequant_weight_kernel
//   Y  = X W~^T        (T x m)                          tcgen05 pair GEMM, A and B K-major
//   dX = D_y W~        (T x n)                          tcgen05 pair GEMM, B MN-major
//   G  = D_y^T X       (m x n, the optimizer's input)   tcgen05 pair GEMM, A and B MN-major
//
// W~ is formed once per optimizer step into a bf16 scratch and read by the
// forward and the data-gradient product: at training batch sizes those GEMMs
// are bound by the tensor cores, and converting W inside every GEMM tile would
// repeat the conversion once per 128-row tile of activations on the same
// schedulers that issue the MMAs, while the separate pass costs three bytes of
// HBM traffic per weight.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "../../include/qgalore.h"
#include "qg_gemm.cuh"
#include "qg_internal.h"

namespace qg {

namespace {

// ---------------------------------------------------------------- W~ = bf16(q * s)

// Byte k (0..3) of w as a signed integer, converted to float exactly without the
// conversion unit: the sign-extended byte added to the bits of 1.5 * 2^23 gives
// the float 1.5 * 2^23 + byte (exact for |byte| < 2^22), less 1.5 * 2^23.
QG_DEV float sbyte_f32(uint32_t w, int k) {
  const uint32_t sel = k | ((k | 8) << 4) | ((k | 8) << 8) | ((k | 8) << 12);
  uint32_t sx;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(sx) : "r"(w), "r"(0u), "r"(sel));
  return __fsub_rn(__uint_as_float(0x4B400000u + sx), 12582912.0f);
}

// Sixteen consecutive elements of a row of W (row stride ldw bytes, ldw % 16 ==
// 0) per chunk: the group of element (i, j) is (i n + j) / 256, so sixteen
// elements span at most two groups.  One float32 product, rounded to bf16.
QG_DEV void dequant_chunk(const uint4& q, int64_t i, int j0, int32_t n, const float* __restrict__ sW,
                          uint16_t* __restrict__ Wt, int64_t ldt) {
  const int64_t e0 = i * n + j0;
  const int valid = min(16, n - j0);
  const int64_t g0 = e0 >> 8, g1 = (e0 + valid - 1) >> 8;
  const float s0 = __ldg(sW + g0), s1 = __ldg(sW + g1);
  const int split = g1 != g0 ? static_cast<int>((g1 << 8) - e0) : 16;
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  uint32_t out[8];
#pragma unroll
  for (int k = 0; k < 16; k += 2) {
    const float a = __fmul_rn(sbyte_f32(w[k >> 2], k & 3), k < split ? s0 : s1);
    const float b = __fmul_rn(sbyte_f32(w[k >> 2], (k + 1) & 3), k + 1 < split ? s0 : s1);
    const __nv_bfloat162 p2 = __floats2bfloat162_rn(a, b);  // a in the low half
    out[k >> 1] = *reinterpret_cast<const uint32_t*>(&p2);
  }
  uint16_t* dst = Wt + i * ldt + j0;
  if (valid == 16) {
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(out[0], out[1], out[2], out[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(out[4], out[5], out[6], out[7]);
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k)
      if (k < valid) dst[k] = static_cast<uint16_t>(out[k >> 1] >> (16 * (k & 1)));
  }
}

// A grid-stride loop over groups of kDqChunks chunks per thread, all of whose
// loads are issued before the first conversion (more bytes in flight per SM).
constexpr int kDqChunks = 4;

__global__ void __launch_bounds__(256) dequant_weight_kernel(const int8_t* __restrict__ W, int64_t ldw,
                                                             const float* __restrict__ sW, int32_t m, int32_t n,
                                                             uint16_t* __restrict__ Wt, int64_t ldt) {
  const int64_t chunks = (n + 15) / 16;
  const int64_t total = static_cast<int64_t>(m) * chunks;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t c0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c0 < total;
       c0 += stride * kDqChunks) {
    uint4 q[kDqChunks];
#pragma unroll
    for (int u = 0; u < kDqChunks; ++u) {
      const int64_t c = c0 + u * stride;
      if (c < total) q[u] = __ldg(reinterpret_cast<const uint4*>(W + (c / chunks) * ldw + (c % chunks) * 16));
    }
#pragma unroll
    for (int u = 0; u < kDqChunks; ++u) {
      const int64_t c = c0 + u * stride;
      if (c < total) dequant_chunk(q[u], c / chunks, static_cast<int>(c % chunks) * 16, n, sW, Wt, ldt);
    }
  }
}

// ---------------------------------------------------------------- Y = X W~^T for a few tokens, W read once

// For T <= 64 tokens the forward product is bound by reading the weight: the
// separate dequantization moves three bytes per weight and the GEMM two more,
// where this kernel reads the INT8 codes once and forms W~ = bf16(fp32(q) * s)
// in registers, rounded exactly as dequant_weight_kernel rounds it.
//
// Work split.  A CTA owns kF8Rows rows of W and one slice of its columns; the
// S slices of one row block form a thread-block cluster (split K), sized so
// that the clusters fit the GPU at once.  The partial sums are added across
// the cluster through distributed shared memory in the order of the CTA ranks,
// so every output is the same sum whichever CTA adds it, rounded once to bf16.
//
// Data movement.  One producer thread streams the slice through a ring of
// f8_stages shared-memory stages by TMA, 256 columns a stage; per 128 columns
// the W box (64 rows x 128 bytes) and the X boxes (8, 16, 32 or 64 token rows
// x 64 columns, two), all with the 128-byte swizzle.  Rows past m or T and columns
// past n arrive as zeros, and the bytes in flight cost no registers.  Wider
// stages halve the consumers' per-stage work (waits, arrivals, addresses,
// scales) per weight.
//
// Arithmetic.  Four consumer warps own 16 rows each.  The product runs on the
// tensor cores with mma.sync m16n8k16 (bf16 in, f32 accumulate), whose A
// operand comes from registers: the dequantized weight goes from the
// conversion straight into the fragment.  Any bijection of a stage's columns
// onto k-positions gives the same sum.  In step s (two per 128 columns) the
// lane with thread-in-group t takes the 16 columns of chunk w = 2t + (s ^ (t >>
// 1)) (16 columns, 16 bytes of W); in MMA j its k-pairs (2t, 2t+1) and (2t+8, 2t+9)
// are columns 4j + {0, 1} and 4j + {2, 3} of those 16, and the B fragment of
// token g is the eight bytes of X there.  With this order the eight lanes of a
// quarter warp read eight distinct 16-byte bank groups of the swizzled W tile
// (distinct w >> 1, two rows) and of the X tile (distinct w & 3, two tokens).
// At 2T <= 128 flops per weight byte the work is bound by HBM; the tensor cores
// keep the multiply-adds off the schedulers, which the conversion occupies
// (about 2.75 instructions a weight).  The kernel is launched with
// programmatic stream serialization, so that its launch and set-up overlap the
// end of the kernel before it in the stream.
constexpr int kF8Warps = 4;                        // consumer warps, 16 rows each
constexpr int kF8Rows = 16 * kF8Warps;             // rows of W per CTA
constexpr int kF8Threads = 32 * (kF8Warps + 1);    // + the producer warp
constexpr int kF8Tile = 128;                       // columns per TMA box of W (128 bytes)
constexpr int kF8Halves = 2;                       // W boxes per ring stage
constexpr int kF8StageCols = kF8Tile * kF8Halves;  // columns per ring stage
constexpr int kF8WBytes = kF8Rows * kF8Tile;       // W box: 8 KB
// ring depth in stages of 256 columns: three up to 32 tokens (60, 72 and 96 KB
// with the X boxes of 8, 16 and 32 tokens: three, three and two CTAs a SM), two
// for 64 tokens (96 KB, two CTAs a SM).  Two stages for 16 tokens (four CTAs a
// SM) ran each matrix shape alone slightly faster, but the mixed sequence of a
// decoder stack 9 % slower.
template <int kNT>
__host__ __device__ constexpr int f8_stages() {
  return kNT >= 8 ? 2 : 3;
}
constexpr int kF8MaxCluster = 8;                   // portable cluster size

// X tile of a stage: kNT * 8 token rows x 128 columns of bf16, two 64-column boxes
template <int kNT>
__host__ __device__ constexpr int f8_xbox_bytes() {
  return kNT * 8 * 128;
}

// a stage: per 128 columns, the W box and the two X boxes; a multiple of 1024
// bytes (the swizzle atom), as is every box in it
template <int kNT>
__host__ __device__ constexpr int f8_half_bytes() {
  return kF8WBytes + 2 * f8_xbox_bytes<kNT>();
}

template <int kNT>
__host__ __device__ constexpr int f8_stage_bytes() {
  return kF8Halves * f8_half_bytes<kNT>();
}

template <int kNT>
__host__ __device__ constexpr int f8_smem_bytes() {
  return 1024 + f8_stages<kNT>() * f8_stage_bytes<kNT>();  // + alignment slack for the ring
}

// CTAs per SM for the register budget: at most 136 registers a thread up to 16
// tokens, 204 beyond (the accumulators grow with the tokens)
template <int kNT>
__host__ __device__ constexpr int f8_ctas_per_sm() {
  return kNT <= 2 ? 3 : 2;
}

// barrier among the consumer warps only
QG_DEV void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kF8Warps) : "memory"); }

QG_DEV float ld_shared_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

QG_DEV uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

QG_DEV void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                           uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

QG_DEV uint64_t pack_f32x2(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}

// Four weights (the bytes of a word of codes, lowest first) as two bf16 pairs,
// each bf16(fp32(q) * s) with its own scale (sc01: weights 0, 1; sc23: 2, 3).
// The codes biased by 128 (q ^ 0x80 as unsigned bytes u) are placed in the low
// mantissa bits of 2^23 (the float 2^23 + u, exact); less 2^23 + 128 they are q
// exactly; the products with the scales round to nearest in float32; each pair
// is then rounded to bf16 (nearest even), the lower column in the low half.
// Packed f32x2 arithmetic, two weights per instruction.
QG_DEV void w_tilde4(uint32_t word, uint64_t sc01, uint64_t sc23, uint32_t& p01, uint32_t& p23) {
  const uint32_t biased = word ^ 0x80808080u;
  uint64_t v01 = pack_f32x2(__byte_perm(biased, 0x4B000000u, 0x7540u), __byte_perm(biased, 0x4B000000u, 0x7541u));
  uint64_t v23 = pack_f32x2(__byte_perm(biased, 0x4B000000u, 0x7542u), __byte_perm(biased, 0x4B000000u, 0x7543u));
  const uint64_t offset = pack_f32x2(0x4B000080u, 0x4B000080u);  // 2^23 + 128
  asm("sub.rn.f32x2 %0, %0, %1;" : "+l"(v01) : "l"(offset));
  asm("sub.rn.f32x2 %0, %0, %1;" : "+l"(v23) : "l"(offset));
  asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(v01) : "l"(sc01));
  asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(v23) : "l"(sc23));
  uint32_t a, b, c, d;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(v01));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(c), "=r"(d) : "l"(v23));
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(p01) : "r"(b), "r"(a));
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(p23) : "r"(d), "r"(c));
}

// W~ of sixteen consecutive weights as eight bf16 pairs: weights k < split
// take scale s0, the others s1 (kOneGroup: all take s1).
template <bool kOneGroup>
QG_DEV void w_tilde16(const uint4& q, float s0, float s1, int split, uint32_t (&out)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  const uint64_t one = pack_f32x2(__float_as_uint(s1), __float_as_uint(s1));
#pragma unroll
  for (int k = 0; k < 16; k += 4) {
    uint64_t sc01 = one, sc23 = one;
    if (!kOneGroup) {
      sc01 = pack_f32x2(__float_as_uint(k < split ? s0 : s1), __float_as_uint(k + 1 < split ? s0 : s1));
      sc23 = pack_f32x2(__float_as_uint(k + 2 < split ? s0 : s1), __float_as_uint(k + 3 < split ? s0 : s1));
    }
    w_tilde4(w[k >> 2], sc01, sc23, out[k >> 1], out[(k >> 1) + 1]);
  }
}

// The scales of sixteen consecutive weights of row i (columns j0..j0+15) when
// n is not a multiple of 256: weights k < split take s0, the others s1
// (split <= 0: one group).  Columns at or past n take the group of the row's
// last weight (their codes arrive as zeros), so every index stays inside s_W.
struct Scales16 {
  float s0, s1;
  int split;
};

QG_DEV Scales16 scales16(int64_t i, int j0, int32_t n, const float* __restrict__ sW) {
  const int64_t e0 = i * n + j0;
  const int64_t g0 = (i * n + min(j0, n - 1)) >> 8, g1 = (i * n + min(j0 + 15, n - 1)) >> 8;
  Scales16 r;
  r.s1 = __ldg(sW + g1);
  r.s0 = g1 != g0 ? __ldg(sW + g0) : r.s1;
  r.split = static_cast<int>((g1 << 8) - e0);
  return r;
}

// The four MMAs of a step on two accumulator sets (MMAs 0, 1 and 2, 3), so
// that the chain of dependent MMAs is half as long.  x0, x1: this lane's two
// 8-column chunks of X in the step, for tokens g (+ 8 nt).
template <int kNT>
QG_DEV void f8_mma(const uint32_t (&wa)[8], const uint32_t (&wb)[8], const uint4 (&x0)[kNT], const uint4 (&x1)[kNT],
                   float (&acc)[2][kNT][4]) {
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt) {
    mma_bf16_16816(acc[0][nt], wa[0], wb[0], wa[1], wb[1], x0[nt].x, x0[nt].y);
    mma_bf16_16816(acc[0][nt], wa[2], wb[2], wa[3], wb[3], x0[nt].z, x0[nt].w);
    mma_bf16_16816(acc[1][nt], wa[4], wb[4], wa[5], wb[5], x1[nt].x, x1[nt].y);
    mma_bf16_16816(acc[1][nt], wa[6], wb[6], wa[7], wb[7], x1[nt].z, x1[nt].w);
  }
}

// Grid: one CTA per (row block, column slice), blockIdx.x = block * S + slice,
// launched in clusters of S along x; slice is a multiple of kF8StageCols (and
// of 256 when kGroupRows: n % 256 == 0, so that a group of 256 columns of a row
// lies in one scale group).
template <int kNT, bool kGroupRows>
__global__ void __launch_bounds__(kF8Threads, f8_ctas_per_sm<kNT>()) linear_forward_int8_kernel(
    const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, const float* __restrict__ sW,
    int32_t T, int32_t m, int32_t n, int32_t slice, uint16_t* __restrict__ Y, int64_t ldy) {
  constexpr int kStage = f8_stage_bytes<kNT>();
  constexpr int kXBox = f8_xbox_bytes<kNT>();
  constexpr int kF8Stages = f8_stages<kNT>();
  extern __shared__ uint8_t f8_smem[];
  __shared__ uint64_t full[kF8Stages], empty[kF8Stages];
  __shared__ int abort_flag;
  uint8_t* ring = f8_smem + ((1024 - (smem_u32(f8_smem) & 1023)) & 1023);
  // this CTA's partial sums, [token][row], in the ring once every stage is read
  // (the same offset in every CTA of the cluster)
  float (*red)[kF8Rows] = reinterpret_cast<float (*)[kF8Rows]>(ring);
  static_assert(kNT * 8 * kF8Rows * 4 <= kF8Stages * kStage, "partial sums fit in the ring");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = static_cast<int>(cluster_nctarank());
  const int rank = static_cast<int>(cluster_ctarank());
  const int block = blockIdx.x / S;
  const int kbeg = rank * slice, kend = min(n, kbeg + slice);
  const int nstage = (kend - kbeg + kF8StageCols - 1) / kF8StageCols;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kF8Stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kF8Warps);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // launched with programmatic stream serialization: the set-up above may overlap
  // the end of the preceding kernel, whose writes (X, W, the scales) are visible
  // after this wait; every global access of this kernel comes after it
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == kF8Warps) {
    // producer: one thread streams the slice's stages (W tile, two X boxes) through the ring
    if (lane == 0) {
      tma_prefetch_map(&tmW);
      tma_prefetch_map(&tmX);
      int issued = 0;
      for (int k = 0; k < nstage; ++k) {
        const int slot = k % kF8Stages;
        if (k >= kF8Stages && !mbar_wait(&empty[slot], ((k / kF8Stages) - 1) & 1, &abort_flag, nullptr)) break;
        uint8_t* st = ring + slot * kStage;
        mbar_arrive_expect_tx(&full[slot], kStage);
#pragma unroll
        for (int h = 0; h < kF8Halves; ++h) {
          uint8_t* sh = st + h * f8_half_bytes<kNT>();
          const int col = kbeg + k * kF8StageCols + h * kF8Tile;
          tma_load_2d(sh, &tmW, &full[slot], col, block * kF8Rows);
          tma_load_2d(sh + kF8WBytes, &tmX, &full[slot], col, 0);
          tma_load_2d(sh + kF8WBytes + kXBox, &tmX, &full[slot], col + 64, 0);
        }
        issued = k + 1;
      }
      // every load issued has landed before the CTA can leave (bounded)
      for (int k = max(0, issued - kF8Stages); k < issued; ++k)
        mbar_wait_drain(&full[k % kF8Stages], (k / kF8Stages) & 1);
    }
    __syncwarp();
  } else {
    const int g = lane >> 2, t = lane & 3;
    const int r0 = warp * 16 + g;  // fragment rows r0 and r0 + 8 of the CTA's block
    const int64_t ra = static_cast<int64_t>(block) * kF8Rows + r0, rb = ra + 8;
    const int64_t ia = ra < m ? ra : 0, ib = rb < m ? rb : 0;  // rows past m: zero codes, row 0's scales
    const float* srow_a = sW + (kGroupRows ? ia * (n >> 8) : 0);
    const float* srow_b = sW + (kGroupRows ? ib * (n >> 8) : 0);
    // per step s: the lane's chunk w (16 columns), its swizzled W offset in rows
    // r0 and r0 + 8 (same row & 7), and its two 8-column X chunks (token g)
    int woff[2], xoff0[2], xoff1[2], wcol[2];
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int w = 2 * t + (s ^ (t >> 1));
      wcol[s] = 16 * w;
      woff[s] = r0 * kF8Tile + ((w ^ (r0 & 7)) << 4);
      const int xb = kF8WBytes + (w >> 2) * kXBox + g * 128, c = 2 * (w & 3);
      xoff0[s] = xb + ((c ^ (g & 7)) << 4);
      xoff1[s] = xb + (((c + 1) ^ (g & 7)) << 4);
    }
    float acc[2][kNT][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) acc[h][nt][0] = acc[h][nt][1] = acc[h][nt][2] = acc[h][nt][3] = 0.f;
    // kGroupRows: the scales of the current and the next group of 256 columns (one per row)
    constexpr int kStagesPerGroup = 256 / kF8StageCols;
    float sa = 0.f, sb = 0.f, na = 0.f, nb = 0.f;
    if (kGroupRows) {
      na = __ldg(srow_a + (kbeg >> 8));
      nb = __ldg(srow_b + (kbeg >> 8));
    }
    // after a timed-out wait (abort) the loop does no more work
    bool ok = true;
    for (int k = 0; k < nstage && ok; ++k) {
      const int col0 = kbeg + k * kF8StageCols;
      if (kGroupRows && k % kStagesPerGroup == 0) {
        sa = na;
        sb = nb;
        if (k + kStagesPerGroup < nstage) {
          na = __ldg(srow_a + ((col0 + 256) >> 8));
          nb = __ldg(srow_b + ((col0 + 256) >> 8));
        }
      }
      const int slot = k % kF8Stages;
      // a warp vote, so that the lanes of a warp agree even when a wait times out
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&full[slot], (k / kF8Stages) & 1, &abort_flag, nullptr));
      if (!ok) break;
      const uint8_t* st = ring + slot * kStage;
#pragma unroll
      for (int h = 0; h < kF8Halves; ++h) {
        const uint8_t* sh = st + h * f8_half_bytes<kNT>();
        const int col = col0 + h * kF8Tile;
        // W (and, up to 16 tokens, X) of this half in registers; with more tokens X is
        // read per step, and the stage is released after its last half
        constexpr bool kPrefetchX = kNT <= 2;
        constexpr int kXN = kPrefetchX ? kNT : 1;
        uint4 qa[2], qb[2], x0[2][kXN], x1[2][kXN];
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          qa[s] = *reinterpret_cast<const uint4*>(sh + woff[s]);
          qb[s] = *reinterpret_cast<const uint4*>(sh + woff[s] + 8 * kF8Tile);
          if constexpr (kPrefetchX) {
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt) {
              x0[s][nt] = *reinterpret_cast<const uint4*>(sh + xoff0[s] + nt * 8 * 128);
              x1[s][nt] = *reinterpret_cast<const uint4*>(sh + xoff1[s] + nt * 8 * 128);
            }
          }
        }
        if (kPrefetchX && h == kF8Halves - 1) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[slot]);  // the stage is in registers
        }
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          uint32_t wa[8], wb[8];
          if constexpr (kGroupRows) {
            w_tilde16<true>(qa[s], 0.f, sa, 0, wa);
            w_tilde16<true>(qb[s], 0.f, sb, 0, wb);
          } else {
            const int j0 = col + wcol[s];
            const Scales16 za = scales16(ia, j0, n, sW), zb = scales16(ib, j0, n, sW);
            // a warp vote: every lane takes the same path to the MMAs
            if (__all_sync(0xFFFFFFFFu, za.split <= 0 && zb.split <= 0)) {
              w_tilde16<true>(qa[s], 0.f, za.s1, 0, wa);
              w_tilde16<true>(qb[s], 0.f, zb.s1, 0, wb);
            } else {
              w_tilde16<false>(qa[s], za.s0, za.s1, za.split, wa);
              w_tilde16<false>(qb[s], zb.s0, zb.s1, zb.split, wb);
            }
          }
          if constexpr (kPrefetchX) {
            f8_mma<kNT>(wa, wb, x0[s], x1[s], acc);
          } else {
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt) {
              const uint4 y0 = *reinterpret_cast<const uint4*>(sh + xoff0[s] + nt * 8 * 128);
              const uint4 y1 = *reinterpret_cast<const uint4*>(sh + xoff1[s] + nt * 8 * 128);
              mma_bf16_16816(acc[0][nt], wa[0], wb[0], wa[1], wb[1], y0.x, y0.y);
              mma_bf16_16816(acc[0][nt], wa[2], wb[2], wa[3], wb[3], y0.z, y0.w);
              mma_bf16_16816(acc[1][nt], wa[4], wb[4], wa[5], wb[5], y1.x, y1.y);
              mma_bf16_16816(acc[1][nt], wa[6], wb[6], wa[7], wb[7], y1.z, y1.w);
            }
          }
        }
        if (!kPrefetchX && h == kF8Halves - 1) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[slot]);  // every read of the stage is done
        }
      }
    }
    // partial sums: lane (g, t) holds rows r0 and r0 + 8, tokens 2t, 2t + 1 of each 8;
    // they overwrite the ring once every consumer warp has read its last stage (all
    // the producer's loads have landed by then: each was waited for)
    consumers_sync();
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      const int tok = nt * 8 + 2 * t;
      red[tok][r0] = __fadd_rn(acc[0][nt][0], acc[1][nt][0]);
      red[tok + 1][r0] = __fadd_rn(acc[0][nt][1], acc[1][nt][1]);
      red[tok][r0 + 8] = __fadd_rn(acc[0][nt][2], acc[1][nt][2]);
      red[tok + 1][r0 + 8] = __fadd_rn(acc[0][nt][3], acc[1][nt][3]);
    }
  }
  // the next kernel in the stream may launch now (its own wait orders it after this one)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  cluster_sync();  // every CTA's partial sums are written
  constexpr int kOut = kNT * 8 * kF8Rows;
  const int o0 = rank * kOut / S, o1 = (rank + 1) * kOut / S;
  for (int o = o0 + static_cast<int>(threadIdx.x); o < o1; o += kF8Threads) {
    const int tok = o / kF8Rows, row = o % kF8Rows;
    const int64_t i = static_cast<int64_t>(block) * kF8Rows + row;
    if (tok < T && i < m) {
      const float* mine = &red[0][0] + o;
      float part[kF8MaxCluster];
#pragma unroll
      for (int q = 0; q < kF8MaxCluster; ++q) part[q] = q < S ? ld_shared_cluster_f32(mapa_shared(mine, q)) : 0.f;
      float v = part[0];
#pragma unroll
      for (int q = 1; q < kF8MaxCluster; ++q)
        if (q < S) v = __fadd_rn(v, part[q]);
      Y[static_cast<int64_t>(tok) * ldy + i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
  }
  cluster_sync();  // no CTA leaves while another reads its partial sums
}

// Column slices per row block: as many as keep all clusters resident at once
// (the occupancy query, for each cluster size from the largest down), at most
// a portable cluster, each a multiple of kF8StageCols columns (and of 256
// when n % 256 == 0).
struct F8Split {
  int S, slice, blocks;
};

F8Split forward_int8_split(int32_t m, int32_t n, const int (&clusters_fit)[kF8MaxCluster + 1]) {
  F8Split f;
  f.blocks = (m + kF8Rows - 1) / kF8Rows;
  const int unit = std::max(n % 256 == 0 ? 256 : kF8Tile, kF8StageCols);
  int S = std::max(1, std::min(kF8MaxCluster, (n + unit - 1) / unit));
  while (S > 1 && f.blocks > clusters_fit[S]) --S;
  f.slice = ((n + S - 1) / S + unit - 1) / unit * unit;
  f.S = (n + f.slice - 1) / f.slice;  // no empty slice
  return f;
}

// A row-major 2-D tensor (rows x cols elements of esize bytes, row stride ld
// elements) as TMA boxes of box_rows x box_cols, 128-byte swizzle; rows and
// columns past the edge read as zeros.
PFN_cuTensorMapEncodeTiled_v12000 f8_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_rows(CUtensorMap* map, CUtensorMapDataType dtype, int esize, const void* base, int64_t ld, int64_t rows,
                 int64_t cols, int box_rows, int box_cols) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = f8_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * esize)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per instantiation: the dynamic shared memory attribute, and how many
// clusters of each size fit on the device at once.
template <int kNT, bool kGroupRows>
struct F8Kernel {
  cudaError_t err = cudaSuccess;
  int fit[kF8MaxCluster + 1] = {};
  F8Kernel() {
    const auto kern = linear_forward_int8_kernel<kNT, kGroupRows>;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, f8_smem_bytes<kNT>());
    for (int S = 1; S <= kF8MaxCluster && err == cudaSuccess; ++S) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(S));
      cfg.blockDim = dim3(kF8Threads);
      cfg.dynamicSmemBytes = static_cast<size_t>(f8_smem_bytes<kNT>());
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = static_cast<unsigned>(S);
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      err = cudaOccupancyMaxActiveClusters(&fit[S], kern, &cfg);
    }
  }
};

template <int kNT, bool kGroupRows>
cudaError_t launch_forward_int8_as(const CUtensorMap& tmW, const uint16_t* X, int64_t ldx, const float* sW, int T,
                                   int m, int n, uint16_t* Y, int64_t ldy, cudaStream_t s) {
  static F8Kernel<kNT, kGroupRows> kinfo;  // per process: one device
  if (kinfo.err != cudaSuccess) return kinfo.err;
  const F8Split f = forward_int8_split(m, n, kinfo.fit);
  if (static_cast<int64_t>(f.blocks) * f.S > INT32_MAX) return cudaErrorInvalidValue;
  CUtensorMap tmX;
  if (!encode_rows(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, ldx, T, n, kNT * 8, 64)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(f.blocks * f.S));
  cfg.blockDim = dim3(kF8Threads);
  cfg.dynamicSmemBytes = static_cast<size_t>(f8_smem_bytes<kNT>());
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(f.S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, linear_forward_int8_kernel<kNT, kGroupRows>, tmW, tmX, sW, T, m, n, f.slice, Y,
                            ldy);
}

cudaError_t launch_forward_int8(const uint16_t* X, int64_t ldx, const int8_t* W, int64_t ldw, const float* sW, int T,
                                int m, int n, uint16_t* Y, int64_t ldy, cudaStream_t s) {
  CUtensorMap tmW;
  if (!encode_rows(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, W, ldw, m, n, kF8Rows, kF8Tile))
    return cudaErrorInvalidValue;
  const double bytes = static_cast<double>(m) * n + 4.0 * ((static_cast<double>(m) * n + 255) / 256) +
                       2.0 * T * n + 2.0 * T * m;
  const int tok = profile_begin(s, QG_KERNEL_LINEAR_FUSED, 2.0 * T * m * n, bytes);
  const bool rows = n % 256 == 0;
  cudaError_t e;
  if (T <= 8)
    e = rows ? launch_forward_int8_as<1, true>(tmW, X, ldx, sW, T, m, n, Y, ldy, s)
             : launch_forward_int8_as<1, false>(tmW, X, ldx, sW, T, m, n, Y, ldy, s);
  else if (T <= 16)
    e = rows ? launch_forward_int8_as<2, true>(tmW, X, ldx, sW, T, m, n, Y, ldy, s)
             : launch_forward_int8_as<2, false>(tmW, X, ldx, sW, T, m, n, Y, ldy, s);
  else if (T <= 32)
    e = rows ? launch_forward_int8_as<4, true>(tmW, X, ldx, sW, T, m, n, Y, ldy, s)
             : launch_forward_int8_as<4, false>(tmW, X, ldx, sW, T, m, n, Y, ldy, s);
  else
    e = rows ? launch_forward_int8_as<8, true>(tmW, X, ldx, sW, T, m, n, Y, ldy, s)
             : launch_forward_int8_as<8, false>(tmW, X, ldx, sW, T, m, n, Y, ldy, s);
  profile_end(s, tok);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// ---------------------------------------------------------------- bf16 store epilogue

// The accumulator tile rounded to bf16 (nearest even) and stored row by row;
// two epilogue warpgroups, 128 columns each.
struct StoreBF16Epi {
  static constexpr int kSideBytes = 0;
  static constexpr int kSideBufs = 1;
  static constexpr bool kExchange = false;
  static constexpr int kPairGroups = 2;
  static constexpr int kPairBKMN = 64;
  static constexpr int kPairMaxStages = 6;
  static QG_DEV void issue_side(const CUtensorMap*, int, int, uint8_t*, uint64_t*) {}
  struct Args {
    uint16_t* D;
    int64_t ldd;  // elements, % 8 == 0
  };
  static QG_DEV void apply(const Args& a, int M, int N, int mb, int nb, int row, uint32_t taddr, const EpiPair& ep,
                           const uint8_t*) {
    const int grow = mb * BM + row;
    const bool ok = grow < M;
    const int j0 = nb * BN;
    const int ncols = min(BN, N - j0);
    const int nchunk = BN / 32 / ep.groups;
    const int c0 = ep.group * nchunk;
    const int c1 = min(c0 + nchunk, (ncols + 31) >> 5);
    uint16_t* drow = a.D + static_cast<int64_t>(grow) * a.ldd + j0;
    __syncwarp();
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(taddr + c * 32, v);
      tmem_ld_wait(v);
      // ok varies across the lanes at the matrix's last row; re-read per chunk
      // so that the loop is not unswitched around the warp-collective load
      if (!lane_pred(ok)) continue;
      uint32_t packed[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[e])));
        const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[e + 1])));
        packed[e >> 1] = lo | (hi << 16);
      }
      const int valid = ncols - c * 32;
      uint16_t* dst = drow + c * 32;
      if (valid >= 32) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          reinterpret_cast<uint4*>(dst)[q] =
              make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e < valid) dst[e] = static_cast<uint16_t>(packed[e >> 1] >> (16 * (e & 1)));
      }
    }
  }
};

static_assert(sizeof(GemmParams<StoreBF16Epi>) <= 32764, "kernel parameter block");

// D (M x N bf16) = A B on the CTA-pair kernel.  A: M x K row-major (K-major) or,
// with kAMN, its K x M transpose; B: N x K row-major (K-major) or, with kBMN,
// K x N row-major.
template <bool kAMN, bool kBMN>
cudaError_t launch_bf16(const void* A, int64_t lda, const void* B, int64_t ldb, uint16_t* D, int64_t ldd, int M,
                        int N, int K, cudaStream_t stream) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (K == 0) return cudaMemset2DAsync(D, ldd * 2, 0, static_cast<size_t>(N) * 2, M, stream);
  GemmParams<StoreBF16Epi> p;
  memset(&p, 0, sizeof(p));
  GemmProblem<StoreBF16Epi>& pr = p.prob[0];
  const bool okA = kAMN ? encode_map_bf16(&pr.tmA, A, M, K, lda, 64, 64) : encode_map_bf16(&pr.tmA, A, K, M, lda, 64, 128);
  const bool okB = kBMN ? encode_map_bf16(&pr.tmB, B, N, K, ldb, 64, 64) : encode_map_bf16(&pr.tmB, B, K, N, ldb, 64, 128);
  if (!okA || !okB) return cudaErrorInvalidValue;
  pr.M = M;
  pr.N = N;
  pr.K = K;
  pr.tiles_m = (M + BM - 1) / BM;
  pr.tiles_n = (N + BN - 1) / BN;
  pr.tile_begin = 0;
  pr.status = nullptr;
  pr.epi = StoreBF16Epi::Args{D, ldd};
  p.nprob = 1;
  p.total_tiles = pr.tiles_m * pr.tiles_n;

  auto kern = gemm_tc_pair_kernel<StoreBF16Epi, kAMN, kBMN>;
  using L = typename PairCfg<StoreBF16Epi, kAMN, kBMN>::L;
  constexpr size_t kSmem = L::kSmemBytes;
  static std::once_flag once;  // per instantiation
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [&] {
    attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
  });
  if (attr != cudaSuccess) return attr;
  const int pair_tiles = ((M + 255) / 256) * pr.tiles_n;
  const int clusters = std::min(pair_tiles, std::max(1, sm_count() / 2));
  const double flops = 2.0 * M * N * K, bytes = 2.0 * M * K + 2.0 * K * N + 2.0 * M * N;
  const int tok = profile_begin(stream, QG_KERNEL_LINEAR_GEMM, flops, bytes);
  kern<<<2 * clusters, L::kThreads, kSmem, stream>>>(p);
  profile_end(stream, tok);
  return cudaGetLastError();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qg_status status_of(cudaError_t e) { return e == cudaSuccess ? QG_OK : QG_ECUDA; }

// A bf16 operand: rows x cols with row stride ld elements.
qg_status check_bf16(const void* p, int64_t ld, int64_t rows, int64_t cols) {
  if (rows > 0 && cols > 0 && !p) return QG_EINVAL;
  if (ld < cols || ld % 8 != 0) return QG_ESHAPE;
  if (p && !aligned16(p)) return QG_EALIGN;
  return QG_OK;
}

}  // namespace

}  // namespace qg

using namespace qg;

qg_status qg_linear_dequant_weight(const int8_t* d_W, int64_t ldw, const float* d_sW, int32_t m, int32_t n,
                                   void* d_Wt, int64_t ldwt, void* stream) {
  if (m < 0 || n < 0) return QG_ESHAPE;
  if (m == 0 || n == 0) return QG_OK;
  if (!d_W || !d_sW || !d_Wt) return QG_EINVAL;
  if (ldw < n || ldw % 16 != 0 || ldwt < n || ldwt % 8 != 0) return QG_ESHAPE;
  if (!aligned16(d_W) || !aligned16(d_Wt)) return QG_EALIGN;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t work = static_cast<int64_t>(m) * ((n + 15) / 16);
  const int blocks = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>((work + 256 * kDqChunks - 1) / (256 * kDqChunks), int64_t(sm_count()) * 8)));
  const double bytes = 3.0 * m * n + 4.0 * ((static_cast<double>(m) * n + 255) / 256);
  const int tok = profile_begin(s, QG_KERNEL_LINEAR_DEQUANT, 0.0, bytes);
  dequant_weight_kernel<<<blocks, 256, 0, s>>>(d_W, ldw, d_sW, m, n, static_cast<uint16_t*>(d_Wt), ldwt);
  profile_end(s, tok);
  return status_of(cudaGetLastError());
}

qg_status qg_linear_forward(const void* d_X, int64_t ldx, const void* d_Wt, int64_t ldwt, int32_t T, int32_t m,
                            int32_t n, void* d_Y, int64_t ldy, void* stream) {
  if (T < 0 || m <= 0 || n <= 0) return QG_ESHAPE;
  qg_status st;
  if ((st = check_bf16(d_X, ldx, T, n)) != QG_OK || (st = check_bf16(d_Wt, ldwt, m, n)) != QG_OK ||
      (st = check_bf16(d_Y, ldy, T, m)) != QG_OK)
    return st;
  if (T == 0) return QG_OK;
  // Y (T x m) = X (T x n, K-major) W~^T (W~ m x n is B given N x K: K-major)
  return status_of(launch_bf16<false, false>(d_X, ldx, d_Wt, ldwt, static_cast<uint16_t*>(d_Y), ldy, T, m, n,
                                             static_cast<cudaStream_t>(stream)));
}

qg_status qg_linear_forward_int8(const void* d_X, int64_t ldx, const int8_t* d_W, int64_t ldw, const float* d_sW,
                                 int32_t T, int32_t m, int32_t n, void* d_Y, int64_t ldy, void* stream) {
  if (T < 0 || T > 64 || m <= 0 || n <= 0) return QG_ESHAPE;
  if (!d_W || !d_sW) return QG_EINVAL;
  if (ldw < n || ldw % 16 != 0) return QG_ESHAPE;
  if (!aligned16(d_W)) return QG_EALIGN;
  qg_status st;
  if ((st = check_bf16(d_X, ldx, T, n)) != QG_OK || (st = check_bf16(d_Y, ldy, T, m)) != QG_OK) return st;
  if (T == 0) return QG_OK;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint16_t* X = static_cast<const uint16_t*>(d_X);
  uint16_t* Y = static_cast<uint16_t*>(d_Y);
  return status_of(launch_forward_int8(X, ldx, d_W, ldw, d_sW, T, m, n, Y, ldy, s));
}

qg_status qg_linear_backward_data(const void* d_dY, int64_t lddy, const void* d_Wt, int64_t ldwt, int32_t T,
                                  int32_t m, int32_t n, void* d_dX, int64_t lddx, void* stream) {
  if (T < 0 || m <= 0 || n <= 0) return QG_ESHAPE;
  qg_status st;
  if ((st = check_bf16(d_dY, lddy, T, m)) != QG_OK || (st = check_bf16(d_Wt, ldwt, m, n)) != QG_OK ||
      (st = check_bf16(d_dX, lddx, T, n)) != QG_OK)
    return st;
  if (T == 0) return QG_OK;
  // dX (T x n) = D_y (T x m, K-major) W~ (m x n given K x N: MN-major)
  return status_of(launch_bf16<false, true>(d_dY, lddy, d_Wt, ldwt, static_cast<uint16_t*>(d_dX), lddx, T, n, m,
                                            static_cast<cudaStream_t>(stream)));
}

qg_status qg_linear_backward_weight(const void* d_dY, int64_t lddy, const void* d_X, int64_t ldx, int32_t T,
                                    int32_t m, int32_t n, void* d_G, int64_t ldg, void* stream) {
  if (T < 0 || m <= 0 || n <= 0) return QG_ESHAPE;
  qg_status st;
  if ((st = check_bf16(d_dY, lddy, T, m)) != QG_OK || (st = check_bf16(d_X, ldx, T, n)) != QG_OK ||
      (st = check_bf16(d_G, ldg, m, n)) != QG_OK)
    return st;
  // G (m x n) = D_y^T (D_y T x m given K x M: MN-major) X (T x n given K x N: MN-major);
  // T = 0 gives G = 0
  return status_of(launch_bf16<true, true>(d_dY, lddy, d_X, ldx, static_cast<uint16_t*>(d_G), ldg, m, n, T,
                                           static_cast<cudaStream_t>(stream)));
}
