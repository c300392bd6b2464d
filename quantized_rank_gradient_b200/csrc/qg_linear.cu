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
