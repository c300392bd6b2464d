// Layer-adaptive subspace refresh on sm_100a (the method's SVD step and its
// CosSim interval rule: AIMech Q-GaLore page, mechanism "layer-adaptive
// subspace cosine schedule", paper section 3.1, Eq. (5)).
//
// Top-r left singular vectors of G by randomized subspace iteration (Halko,
// Martinsson, Tropp 2011): Omega (n x k, Rademacher from Philox), Y = G Omega,
// Q = orth(Y); q times { Z = orth(G^T Q); Q = orth(G Z) }; B = Q^T G;
// S = B B^T = V diag(lambda) V^T; P = Q V[:, top r].  The products with G and
// S = B B^T run on the tcgen05 core (bf16 operands, fp32 accumulation; float32
// operands as bf16 hi + lo parts); orth() is shifted
// Cholesky-QR (Fukaya et al. 2020) with fp32 SIMT Gram matrices and X L^-T
// formed on the tensor cores from the explicit inverse: two passes for the
// intermediate bases of the power iterations, three for the final Q;
// the k x k eigenproblem uses a block one-sided Jacobi with bounded grid
// barriers.  Then: sign canonicalisation, INT4 quantization, and
// CosSim(P_new, P_prev) = (1/r) sum_i sigma_i(P_new^T P_prev) on the dequantized
// projections, the nuclear norm by a Newton-Schulz polar iteration.
#include <algorithm>
#include <cstring>

#include "qg_device.cuh"
#include "qg_internal.h"
#include "qg_linalg.cuh"
#include "qg_philox.cuh"
#include "qg_refresh.h"

namespace qg {

namespace {

constexpr float kAbsmaxFloorR = 7.52316384526264e-37f;  // 2^-120
constexpr uint32_t kOmegaSalt = 0x52454652u;
constexpr int kJacobiMaxSweeps = 30;
// Columns count as orthogonal once |a_p . a_q| <= tol |a_p| |a_q|; float32 dot
// products of length ~1000 carry relative noise of a few 1e-6, so the bound
// sits above that.
constexpr float kJacobiTol = 1e-5f;

size_t r256(size_t x) { return (x + 255) / 256 * 256; }

// CosSim's buffers for an r x r problem: four float32 r x r matrices (C, the
// iterate, the next iterate, the product), then, when the tensor cores take the
// Newton-Schulz steps, four bf16 r x 3r operand stacks.
bool ns_on_tensor_cores(int r) { return r % 32 == 0 && r >= 128; }
size_t cossim_buffer_bytes(int r) {
  const size_t rr = size_t(r) * r;
  return r256(rr * 4 * 4) + (ns_on_tensor_cores(r) ? 4 * r256(rr * 3 * 2) : 0);
}

struct RefreshLayout {
  int k, ldk, ldn4, ldn8;
  size_t P, omega, Y, Yb, Ylo, Z, Zb, Zlo, gram, gpart, linv, Li, Tt, Lih, Lil, Bm, Bh, Bl, At, Vt, lam, perm, Vsel, Pa, Pb,
      Ct, jx,
      mom, misc, total;
};

// Scratch of the split Jacobi on a k x k matrix: one exchange counter per block
// pair, then two buffers of kBJSplit partial Gram matrices per pair.
size_t jacobi_scratch_bytes(int k) {
  const int nblk = (k + kBJW - 1) / kBJW, pairs = (nblk + (nblk & 1)) / 2;
  return r256(size_t(pairs) * 4) + size_t(pairs) * 2 * kBJSplit * kBJP * kBJP * 4;
}

constexpr int kGramSlicesMax = 32;
int gram_tiles(int k) {
  const int t = (k + 63) / 64;
  return t * (t + 1) / 2;
}

RefreshLayout refresh_layout(int m, int n, int r, int p) {
  RefreshLayout L;
  L.k = std::min(std::min(r + p, m), n);
  L.ldk = (L.k + 7) / 8 * 8;
  L.ldn4 = (n + 3) / 4 * 4;
  L.ldn8 = (n + 7) / 8 * 8;
  const size_t k = L.k, ldk = L.ldk;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += r256(bytes);
    return o;
  };
  L.P = take(size_t(m) * r * 4);
  L.omega = take(size_t(n) * ldk * 2);
  L.Y = take(size_t(m) * ldk * 4);
  L.Yb = take(size_t(m) * ldk * 2);
  L.Ylo = take(size_t(m) * ldk * 2);
  L.Z = take(size_t(n) * ldk * 4);
  L.Zb = take(size_t(n) * ldk * 2);
  L.Zlo = take(size_t(n) * ldk * 2);
  L.gram = take(k * ldk * 4);
  L.gpart = take(size_t(kGramSlicesMax) * gram_tiles(L.k) * 64 * 64 * 4);
  L.linv = take(((k + 31) / 32) * 1024 * 4);
  L.Li = take(k * ldk * 4);
  L.Tt = take(k * ldk * 4);
  L.Lih = take(k * ldk * 2);
  L.Lil = take(k * ldk * 2);
  L.Bm = take(k * L.ldn4 * 4);
  L.Bh = take(k * L.ldn8 * 2);
  L.Bl = take(k * L.ldn8 * 2);
  L.At = take(k * ldk * 4);
  L.Vt = take(k * ldk * 4);
  L.lam = take(k * 4);
  L.perm = take(k * 4);
  L.Vsel = take(k * size_t(r) * 4);
  L.Pa = take(size_t(m) * r * 4);
  L.Pb = take(size_t(m) * r * 4);
  L.Ct = take(cossim_buffer_bytes(r));  // CosSim: C, the Newton-Schulz iterates and their bf16 operands
  L.jx = take(jacobi_scratch_bytes(L.k));
  // the rotated moments: r x n fp32 for the left projection; for the right one
  // (refresh called with m and n swapped) n x r, which is r x n here as well
  L.mom = take(size_t(r) * L.ldn4 * 4);
  L.misc = take(256);
  L.total = off;
  return L;
}

// misc region: [0..7] grid barrier, rotation counter, sweep's largest
// off-diagonal; then the Cholesky flag, the Jacobi sweeps, the CosSim value and
// the scale of its Newton-Schulz start
struct Misc {
  unsigned bar[8];
  int chol_flag;
  int sweeps;
  float cossim;
  float ns_scale;  // 1 / ||C||_F of CosSim's Newton-Schulz start
};

// ------------------------------------------------------------------ kernels

// Omega (n x ldk bf16): entry e = j*k + c (c < k) takes bit (e mod 32) of word
// ((e / 32) mod 4) of Philox-4x32-10(counter = (e / 128, refresh, layer, 0),
// key = (seed_lo ^ salt, seed_hi)); a set bit gives -1, else +1.  Padding 0.
__global__ void omega_kernel(uint16_t* Om, int64_t ld, int n, int k, uint32_t refresh_idx, uint32_t layer_id,
                             PhiloxKey key) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(n) * ld) return;
  const int64_t j = idx / ld, c = idx % ld;
  uint16_t out = 0;
  if (c < k) {
    const uint64_t e = static_cast<uint64_t>(j) * k + c;
    uint32_t w[4];
    philox4x32_10(static_cast<uint32_t>(e >> 7), refresh_idx, layer_id, 0u, key, w);
    const uint32_t word = w[(e >> 5) & 3];
    out = ((word >> (e & 31)) & 1u) ? 0xBF80u : 0x3F80u;  // bf16 -1 / +1
  }
  Om[idx] = out;
}

// Diagonal shift of the first Cholesky-QR pass: s = 11 (rows k + k (k + 1)) u tr(A),
// u = 2^-24, tr(A) = ||X||_F^2.
__global__ void __launch_bounds__(1024) add_shift_kernel(float* A, int64_t ld, int k, int rows) {
  __shared__ float part[32];
  float s = 0.f;
  for (int i = threadIdx.x; i < k; i += blockDim.x) s += A[static_cast<int64_t>(i) * ld + i];
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = (threadIdx.x < (blockDim.x >> 5)) ? part[threadIdx.x] : 0.f;
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
    if (threadIdx.x == 0) part[0] = t;
  }
  __syncthreads();
  const float shift = 11.f * (static_cast<float>(rows) * k + static_cast<float>(k) * (k + 1)) * 5.9604645e-8f * part[0];
  for (int i = threadIdx.x; i < k; i += blockDim.x) A[static_cast<int64_t>(i) * ld + i] += shift;
}

// ---- the low-rank moments at a refresh (cfg.mom_refresh = 2, rotation)

// out = code * scale (fp32), squared when kSquare: the first moment from its
// linear grid, or v = (code * scale)^2 from the square-root grid of the second
// (row blocks of 256 columns).
template <bool kSquare>
__global__ void moment_dequant_kernel(const int8_t* __restrict__ codes, int64_t ld_mom,
                                      const float* __restrict__ scales, int nblk, int r, int n, float* __restrict__ out,
                                      int64_t ldo) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(r) * n) return;
  const int64_t i = idx / n;
  const int j = static_cast<int>(idx % n);
  const float x = __fmul_rn(static_cast<float>(codes[i * ld_mom + j]), scales[i * nblk + (j >> 8)]);
  out[i * ldo + j] = kSquare ? __fmul_rn(x, x) : x;
}

// Re-quantization on the step's row-block grid, one warp per (row, block of 256
// columns): y = x (kSqrt: y = sqrt(x), correctly rounded), scale = absmax / 127,
// codes rint(y * (127 / absmax)) with both divisions IEEE; a block whose absmax
// is below 2^-120 gets scale 0 and codes 0.
template <bool kSqrt>
__global__ void moment_quant_kernel(const float* __restrict__ x, int64_t ldx, int r, int n, int nblk,
                                    int8_t* __restrict__ codes, int64_t ld_mom, float* __restrict__ scales) {
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<int64_t>(r) * nblk) return;
  const int64_t i = w / nblk;
  const int j0 = static_cast<int>(w % nblk) * 256;
  float y[8];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int j = j0 + lane + 32 * k;
    const float v = j < n ? x[i * ldx + j] : 0.f;
    y[k] = kSqrt ? __fsqrt_rn(v) : v;
    amax = fmaxf(amax, fabsf(y[k]));
  }
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  const bool live = amax >= kAbsmaxFloorR;
  const float inv = live ? __fdiv_rn(127.0f, amax) : 0.f;
  const float lo = kSqrt ? 0.f : -127.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int j = j0 + lane + 32 * k;
    if (j < n) codes[i * ld_mom + j] = static_cast<int8_t>(fminf(fmaxf(rintf(__fmul_rn(y[k], inv)), lo), 127.f));
  }
  if (lane == 0) scales[i * nblk + (j0 >> 8)] = live ? __fdiv_rn(amax, 127.0f) : 0.f;
}

__global__ void square_kernel(const float* __restrict__ a, float* __restrict__ b, int64_t count) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx < count) b[idx] = __fmul_rn(a[idx], a[idx]);
}

__global__ void identity_kernel(float* V, int64_t ld, int k) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(k) * ld) return;
  V[idx] = (idx / ld == idx % ld) ? 1.f : 0.f;
}

// out[p] = || row p of At ||  (one warp per row)
__global__ void row_norms_kernel(const float* At, int64_t ld, int k, int cols, float* out) {
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (w >= k) return;
  float s = 0.f;
  for (int t = lane; t < cols; t += 32) {
    const float x = __ldcg(At + static_cast<int64_t>(w) * ld + t);
    s = __fmaf_rn(x, x, s);
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if (lane == 0) out[w] = sqrtf(s);
}

// perm[rank] = p with ranks by descending lambda, ties to the lower index.
__global__ void __launch_bounds__(1024) rank_sort_kernel(const float* lam, int k, int* perm) {
  for (int p = threadIdx.x; p < k; p += blockDim.x) {
    const float v = lam[p];
    int rank = 0;
    for (int q = 0; q < k; ++q) {
      const float u = lam[q];
      rank += (u > v) || (u == v && q < p);
    }
    perm[rank] = p;
  }
}

// Vsel[t][c] = V[t][perm[c]] = Vt[perm[c]][t]  (k x r)
__global__ void gather_kernel(const float* Vt, int64_t ld, const int* perm, int k, int r, float* Vsel) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(k) * r) return;
  const int t = static_cast<int>(idx / r), c = static_cast<int>(idx % r);
  int pc = perm[c];
  if (pc < 0 || pc >= k) pc = 0;  // only reachable with non-finite eigenvalues
  Vsel[idx] = Vt[static_cast<int64_t>(pc) * ld + t];
}

// Column c of P (m x r): the entry of largest magnitude (first row on ties) is
// made positive by negating the column when needed.
__global__ void __launch_bounds__(256) canonical_signs_kernel(float* P, int m, int r) {
  const int c = blockIdx.x;
  __shared__ float bv[256];
  __shared__ int bi[256];
  float best = -1.f;
  int besti = 0x7FFFFFFF;
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    const float a = fabsf(P[static_cast<int64_t>(i) * r + c]);
    if (a > best) {
      best = a;
      besti = i;
    }
  }
  bv[threadIdx.x] = best;
  bi[threadIdx.x] = besti;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) {
      const float ov = bv[threadIdx.x + s];
      const int oi = bi[threadIdx.x + s];
      if (ov > bv[threadIdx.x] || (ov == bv[threadIdx.x] && oi < bi[threadIdx.x])) {
        bv[threadIdx.x] = ov;
        bi[threadIdx.x] = oi;
      }
    }
    __syncthreads();
  }
  __shared__ int flip_s;
  if (threadIdx.x == 0) flip_s = bi[0] < m && P[static_cast<int64_t>(bi[0]) * r + c] < 0.f;
  __syncthreads();
  if (flip_s)
    for (int i = threadIdx.x; i < m; i += blockDim.x) P[static_cast<int64_t>(i) * r + c] = -P[static_cast<int64_t>(i) * r + c];
}

// P = code * scale in float32 (m x r, row stride r) from packed INT4.
__global__ void dequant_f32_kernel(const uint8_t* Pq, const float* sP, int64_t total, float* out) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= total) return;
  const uint8_t b = Pq[e >> 1];
  const int nib = (e & 1) ? (b >> 4) : (b & 0xF);
  const int code = (nib ^ 8) - 8;
  out[e] = __fmul_rn(static_cast<float>(code), sP[e >> 6]);
}

// ---- CosSim = (1/r) sum_i sigma_i(C): the nuclear norm of C, which is
// trace(U^T C) for the polar factor U of C.  U by the Newton-Schulz iteration
// X <- X (3 I - X^T X) / 2 (Bjorck and Bowie 1971; Higham, "Functions of
// Matrices", 2008, section 8.3), from X_0 = C / ||C||_F: every singular value
// of X_0 lies in [0, 1] and moves to 1, small ones growing by 3/2 per step and
// then converging quadratically.  A direction still short of 1 after the last
// step adds less than its own sigma_i to the error.  After kNsIters = 40 steps
// every sigma_i / ||C||_F >= (2/3)^35 (about 7e-7) has converged; ||C||_F <=
// sqrt(r) for projections with orthonormal columns, so every sigma_i >= 2.3e-5
// has at r = 1024, and CosSim is within about 2.3e-5.
constexpr int kNsIters = 40;

// out[0] = 1 / ||A||_F for the n-element array A (0 for a zero array); one block.
__global__ void __launch_bounds__(1024) inv_frobenius_kernel(const float* __restrict__ A, int64_t n, float* out) {
  __shared__ float part[32];
  float s = 0.f;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s = __fmaf_rn(A[i], A[i], s);
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < (blockDim.x >> 5); ++i) t += part[i];
    out[0] = t > 0.f ? rsqrtf(t) : 0.f;
  }
}

__global__ void scale_kernel(const float* __restrict__ A, const float* __restrict__ factor, float* __restrict__ B,
                             int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) B[i] = __fmul_rn(A[i], factor[0]);
}

// T <- 1.5 I - 0.5 T for the r x r matrix T.
__global__ void ns_shift_kernel(float* __restrict__ T, int r) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(r) * r) return;
  const float d = (i / r == i % r) ? 1.5f : 0.f;
  T[i] = __fmaf_rn(-0.5f, T[i], d);
}

// bf16 hi + lo parts of the r x r float32 matrix M (or of 1.5 I - 0.5 M when
// kShift), written into the operand stacks of a product whose K is tripled:
// with A' = [A_hi | A_hi | A_lo] and B' = [B_hi ; B_lo ; B_hi], A' B' is
// A_hi B_hi + A_hi B_lo + A_lo B_hi, the float32 product up to the lo-lo term
// and about 2^-17 relative rounding of each operand.
//   ha (r x 3r): [hi | hi | lo]   the left operand, K-major
//   hb (r x 3r): [hi | lo | hi]   the right operand given transposed (K-major)
//   vb (3r x r): [hi ; lo ; hi]   the right operand as it stands (MN-major)
// Each may be null.
template <bool kShift>
__global__ void ns_split_kernel(const float* __restrict__ M, int r, uint16_t* __restrict__ ha,
                                uint16_t* __restrict__ hb, uint16_t* __restrict__ vb) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t rr = static_cast<int64_t>(r) * r;
  if (idx >= rr) return;
  const int64_t i = idx / r, j = idx % r;
  float x = M[idx];
  if (kShift) x = __fmaf_rn(-0.5f, x, i == j ? 1.5f : 0.f);
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  const __nv_bfloat16 l = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(h)));
  const uint16_t hu = __bfloat16_as_ushort(h), lu = __bfloat16_as_ushort(l);
  if (ha) {
    uint16_t* row = ha + i * 3 * r;
    row[j] = hu;
    row[r + j] = hu;
    row[2 * r + j] = lu;
  }
  if (hb) {
    uint16_t* row = hb + i * 3 * r;
    row[j] = hu;
    row[r + j] = lu;
    row[2 * r + j] = hu;
  }
  if (vb) {
    vb[idx] = hu;
    vb[rr + idx] = lu;
    vb[2 * rr + idx] = hu;
  }
}

// out[0] = (1/r) sum_ij X_ij C_ij = (1/r) trace(X^T C); one block.
__global__ void __launch_bounds__(1024) trace_product_kernel(const float* __restrict__ X, const float* __restrict__ C,
                                                             int r, float* out) {
  __shared__ float part[32];
  const int64_t n = static_cast<int64_t>(r) * r;
  float s = 0.f;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s = __fmaf_rn(X[i], C[i], s);
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < (blockDim.x >> 5); ++i) t += part[i];
    out[0] = t / static_cast<float>(r);
  }
}

// ------------------------------------------------------------------ host helpers

cudaError_t sgemm(bool ta, bool tb, const float* A, int64_t lda, const float* B, int64_t ldb, float* C, int64_t ldc,
                  int M, int N, int K, cudaStream_t s) {
  const dim3 grid((N + kSgBN - 1) / kSgBN, (M + kSgBM - 1) / kSgBM);
  const int tok = profile_begin(s, QG_KERNEL_OTHER, 2.0 * M * N * K, 4.0 * (double(M) * K + double(K) * N + double(M) * N));
  if (ta && tb)
    sgemm_kernel<true, true><<<grid, 256, 0, s>>>(A, lda, B, ldb, C, ldc, M, N, K, 1.f, 0.f);
  else if (ta)
    sgemm_kernel<true, false><<<grid, 256, 0, s>>>(A, lda, B, ldb, C, ldc, M, N, K, 1.f, 0.f);
  else if (tb)
    sgemm_kernel<false, true><<<grid, 256, 0, s>>>(A, lda, B, ldb, C, ldc, M, N, K, 1.f, 0.f);
  else
    sgemm_kernel<false, false><<<grid, 256, 0, s>>>(A, lda, B, ldb, C, ldc, M, N, K, 1.f, 0.f);
  profile_end(s, tok);
  return cudaGetLastError();
}

// Lower Cholesky factor of the k x k matrix A in place (blocked, 32-wide panels,
// one cooperative launch); Linv receives the inverses of the diagonal blocks.
cudaError_t cholesky(float* A, int64_t ld, int k, float* Linv, int* flag, unsigned* bar, uint32_t* status,
                     cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(bar, 0, 8 * sizeof(unsigned), s);
  if (e != cudaSuccess) return e;
  const int nblk = (k + 31) / 32;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, cholesky_kernel, 256, 0);
  if (e != cudaSuccess) return e;
  // one CTA per SM at most: the grid barriers cost grows with the CTA count
  const int want = std::max(1, (nblk - 1) * nblk / 2);
  const int grid = std::min(want, std::min(std::max(1, per_sm), 1) * sm_count());
  void* args[] = {&A, &ld, &k, &Linv, &flag, &bar, &status};
  return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(cholesky_kernel), dim3(grid), dim3(256), args, 0, s);
}

// Li <- L^-1 for the lower Cholesky factor L (k x k, stride ld, lower triangle
// of `Lf`), by recursive doubling from the 32 x 32 diagonal-block inverses:
// for blocks [A 0; C B] already inverted on the diagonal,
// the off-diagonal block of the inverse is -B^-1 (C A^-1).  Tt is k x ld scratch.
cudaError_t tri_inverse(const float* Lf, float* Li, float* Tt, int64_t ld, int k, const float* linv, cudaStream_t s) {
  const int64_t cnt = int64_t(k) * ld;
  trinv_init_kernel<<<static_cast<unsigned>((cnt + 255) / 256), 256, 0, s>>>(Li, ld, k, linv);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  for (int b = 32; b < k; b *= 2) {
    const int step = 2 * b;
    const int pairs = (k + step - 1) / step;
    const dim3 grid((b + kSgBN - 1) / kSgBN, (b + kSgBM - 1) / kSgBM, pairs);
    const int64_t st = int64_t(step) * ld + step;
    // T = C A^-1   (C = L[base + b.., base..], A^-1 = Li[base.., base..])
    sgemm_batched_kernel<false, false><<<grid, 256, 0, s>>>(Lf + int64_t(b) * ld, ld, st, Li, ld, st,
                                                            Tt + int64_t(b) * ld, ld, st, b, step, k, b, 0, 0, 1.f);
    // Li[base + b.., base..] = -B^-1 T   (B^-1 = Li[base + b.., base + b..])
    sgemm_batched_kernel<false, false><<<grid, 256, 0, s>>>(Li + int64_t(b) * ld + b, ld, st, Tt + int64_t(b) * ld, ld,
                                                            st, Li + int64_t(b) * ld, ld, st, b, step, k, b, 0, b,
                                                            -1.f);
  }
  return cudaGetLastError();
}

struct OrthBufs {
  unsigned* bar;
  uint32_t* status;
  float* gram;
  float* gpart;
  float* linv;
  float* Li;
  float* Tt;
  uint16_t* Lih;
  uint16_t* Lil;
  int* flag;
};

// Shifted Cholesky-QR (Fukaya et al. 2020): X (rows x k fp32, stride ld)
// becomes a basis of its column span.  The first pass adds the shift to the
// Gram matrix (it keeps the Cholesky factorisation from breaking down, whatever
// the condition number of X); the others are plain Cholesky-QR.  Each pass: Gram
// matrix in float32 (SIMT), Cholesky L L^T, the explicit inverse L^-1, then
// X <- X L^-T on the tensor cores with bf16 hi + lo parts of both operands
// (three products, fp32 accumulation, about 16 significant bits per pass; the
// next pass corrects the residual).  On return Xb and Xlo hold the bf16 hi and
// lo parts of the result (both are also used as scratch).
//   Subspace iteration depends only on the subspaces its bases span, so an
// intermediate basis needs to be well conditioned, not orthonormal to working
// precision: after the shifted and one plain pass its columns are orthonormal
// to about kappa^2 u (kappa the condition number of the product with G it came
// from), so the next product's condition number stays that of G's top
// directions, and that product reads only the basis' bf16 hi part.  The final
// basis, which Rayleigh-Ritz needs orthonormal, takes the third pass.  (The
// shifted pass alone does not lower the condition number much at these sizes:
// the shift exceeds sigma_max^2 of X once rows k is large, so one shifted pass
// per intermediate basis lets the condition numbers compound from one product
// with G to the next.)
cudaError_t orth(float* X, uint16_t* Xb, uint16_t* Xlo, int rows, int k, int64_t ld, const OrthBufs& ob,
                 int passes, cudaStream_t s) {
  cudaError_t e;
  const int64_t xcnt = int64_t(rows) * ld, lcnt = int64_t(k) * ld;
  for (int pass = 0; pass < passes; ++pass) {
    {
      const int ntiles = gram_tiles(k);
      const int slices = std::max(1, std::min(kGramSlicesMax, rows / 512));
      const int slice = (rows + slices - 1) / slices;
      const int tok = profile_begin(s, QG_KERNEL_OTHER, double(k) * k * rows, 4.0 * rows * k);
      gram_partial_kernel<<<dim3(ntiles, slices), 256, 0, s>>>(X, ld, rows, k, slice, ob.gpart, ntiles);
      gram_reduce_kernel<<<ntiles, 256, 0, s>>>(ob.gpart, ntiles, slices, ob.gram, ld, k);
      profile_end(s, tok);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (pass == 0) {
      add_shift_kernel<<<1, 1024, 0, s>>>(ob.gram, ld, k, rows);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if ((e = cholesky(ob.gram, ld, k, ob.linv, ob.flag, ob.bar, ob.status, s)) != cudaSuccess) return e;
    if ((e = tri_inverse(ob.gram, ob.Li, ob.Tt, ld, k, ob.linv, s)) != cudaSuccess) return e;
    split_bf16_kernel<<<static_cast<unsigned>((lcnt + 255) / 256), 256, 0, s>>>(ob.Li, ld, k, k, ob.Lih, ob.Lil, ld);
    split_bf16_kernel<<<static_cast<unsigned>((xcnt + 255) / 256), 256, 0, s>>>(X, ld, rows, k, Xb, Xlo, ld);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // X = Xhi Lhi^T + Xhi Llo^T + Xlo Lhi^T
    if ((e = launch_gemm_f32(Xb, ld, false, ob.Lih, ld, true, X, ld, rows, k, k, s)) != cudaSuccess) return e;
    if ((e = launch_gemm_f32(Xb, ld, false, ob.Lil, ld, true, X, ld, rows, k, k, s, true)) != cudaSuccess) return e;
    if ((e = launch_gemm_f32(Xlo, ld, false, ob.Lih, ld, true, X, ld, rows, k, k, s, true)) != cudaSuccess) return e;
  }
  split_bf16_kernel<<<static_cast<unsigned>((xcnt + 255) / 256), 256, 0, s>>>(X, ld, rows, k, Xb, Xlo, ld);
  return cudaGetLastError();
}

// One-sided Jacobi on the k x k matrix stored transposed in At (and Vt, if any);
// jx: jacobi_scratch_bytes(k) bytes.  Up to kBJResidentMaxK each block pair is
// shared by kBJSplit CTAs (jacobi_split_kernel); above, one CTA per pair streams
// its rows through shared memory.
cudaError_t jacobi(float* At, float* Vt, int64_t ld, int k, unsigned* bar, int* sweeps, uint32_t* status,
                   uint8_t* jx, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(bar, 0, 8 * sizeof(unsigned), s);
  if (e != cudaSuccess) return e;
  const int nblk = (k + kBJW - 1) / kBJW;
  const int pairs = (nblk + (nblk & 1)) / 2;
  int max_sweeps = kJacobiMaxSweeps;
  float tol = kJacobiTol;
  int per_sm = 0;
  if (k <= kBJResidentMaxK) {
    unsigned* pair_ctr = reinterpret_cast<unsigned*>(jx);
    float* gx = reinterpret_cast<float*>(jx + r256(size_t(pairs) * 4));
    if ((e = cudaMemsetAsync(pair_ctr, 0, size_t(pairs) * 4, s)) != cudaSuccess) return e;
    const size_t dyn = size_t(kBJP) * bj_resident_stride(bj_split_width(k)) * sizeof(float);
    void* fn = reinterpret_cast<void*>(jacobi_split_kernel);
    if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dyn))) !=
        cudaSuccess)
      return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, 256, dyn)) != cudaSuccess) return e;
    // every CTA of a cooperative launch is resident: as many pair slots as fit
    const int slots = std::max(1, std::min(pairs, std::max(1, per_sm) * sm_count() / kBJSplit));
    void* args[] = {&At, &Vt, &ld, &k, &max_sweeps, &tol, &bar, &pair_ctr, &gx, &sweeps, &status};
    const int tok = profile_begin(s, QG_KERNEL_OTHER, 0.0, 0.0);
    e = cudaLaunchCooperativeKernel(fn, dim3(slots * kBJSplit), dim3(256), args, dyn, s);
    profile_end(s, tok);
    return e;
  }
  void* fn = reinterpret_cast<void*>(jacobi_kernel<false>);
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, 256, 0)) != cudaSuccess) return e;
  const int grid = std::min(std::max(1, pairs), std::max(1, per_sm) * sm_count());
  void* args[] = {&At, &Vt, &ld, &k, &max_sweeps, &tol, &bar, &sweeps, &status};
  const int tok = profile_begin(s, QG_KERNEL_OTHER, 0.0, 0.0);
  e = cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(256), args, 0, s);
  profile_end(s, tok);
  return e;
}

// CosSim of Pa, Pb (fp32 m x r, stride ld) into d_out.  The Newton-Schulz
// iteration above runs on Y = X^T, where it reads
//   T = Y Y^T,   Y <- (1.5 I - 0.5 T) Y,
// two left-multiplications, from Y_0 = C' / ||C'||_F with C' = Pa^T Pb (= C^T:
// the same singular values).  The nuclear norm is then (1/r) trace(Y C') summed
// as sum_ij Y_ij C'_ij.  For r % 32 == 0 and r >= 128 the first
// kNsIters - kNsPolish steps run on the tcgen05 core with bf16 hi + lo operands
// (one launch per product, K = 3r); each step's rounding is then about 2^-17
// of the iterate, which the iteration itself damps, and the last kNsPolish
// steps run in float32 to bring the iterate to float32 orthogonality.
// buf: cossim_buffer_bytes(r); scal: one float.
constexpr int kNsPolish = 2;

cudaError_t cossim_core(const float* Pa, const float* Pb, int m, int r, int64_t ld, float* buf, float* scal,
                        float* d_out, cudaStream_t s) {
  const int64_t rr = int64_t(r) * r;
  float* C = buf;
  float* Y = buf + rr;
  float* Yn = buf + 2 * rr;
  float* T = buf + 3 * rr;
  cudaError_t e = sgemm(true, false, Pa, ld, Pb, ld, C, r, r, r, m, s);
  if (e != cudaSuccess) return e;
  const unsigned blocks = static_cast<unsigned>((rr + 255) / 256);
  inv_frobenius_kernel<<<1, 1024, 0, s>>>(C, rr, scal);
  scale_kernel<<<blocks, 256, 0, s>>>(C, scal, Y, rr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  int it = 0;
  if (ns_on_tensor_cores(r)) {
    uint8_t* ops = reinterpret_cast<uint8_t*>(buf) + r256(size_t(rr) * 4 * 4);
    const size_t stack = r256(size_t(rr) * 3 * 2);
    uint16_t* Yha = reinterpret_cast<uint16_t*>(ops);
    uint16_t* Yhb = reinterpret_cast<uint16_t*>(ops + stack);
    uint16_t* Yvb = reinterpret_cast<uint16_t*>(ops + 2 * stack);
    uint16_t* Tha = reinterpret_cast<uint16_t*>(ops + 3 * stack);
    const int64_t l3 = 3 * int64_t(r);
    for (; it < kNsIters - kNsPolish; ++it) {
      ns_split_kernel<false><<<blocks, 256, 0, s>>>(Y, r, Yha, Yhb, Yvb);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      // T = Y Y^T
      if ((e = launch_gemm_f32(Yha, l3, false, Yhb, l3, true, T, r, r, r, 3 * r, s)) != cudaSuccess) return e;
      ns_split_kernel<true><<<blocks, 256, 0, s>>>(T, r, Tha, nullptr, nullptr);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      // Y <- (1.5 I - 0.5 T) Y
      if ((e = launch_gemm_f32(Tha, l3, false, Yvb, r, false, Y, r, r, r, 3 * r, s)) != cudaSuccess) return e;
    }
  }
  for (; it < kNsIters; ++it) {
    if ((e = sgemm(false, true, Y, r, Y, r, T, r, r, r, r, s)) != cudaSuccess) return e;
    ns_shift_kernel<<<blocks, 256, 0, s>>>(T, r);
    if ((e = sgemm(false, false, T, r, Y, r, Yn, r, r, r, r, s)) != cudaSuccess) return e;
    std::swap(Y, Yn);
  }
  trace_product_kernel<<<1, 1024, 0, s>>>(Y, C, r, d_out);
  return cudaGetLastError();
}

qg_status st_of(cudaError_t e) { return e == cudaSuccess ? QG_OK : QG_ECUDA; }

// The moments at a refresh that replaces the projection Pb (dequantized, m x r)
// by Pa: kept, reset to zero, or rotated with C = Pa^T Pb (m' = C m,
// v' = (C o C) v) and re-quantized.  C and C2 are r x r scratch, X and Y r x ldx.
cudaError_t refresh_moments(const RefreshArgs& a, const float* Pa, const float* Pb, float* C, float* C2, float* X,
                            float* Y, cudaStream_t s) {
  // the moments are rows x cols (r x n, or m x r for the right-side projection,
  // whose r coordinates run along the columns); X and Y rows x cols, stride cols
  const int pm = a.m, r = a.r, rows = a.mom_rows, cols = a.mom_cols;
  const int64_t ldx = cols;
  cudaError_t e;
  if (a.mom_refresh == 0) return cudaSuccess;
  if (a.mom_refresh == 1) {
    const size_t codes = size_t(rows) * a.ld_mom, sc = size_t(rows) * a.nblk * 4;
    if ((e = cudaMemsetAsync(a.Mq, 0, codes, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(a.Vq, 0, codes, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(a.sM, 0, sc, s)) != cudaSuccess) return e;
    return cudaMemsetAsync(a.sV, 0, sc, s);
  }
  if ((e = sgemm(true, false, Pa, r, Pb, r, C, r, r, r, pm, s)) != cudaSuccess) return e;
  const int64_t rr = int64_t(r) * r, rc = int64_t(rows) * cols;
  square_kernel<<<static_cast<unsigned>((rr + 255) / 256), 256, 0, s>>>(C, C2, rr);
  const unsigned eb = static_cast<unsigned>((rc + 255) / 256);
  const unsigned qb = static_cast<unsigned>((int64_t(rows) * a.nblk * 32 + 255) / 256);
  // m' = C m (left) or m C^T (right)
  moment_dequant_kernel<false><<<eb, 256, 0, s>>>(a.Mq, a.ld_mom, a.sM, a.nblk, rows, cols, X, ldx);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  e = a.transpose_g ? sgemm(false, true, X, ldx, C, r, Y, ldx, rows, cols, r, s)
                    : sgemm(false, false, C, r, X, ldx, Y, ldx, rows, cols, r, s);
  if (e != cudaSuccess) return e;
  moment_quant_kernel<false><<<qb, 256, 0, s>>>(Y, ldx, rows, cols, a.nblk, a.Mq, a.ld_mom, a.sM);
  // v' = (C o C) v (left) or v (C o C)^T (right)
  moment_dequant_kernel<true><<<eb, 256, 0, s>>>(a.Vq, a.ld_mom, a.sV, a.nblk, rows, cols, X, ldx);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  e = a.transpose_g ? sgemm(false, true, X, ldx, C2, r, Y, ldx, rows, cols, r, s)
                    : sgemm(false, false, C2, r, X, ldx, Y, ldx, rows, cols, r, s);
  if (e != cudaSuccess) return e;
  moment_quant_kernel<true><<<qb, 256, 0, s>>>(Y, ldx, rows, cols, a.nblk, a.Vq, a.ld_mom, a.sV);
  return cudaGetLastError();
}

}  // namespace

// ------------------------------------------------------------------ INT4 quantizer

// One warp per group of 64 consecutive elements of the row-major m x r array:
// scale = absmax / 7, code = clamp(rint(x * (7 / absmax)), -7, 7) (both IEEE
// divisions once per group), packed two per byte, even element in the low nibble.
__global__ void quantize_int4_kernel(const float* __restrict__ P, int64_t ld, int32_t m, int32_t r,
                                     uint8_t* __restrict__ Pq, float* __restrict__ sP, int64_t ngroups) {
  const int64_t g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (g >= ngroups) return;
  const int64_t total = static_cast<int64_t>(m) * r;
  float x[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int64_t e = g * 64 + 2 * lane + k;
    x[k] = 0.f;
    if (e < total) x[k] = P[(e / r) * ld + (e % r)];
  }
  float amax = fmaxf(fabsf(x[0]), fabsf(x[1]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  // scale absmax / 7, codes rint(x * (7 / absmax)); absmax below 2^-120: zero group
  const bool live = amax >= kAbsmaxFloorR;
  const float s = live ? __fdiv_rn(amax, 7.0f) : 0.f;
  const float inv = live ? __fdiv_rn(7.0f, amax) : 0.f;
  int q[2] = {0, 0};
  if (live) {
#pragma unroll
    for (int k = 0; k < 2; ++k) q[k] = static_cast<int>(fminf(fmaxf(rintf(__fmul_rn(x[k], inv)), -7.f), 7.f));
  }
  const int64_t e0 = g * 64 + 2 * lane;
  if (e0 < total) Pq[e0 >> 1] = static_cast<uint8_t>((q[0] & 0xF) | ((q[1] & 0xF) << 4));
  if (lane == 0) sP[g] = s;
}

cudaError_t launch_quantize_projection(const float* P, int64_t ld, int32_t m, int32_t r, uint8_t* Pq, float* sP,
                                       cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(m) * r;
  const int64_t ngroups = (total + 63) / 64;
  if (ngroups == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (ngroups * 32 + threads - 1) / threads;
  const int tok = profile_begin(stream, QG_KERNEL_OTHER, 0.0, total * 4.0 + total / 2.0 + ngroups * 4.0);
  quantize_int4_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(P, ld, m, r, Pq, sP, ngroups);
  profile_end(stream, tok);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ refresh

size_t refresh_scratch_bytes(int32_t m, int32_t n, int32_t r, int32_t oversample) {
  return refresh_layout(m, n, r, oversample).total;
}

size_t cossim_scratch_bytes(int32_t, int32_t r) { return cossim_buffer_bytes(r) + 256; }

qg_status run_refresh(const RefreshArgs& a, uint8_t* ws, size_t ws_bytes, cudaStream_t s, float* cossim) {
  const RefreshLayout L = refresh_layout(a.m, a.n, a.r, a.oversample);
  if (ws_bytes < L.total) return QG_ESTATE;
  const int m = a.m, n = a.n, r = a.r, k = L.k;
  const int64_t ldk = L.ldk;
  float* P = reinterpret_cast<float*>(ws + L.P);
  uint16_t* Om = reinterpret_cast<uint16_t*>(ws + L.omega);
  float* Y = reinterpret_cast<float*>(ws + L.Y);
  uint16_t* Yb = reinterpret_cast<uint16_t*>(ws + L.Yb);
  uint16_t* Ylo = reinterpret_cast<uint16_t*>(ws + L.Ylo);
  float* Z = reinterpret_cast<float*>(ws + L.Z);
  uint16_t* Zb = reinterpret_cast<uint16_t*>(ws + L.Zb);
  uint16_t* Zlo = reinterpret_cast<uint16_t*>(ws + L.Zlo);
  float* gram = reinterpret_cast<float*>(ws + L.gram);
  float* linv = reinterpret_cast<float*>(ws + L.linv);
  float* Bm = reinterpret_cast<float*>(ws + L.Bm);
  float* At = reinterpret_cast<float*>(ws + L.At);
  float* Vt = reinterpret_cast<float*>(ws + L.Vt);
  float* lam = reinterpret_cast<float*>(ws + L.lam);
  int* perm = reinterpret_cast<int*>(ws + L.perm);
  float* Vsel = reinterpret_cast<float*>(ws + L.Vsel);
  Misc* misc = reinterpret_cast<Misc*>(ws + L.misc);
  if (cudaMemsetAsync(misc, 0, sizeof(Misc), s) != cudaSuccess) return QG_ECUDA;
  const OrthBufs ob{misc->bar, a.status, gram, reinterpret_cast<float*>(ws + L.gpart), linv, reinterpret_cast<float*>(ws + L.Li),
                    reinterpret_cast<float*>(ws + L.Tt),
                    reinterpret_cast<uint16_t*>(ws + L.Lih), reinterpret_cast<uint16_t*>(ws + L.Lil),
                    &misc->chol_flag};

  // Omega and the range finder
  {
    const int64_t cnt = int64_t(n) * ldk;
    const PhiloxKey key{static_cast<uint32_t>(a.seed) ^ kOmegaSalt, static_cast<uint32_t>(a.seed >> 32)};
    omega_kernel<<<static_cast<unsigned>((cnt + 255) / 256), 256, 0, s>>>(Om, ldk, n, k, a.refresh_idx, a.layer_id,
                                                                          key);
    if (cudaGetLastError() != cudaSuccess) return QG_ECUDA;
  }
  // G_eff (m x n) is G, or G^T for the right-side projection: the products
  // below take G as stored with the transposition flags flipped
  const bool tr = a.transpose_g != 0;
  if (launch_gemm_f32(a.G, a.ldg, tr, Om, ldk, false, Y, ldk, m, k, n, s) != cudaSuccess) return QG_ECUDA;
  // two passes for the intermediate bases, three for the final Q
  constexpr int kInterPasses = 2, kFinalPasses = 3;
  if (orth(Y, Yb, Ylo, m, k, ldk, ob, a.power_iters > 0 ? kInterPasses : kFinalPasses, s) != cudaSuccess)
    return QG_ECUDA;
  for (int it = 0; it < a.power_iters; ++it) {
    if (launch_gemm_f32(a.G, a.ldg, !tr, Yb, ldk, false, Z, ldk, n, k, m, s) != cudaSuccess) return QG_ECUDA;
    if (orth(Z, Zb, Zlo, n, k, ldk, ob, kInterPasses, s) != cudaSuccess) return QG_ECUDA;
    if (launch_gemm_f32(a.G, a.ldg, tr, Zb, ldk, false, Y, ldk, m, k, n, s) != cudaSuccess) return QG_ECUDA;
    const int passes = it + 1 == a.power_iters ? kFinalPasses : kInterPasses;
    if (orth(Y, Yb, Ylo, m, k, ldk, ob, passes, s) != cudaSuccess) return QG_ECUDA;
  }
  // Rayleigh-Ritz: B = Q^T G, S = B B^T, eigenpairs of S
  // B = Q^T G with Q split into bf16 hi + lo parts (about 16 significant bits)
  if (launch_gemm_f32(Yb, ldk, true, a.G, a.ldg, tr, Bm, L.ldn4, k, n, m, s) != cudaSuccess) return QG_ECUDA;
  if (launch_gemm_f32(Ylo, ldk, true, a.G, a.ldg, tr, Bm, L.ldn4, k, n, m, s, true) != cudaSuccess)
    return QG_ECUDA;
  // S = B B^T on the tensor cores: B split into bf16 hi + lo parts, three
  // products accumulated in float32 (hi hi^T + hi lo^T + lo hi^T)
  {
    uint16_t* Bh = reinterpret_cast<uint16_t*>(ws + L.Bh);
    uint16_t* Bl = reinterpret_cast<uint16_t*>(ws + L.Bl);
    const int64_t cnt = int64_t(k) * L.ldn8;
    split_bf16_kernel<<<static_cast<unsigned>((cnt + 255) / 256), 256, 0, s>>>(Bm, L.ldn4, k, n, Bh, Bl, L.ldn8);
    if (cudaGetLastError() != cudaSuccess) return QG_ECUDA;
    if (launch_gemm_f32(Bh, L.ldn8, false, Bh, L.ldn8, true, At, ldk, k, k, n, s) != cudaSuccess) return QG_ECUDA;
    if (launch_gemm_f32(Bh, L.ldn8, false, Bl, L.ldn8, true, At, ldk, k, k, n, s, true) != cudaSuccess)
      return QG_ECUDA;
    if (launch_gemm_f32(Bl, L.ldn8, false, Bh, L.ldn8, true, At, ldk, k, k, n, s, true) != cudaSuccess)
      return QG_ECUDA;
  }
  {
    const int64_t cnt = int64_t(k) * ldk;
    identity_kernel<<<static_cast<unsigned>((cnt + 255) / 256), 256, 0, s>>>(Vt, ldk, k);
    if (cudaGetLastError() != cudaSuccess) return QG_ECUDA;
  }
  if (jacobi(At, Vt, ldk, k, misc->bar, &misc->sweeps, a.status, ws + L.jx, s) != cudaSuccess) return QG_ECUDA;
  row_norms_kernel<<<(k * 32 + 255) / 256, 256, 0, s>>>(At, ldk, k, k, lam);
  if (cudaMemsetAsync(perm, 0, size_t(k) * sizeof(int), s) != cudaSuccess) return QG_ECUDA;
  rank_sort_kernel<<<1, 1024, 0, s>>>(lam, k, perm);
  gather_kernel<<<static_cast<unsigned>((int64_t(k) * r + 255) / 256), 256, 0, s>>>(Vt, ldk, perm, k, r, Vsel);
  if (cudaGetLastError() != cudaSuccess) return QG_ECUDA;
  // P = Q V[:, top r], sign-canonical, INT4
  if (sgemm(false, false, Y, ldk, Vsel, r, P, r, m, r, k, s) != cudaSuccess) return QG_ECUDA;
  canonical_signs_kernel<<<r, 256, 0, s>>>(P, m, r);
  if (cudaGetLastError() != cudaSuccess) return QG_ECUDA;
  const size_t mr = size_t(m) * r, pq = (mr + 1) / 2, ps = ((mr + 63) / 64) * 4;
  if (a.has_prev) {
    if (cudaMemcpyAsync(a.Pq_prev, a.Pq, pq, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return QG_ECUDA;
    if (cudaMemcpyAsync(a.sP_prev, a.sP, ps, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return QG_ECUDA;
  }
  if (launch_quantize_projection(P, r, m, r, a.Pq, a.sP, s) != cudaSuccess) return QG_ECUDA;
  // CosSim on the dequantized INT4 projections
  *cossim = 0.f;
  if (a.has_prev) {
    float* Pa = reinterpret_cast<float*>(ws + L.Pa);
    float* Pb = reinterpret_cast<float*>(ws + L.Pb);
    float* Ct = reinterpret_cast<float*>(ws + L.Ct);
    const unsigned blocks = static_cast<unsigned>((mr + 255) / 256);
    dequant_f32_kernel<<<blocks, 256, 0, s>>>(a.Pq, a.sP, static_cast<int64_t>(mr), Pa);
    dequant_f32_kernel<<<blocks, 256, 0, s>>>(a.Pq_prev, a.sP_prev, static_cast<int64_t>(mr), Pb);
    if (cudaGetLastError() != cudaSuccess) return QG_ECUDA;
    if (cossim_core(Pa, Pb, m, r, r, Ct, &misc->ns_scale, &misc->cossim, s) != cudaSuccess) return QG_ECUDA;
    if (refresh_moments(a, Pa, Pb, reinterpret_cast<float*>(ws + L.At), reinterpret_cast<float*>(ws + L.Vt),
                        reinterpret_cast<float*>(ws + L.Bm), reinterpret_cast<float*>(ws + L.mom), s) != cudaSuccess)
      return QG_ECUDA;
    float host = 0.f;
    if (cudaMemcpyAsync(&host, &misc->cossim, sizeof(float), cudaMemcpyDeviceToHost, s) != cudaSuccess) return QG_ECUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return QG_ECUDA;
    *cossim = host;
  }
  return QG_OK;
}

qg_status run_cossim(const float* Pa, const float* Pb, int32_t m, int32_t r, int64_t ld, float* d_out, uint8_t* ws,
                     cudaStream_t stream) {
  float* buf = reinterpret_cast<float*>(ws);
  float* scal = reinterpret_cast<float*>(ws + cossim_buffer_bytes(r));
  return st_of(cossim_core(Pa, Pb, m, r, ld, buf, scal, d_out, stream));
}

}  // namespace qg
