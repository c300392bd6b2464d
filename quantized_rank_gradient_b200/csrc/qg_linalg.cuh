// Small dense linear algebra for the subspace refresh (float32, SIMT):
//   sgemm_kernel        C = op(A) op(B) (64 x 64 tiles, 4 x 4 outputs per thread)
//   cholesky_kernel     blocked (32-wide) Cholesky in one cooperative launch
//   sgemm_batched_kernel  the same tiles over a batch of equal-size blocks
//   gram_partial_kernel, gram_reduce_kernel
//                       lower triangle of X^T X, split over row slices with a
//                       fixed-order reduction
//   trinv_init_kernel   block-diagonal start of L^-1 by recursive doubling
//   split_bf16_kernel   float32 -> bf16 hi + lo parts (tensor-core operands)
//   jacobi_kernel       block one-sided (Hestenes) Jacobi on the columns of a
//                       square matrix: round-robin pairs of 16-column blocks, one
//                       CTA per pair, the pair's 32 x 32 Gram diagonalised in
//                       shared memory, a bounded grid barrier between rounds
//                       (cooperative launch)
//   jacobi_split_kernel the same with each pair shared by four CTAs
#pragma once

#include "qg_device.cuh"

namespace qg {

// ------------------------------------------------------------------ SGEMM

constexpr int kSgBM = 64, kSgBN = 64, kSgBK = 16;

// C[M x N] = alpha * op(A) op(B) (+ beta * C).  A is M x K (kTA = false, row
// stride lda) or given as its K x M transpose (kTA = true); B is K x N or given as
// N x K (kTB = true).
template <bool kTA, bool kTB>
__global__ void __launch_bounds__(256) sgemm_kernel(const float* __restrict__ A, int64_t lda,
                                                    const float* __restrict__ B, int64_t ldb, float* __restrict__ C,
                                                    int64_t ldc, int M, int N, int K, float alpha, float beta) {
  __shared__ float As[kSgBK][kSgBM + 4];
  __shared__ float Bs[kSgBK][kSgBN + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * kSgBM, n0 = blockIdx.x * kSgBN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kSgBK) {
#pragma unroll
    for (int l = 0; l < 4; ++l) {
      const int e = tid + l * 256;  // 0..1023 over a 64 x 16 tile
      int mi, kk;
      if (kTA) {
        kk = e >> 6;
        mi = e & 63;
      } else {
        mi = e >> 4;
        kk = e & 15;
      }
      const int gm = m0 + mi, gk = k0 + kk;
      float v = 0.f;
      if (gm < M && gk < K) v = kTA ? A[static_cast<int64_t>(gk) * lda + gm] : A[static_cast<int64_t>(gm) * lda + gk];
      As[kk][mi] = v;
      int ni;
      if (kTB) {
        ni = e >> 4;
        kk = e & 15;
      } else {
        kk = e >> 6;
        ni = e & 63;
      }
      const int gn = n0 + ni, gk2 = k0 + kk;
      float w = 0.f;
      if (gn < N && gk2 < K) w = kTB ? B[static_cast<int64_t>(gn) * ldb + gk2] : B[static_cast<int64_t>(gk2) * ldb + gn];
      Bs[kk][ni] = w;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSgBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn >= N) continue;
      float* c = C + static_cast<int64_t>(gm) * ldc + gn;
      *c = beta == 0.f ? alpha * acc[i][j] : alpha * acc[i][j] + beta * *c;
    }
  }
}

// Batched form: blockIdx.z selects the problem; operand and result pointers
// advance by the given element strides, and each problem's M, N, K are clipped
// to the rows that remain below `limit` (M, N, K = min(b, limit - z * step)).
template <bool kTA, bool kTB>
__global__ void __launch_bounds__(256) sgemm_batched_kernel(const float* A, int64_t lda, int64_t sa,
                                                            const float* B, int64_t ldb, int64_t sb, float* C,
                                                            int64_t ldc, int64_t sc, int b, int step, int limit,
                                                            int mlead, int nlead, int klead, float alpha) {
  // problem z: M rows start at z*step + mlead, N at z*step + nlead, K at z*step + klead
  const int z = blockIdx.z;
  const int base = z * step;
  const int M = min(b, limit - (base + mlead)), N = min(b, limit - (base + nlead)), K = min(b, limit - (base + klead));
  if (M <= 0 || N <= 0 || K <= 0) return;
  __shared__ float As[kSgBK][kSgBM + 4];
  __shared__ float Bs[kSgBK][kSgBN + 4];
  A += z * sa;
  B += z * sb;
  C += z * sc;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * kSgBM, n0 = blockIdx.x * kSgBN;
  if (m0 >= M || n0 >= N) return;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kSgBK) {
#pragma unroll
    for (int l = 0; l < 4; ++l) {
      const int e = tid + l * 256;
      int mi, kk;
      if (kTA) {
        kk = e >> 6;
        mi = e & 63;
      } else {
        mi = e >> 4;
        kk = e & 15;
      }
      const int gm = m0 + mi, gk = k0 + kk;
      float v = 0.f;
      if (gm < M && gk < K) v = kTA ? A[static_cast<int64_t>(gk) * lda + gm] : A[static_cast<int64_t>(gm) * lda + gk];
      As[kk][mi] = v;
      int ni;
      if (kTB) {
        ni = e >> 4;
        kk = e & 15;
      } else {
        kk = e >> 6;
        ni = e & 63;
      }
      const int gn = n0 + ni, gk2 = k0 + kk;
      float w = 0.f;
      if (gn < N && gk2 < K) w = kTB ? B[static_cast<int64_t>(gn) * ldb + gk2] : B[static_cast<int64_t>(gk2) * ldb + gn];
      Bs[kk][ni] = w;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSgBK; ++kk) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bb[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn < N) C[static_cast<int64_t>(gm) * ldc + gn] = alpha * acc[i][j];
    }
  }
}

// Gram matrix G = X^T X (X: rows x k, stride ld) for the 64 x 64 tiles on or below
// the diagonal only (all a Cholesky factorisation reads), with the rows split
// into gridDim.y slices: CTA (t, s) writes the partial sum of slice s of tile t
// to Part[s][t] (64 x 64), and gram_reduce_kernel adds the slices in order, so
// the result does not depend on scheduling.
QG_DEV void lower_tile(int t, int& tm, int& tn) {
  int r = static_cast<int>((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
  while (r * (r + 1) / 2 > t) --r;
  while ((r + 1) * (r + 2) / 2 <= t) ++r;
  tm = r;
  tn = t - r * (r + 1) / 2;
}

__global__ void __launch_bounds__(256) gram_partial_kernel(const float* __restrict__ X, int64_t ld, int rows, int k,
                                                           int slice, float* __restrict__ Part, int ntiles) {
  __shared__ float As[kSgBK][kSgBM + 4];
  __shared__ float Bs[kSgBK][kSgBN + 4];
  int tm, tn;
  lower_tile(blockIdx.x, tm, tn);
  const int r0 = blockIdx.y * slice, r1 = min(rows, r0 + slice);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = tm * kSgBM, n0 = tn * kSgBN;
  float acc[4][4] = {};
  for (int k0 = r0; k0 < r1; k0 += kSgBK) {
#pragma unroll
    for (int l = 0; l < 4; ++l) {
      const int e = tid + l * 256;
      const int kk = e >> 6, mi = e & 63;
      const int gk = k0 + kk;
      As[kk][mi] = (gk < r1 && m0 + mi < k) ? X[static_cast<int64_t>(gk) * ld + m0 + mi] : 0.f;
      Bs[kk][mi] = (gk < r1 && n0 + mi < k) ? X[static_cast<int64_t>(gk) * ld + n0 + mi] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSgBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* out = Part + (static_cast<int64_t>(blockIdx.y) * ntiles + blockIdx.x) * (kSgBM * kSgBN);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) out[(ty * 4 + i) * kSgBN + tx * 4 + j] = acc[i][j];
}

__global__ void gram_reduce_kernel(const float* __restrict__ Part, int ntiles, int slices, float* __restrict__ G,
                                   int64_t ld, int k) {
  const int t = blockIdx.x;
  int tm, tn;
  lower_tile(t, tm, tn);
  for (int e = threadIdx.x; e < kSgBM * kSgBN; e += blockDim.x) {
    const int i = tm * kSgBM + e / kSgBN, j = tn * kSgBN + e % kSgBN;
    if (i >= k || j >= k) continue;
    float sum = 0.f;
    for (int s = 0; s < slices; ++s) sum += Part[(static_cast<int64_t>(s) * ntiles + t) * (kSgBM * kSgBN) + e];
    G[static_cast<int64_t>(i) * ld + j] = sum;
  }
}

// Li (k x k, stride ld) <- the block-diagonal of L^-1 from the 32 x 32 diagonal
// block inverses (Linv, 1024 floats each), zero elsewhere.
__global__ void trinv_init_kernel(float* Li, int64_t ld, int k, const float* Linv) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(k) * ld) return;
  const int i = static_cast<int>(idx / ld), j = static_cast<int>(idx % ld);
  float v = 0.f;
  if (j < k && (i >> 5) == (j >> 5)) v = Linv[static_cast<int64_t>(i >> 5) * 1024 + (i & 31) * 32 + (j & 31)];
  Li[idx] = v;
}

// float32 (rows x cols, stride ld) -> bf16 hi (= rn(x)) and lo (= rn(x - hi)),
// stride ldb; Xlo may be null.
__global__ void split_bf16_kernel(const float* X, int64_t ld, int rows, int cols, uint16_t* Xhi, uint16_t* Xlo,
                                  int64_t ldb) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(rows) * ldb) return;
  const int64_t i = idx / ldb, j = idx % ldb;
  const float x = j < cols ? X[i * ld + j] : 0.f;
  const __nv_bfloat16 hi = __float2bfloat16_rn(x);
  Xhi[idx] = __bfloat16_as_ushort(hi);
  if (Xlo) Xlo[idx] = __bfloat16_as_ushort(__float2bfloat16_rn(__fsub_rn(x, __bfloat162float(hi))));
}

// ------------------------------------------------------------------ Cholesky

// ------------------------------------------------------------------ Cholesky, one launch

QG_DEV bool grid_barrier(unsigned* bar, unsigned nblocks, uint32_t* status);

// Cholesky of the nb x nb diagonal block at (j0, j0) (lower triangle of A, read
// through L2) by one CTA: written back as L, its 32 x 32 inverse (lower,
// identity-padded) to Linv.  Non-positive pivots raise *flag (see below).
QG_DEV void chol_factor_diag(float* A, int64_t ld, int j0, int nb, float* Linv, int* flag, float (&T)[32][33],
                             float (&X)[32][33]) {
  __syncthreads();
  for (int e = threadIdx.x; e < 1024; e += blockDim.x) {
    const int i = e >> 5, j = e & 31;
    float v = (i == j) ? 1.f : 0.f;
    if (i < nb && j < nb && j <= i) v = __ldcg(A + static_cast<int64_t>(j0 + i) * ld + j0 + j);
    T[i][j] = (j <= i) ? v : 0.f;
  }
  __syncthreads();
  for (int c = 0; c < 32; ++c) {
    if (threadIdx.x == 0) {
      float d = T[c][c];
      if (!(d > 0.f)) {
        if (c < nb) atomicOr(flag, 1);
        d = 1e-30f;
      }
      T[c][c] = sqrtf(d);
    }
    __syncthreads();
    if (threadIdx.x > c && threadIdx.x < 32) T[threadIdx.x][c] = T[threadIdx.x][c] / T[c][c];
    __syncthreads();
    for (int e = threadIdx.x; e < 1024; e += blockDim.x) {
      const int i = e >> 5, j = e & 31;
      if (i > c && j > c && j <= i) T[i][j] = __fmaf_rn(-T[i][c], T[j][c], T[i][j]);
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < 1024; e += blockDim.x) {
    const int i = e >> 5, j = e & 31;
    if (i < nb && j < nb) __stcg(A + static_cast<int64_t>(j0 + i) * ld + j0 + j, (j <= i) ? T[i][j] : 0.f);
  }
  // inverse, row by row: X[r][j] = (delta_rj - sum_{t<r} T[r][t] X[t][j]) / T[r][r]
  for (int r = 0; r < 32; ++r) {
    if (threadIdx.x < 32) {
      const int j = threadIdx.x;
      float acc = (r == j) ? 1.f : 0.f;
      for (int t = j; t < r; ++t) acc = __fmaf_rn(-T[r][t], X[t][j], acc);
      X[r][j] = (r >= j) ? acc / T[r][r] : 0.f;
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < 1024; e += blockDim.x) __stcg(Linv + e, X[e >> 5][e & 31]);
}

// The whole blocked (32-wide) Cholesky of the k x k matrix A in one cooperative
// launch: per panel, the tiles below the diagonal block are solved against its
// inverse (TRSM), then the trailing lower tiles are updated (SYRK) and the CTA
// that updates the next diagonal tile factorises it right away; a bounded grid
// barrier follows each phase.  Linv receives the diagonal blocks' inverses.
__global__ void __launch_bounds__(256) cholesky_kernel(float* A, int64_t ld, int k, float* Linv, int* flag,
                                                       unsigned* bar, uint32_t* status) {
  __shared__ float T[32][33];
  __shared__ float X[32][33];
  __shared__ float Li[32][33];
  const int nblk = (k + 31) / 32;
  if (blockIdx.x == 0) chol_factor_diag(A, ld, 0, min(32, k), Linv, flag, T, X);
  if (!grid_barrier(bar, gridDim.x, status)) return;
  for (int jb = 0; jb < nblk; ++jb) {
    const int j0 = jb * 32;
    const int tiles = nblk - jb - 1;
    if (tiles == 0) break;
    // TRSM: L[i, j0 + c] = sum_c' A[i, j0 + c'] Linv[c][c'] for the rows below
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      __syncthreads();
      for (int e = threadIdx.x; e < 1024; e += blockDim.x) {
        const int r = e >> 5, c = e & 31;
        const int row = j0 + 32 + t * 32 + r;
        Li[r][c] = __ldcg(Linv + static_cast<int64_t>(jb) * 1024 + e);
        T[r][c] = (row < k && j0 + c < k) ? __ldcg(A + static_cast<int64_t>(row) * ld + j0 + c) : 0.f;
      }
      __syncthreads();
      for (int e = threadIdx.x; e < 1024; e += blockDim.x) {
        const int r = e >> 5, c = e & 31;
        const int row = j0 + 32 + t * 32 + r;
        float acc = 0.f;
        for (int q = 0; q <= c; ++q) acc = __fmaf_rn(T[r][q], Li[c][q], acc);
        if (row < k && j0 + c < k) __stcg(A + static_cast<int64_t>(row) * ld + j0 + c, acc);
      }
    }
    if (!grid_barrier(bar, gridDim.x, status)) return;
    // SYRK on the lower tiles of the trailing matrix; tile 0 is the next
    // diagonal block, factorised by its CTA as soon as it is updated
    // tile 0 (the next diagonal block, factorised right after its update) goes
    // to CTA 0 alone; the other tiles are spread over the other CTAs
    const int ntiles = tiles * (tiles + 1) / 2;
    const int others = gridDim.x > 1 ? static_cast<int>(gridDim.x) - 1 : 1;
    const int first = gridDim.x > 1 ? (blockIdx.x == 0 ? 0 : static_cast<int>(blockIdx.x)) : 0;
    const int stride = gridDim.x > 1 ? (blockIdx.x == 0 ? ntiles : others) : 1;
    for (int t = first; t < ntiles; t += stride) {
      int ti = static_cast<int>((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
      while (ti * (ti + 1) / 2 > t) --ti;
      while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
      const int tl = t - ti * (ti + 1) / 2;
      const int base = j0 + 32;
      __syncthreads();
      for (int e = threadIdx.x; e < 1024; e += blockDim.x) {
        const int r = e >> 5, c = e & 31;
        const int ri = base + ti * 32 + r, rl = base + tl * 32 + r;
        T[r][c] = (ri < k) ? __ldcg(A + static_cast<int64_t>(ri) * ld + j0 + c) : 0.f;
        X[r][c] = (rl < k) ? __ldcg(A + static_cast<int64_t>(rl) * ld + j0 + c) : 0.f;
      }
      __syncthreads();
      for (int e = threadIdx.x; e < 1024; e += blockDim.x) {
        const int r = e >> 5, c = e & 31;
        const int gi = base + ti * 32 + r, gl = base + tl * 32 + c;
        if (gi < k && gl < k && gl <= gi) {
          float acc = 0.f;
          for (int q = 0; q < 32; ++q) acc = __fmaf_rn(T[r][q], X[c][q], acc);
          float* a = A + static_cast<int64_t>(gi) * ld + gl;
          __stcg(a, __ldcg(a) - acc);
        }
      }
      if (t == 0) {
        __threadfence_block();
        chol_factor_diag(A, ld, base, min(32, k - base), Linv + static_cast<int64_t>(jb + 1) * 1024, flag, T, X);
      }
    }
    if (!grid_barrier(bar, gridDim.x, status)) return;
  }
}

// ------------------------------------------------------------------ Jacobi

// Bounded grid barrier for a cooperative launch.  bar[0] counts arrivals,
// bar[1] is the generation.  Returns false if the wait ran out (then *status
// gets the timeout bit) or another CTA gave up (bar[2] != 0).
QG_DEV bool grid_barrier(unsigned* bar, unsigned nblocks, uint32_t* status) {
  __shared__ int ok_s;
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile unsigned* gen = bar + 1;
    volatile unsigned* bad = bar + 2;
    const unsigned g = *gen;
    __threadfence();
    int ok = 1;
    if (atomicAdd(bar, 1u) == nblocks - 1) {
      atomicExch(bar, 0u);
      __threadfence();
      atomicAdd(bar + 1, 1u);
    } else {
      const uint64_t t0 = globaltimer();
      while (*gen == g) {
        if (*bad || globaltimer() - t0 > kWaitLimitNs) {
          ok = 0;
          atomicExch(bar + 2, 1u);
          if (status) atomicOr(status, kErrTimeout);
          break;
        }
      }
    }
    __threadfence();
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

// Block one-sided (Hestenes) Jacobi on the columns of a square matrix A
// (k x k, stored transposed: row p of At is column p of A, stride ld), applying
// the same rotations to V (rows of Vt) when Vt is non-null.
//
// The columns are grouped in blocks of kBJW; a round-robin tournament pairs the
// blocks (player 0 fixed, the others rotate; an odd count gets a dummy player),
// so that every pair of blocks meets once per sweep of nb - 1 rounds.  For a
// pair, one CTA forms the Gram matrix M of its 2 kBJW columns (streaming the
// columns through shared memory), and unless every off-diagonal entry already
// satisfies |M_pq| <= tol sqrt(M_pp M_qq), diagonalises M = J L J^T by cyclic
// two-sided Jacobi in shared memory and replaces the columns by A J (and V J).
// The pair's columns are then mutually orthogonal.  Rounds are separated by a
// bounded grid barrier (cooperative launch); bar[3] counts the pairs rotated in
// the current sweep, and the solve stops after a sweep without rotation or
// after max_sweeps.  At convergence the columns of A are orthogonal: for A = S
// symmetric positive semi-definite, V holds eigenvectors and the column norms
// are the eigenvalues; for any A they are its singular values.
constexpr int kBJW = 16;           // columns per block
constexpr int kBJP = 2 * kBJW;     // columns per block pair
constexpr int kBJChunk = 128;      // column entries streamed per pass
constexpr float kBJInnerTol = 1e-7f;
constexpr float kBJStopTol = 1e-4f;

struct BJShared {
  float X[kBJP][kBJChunk + 1];
  float M[kBJP][kBJP + 1];
  float T[kBJP][kBJP + 1];
  float J[kBJP][kBJP + 1];
  float JT[kBJP][kBJP + 1];
  float c[kBJP / 2], s[kBJP / 2];
  int pp[kBJP / 2], qq[kBJP / 2];  // the pairs of the current inner step
  int part[kBJP];                  // pair index of each column, + kBJP for the second member
  int rotate;
  __align__(16) float Jv[kBJP][kBJP];  // J again, rows 16-byte aligned for vector reads
};

// J <- J (3 I - J^T J) / 2: one Newton-Schulz step back towards orthogonality
// (the float32 product of the inner rotations drifts by a few ulps per rotation,
// and every application of J would carry that drift into the column norms).
QG_DEV void bj_reorthogonalize(BJShared& sh) {
  __syncthreads();
  for (int e = threadIdx.x; e < kBJP * kBJP; e += blockDim.x) {
    const int i = e / kBJP, j = e % kBJP;
    float g = 0.f;
#pragma unroll 8
    for (int l = 0; l < kBJP; ++l) g = __fmaf_rn(sh.J[l][i], sh.J[l][j], g);
    sh.T[i][j] = g;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kBJP * kBJP; e += blockDim.x) {
    const int i = e / kBJP, j = e % kBJP;
    float h = 0.f;
#pragma unroll 8
    for (int l = 0; l < kBJP; ++l) h = __fmaf_rn(sh.J[i][l], sh.T[l][j], h);
    sh.JT[i][j] = __fmaf_rn(-0.5f, h, 1.5f * sh.J[i][j]);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kBJP * kBJP; e += blockDim.x) {
    sh.J[e / kBJP][e % kBJP] = sh.JT[e / kBJP][e % kBJP];
    sh.Jv[e / kBJP][e % kBJP] = sh.JT[e / kBJP][e % kBJP];
  }
  __syncthreads();
}

// M = J L J^T by one cyclic Jacobi sweep (parallel ordering of the 2 kBJW
// columns) on the pair's Gram matrix in sh.M; J ends in sh.J.  The rotations
// come from rsqrt and approximate reciprocals: their angles only steer the
// outer iteration, whose stopping rule reads the Gram matrix itself, and the
// Newton-Schulz step that follows puts J back on the orthogonal group.
QG_DEV void bj_inner_sweep(BJShared& sh) {
  const int tid = threadIdx.x;
  {
    float(*Mc)[kBJP + 1] = sh.M;
    float(*Mn)[kBJP + 1] = sh.T;
    float(*Jc)[kBJP + 1] = sh.J;
    float(*Jn)[kBJP + 1] = sh.JT;
    for (int e = tid; e < kBJP * kBJP; e += blockDim.x) Jc[e / kBJP][e % kBJP] = (e / kBJP == e % kBJP) ? 1.f : 0.f;
    for (int step = 0; step < kBJP - 1; ++step) {
      if (tid < kBJP / 2) {
        // round-robin: player 0 fixed, players 1..31 move one place per step;
        // pair tid joins positions tid and kBJP - 1 - tid
        const int vp = tid - 1 + step, vq = kBJP - 2 - tid + step;
        const int p = tid == 0 ? 0 : (vp >= kBJP - 1 ? vp - (kBJP - 1) : vp) + 1;
        const int q = (vq >= kBJP - 1 ? vq - (kBJP - 1) : vq) + 1;
        const float al = Mc[p][p], be = Mc[q][q], ga = Mc[p][q];
        float c = 1.f, sn = 0.f;
        if (fabsf(ga) * rsqrtf(al) * rsqrtf(be) > kBJInnerTol) {
          const float zeta = __fdividef(be - al, 2.f * ga);
          const float az = fabsf(zeta);
          float t;
          if (az < 1e18f) {
            const float x = __fmaf_rn(zeta, zeta, 1.f);
            t = copysignf(__fdividef(1.f, az + x * rsqrtf(x)), zeta);
          } else {
            t = __fdividef(0.5f, zeta);
          }
          c = rsqrtf(__fmaf_rn(t, t, 1.f));
          sn = c * t;
        }
        sh.c[tid] = c;
        sh.s[tid] = sn;
        sh.pp[tid] = p;
        sh.qq[tid] = q;
        sh.part[p] = tid;
        sh.part[q] = tid + kBJP;
      }
      __syncthreads();
      // M' = R^T M R and J' = J R in one pass: thread t owns column t % 32
      // and rows t / 32 + 8 u.  Every load comes before the first store (the
      // buffers are distinct, but the compiler cannot know it, and would
      // otherwise keep each row's loads behind the previous row's stores).
      {
        constexpr int kU = kBJP / 8;
        const int j = tid & (kBJP - 1), i0 = tid >> 5;
        const int paj = sh.part[j], prj = paj & (kBJP - 1);
        const int pj = sh.pp[prj], qj = sh.qq[prj];
        const float cj = sh.c[prj], sj = sh.s[prj];
        const float cpj = paj >= kBJP ? sj : cj, cqj = paj >= kBJP ? cj : -sj;
        float cpi[kU], cqi[kU], mpp[kU], mpq[kU], mqp[kU], mqq[kU], jp[kU], jq[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int i = i0 + 8 * u;
          const int pai = sh.part[i], pri = pai & (kBJP - 1);
          const int pi = sh.pp[pri], qi = sh.qq[pri];
          const float ci = sh.c[pri], si = sh.s[pri];
          cpi[u] = pai >= kBJP ? si : ci;
          cqi[u] = pai >= kBJP ? ci : -si;
          mpp[u] = Mc[pi][pj];
          mpq[u] = Mc[pi][qj];
          mqp[u] = Mc[qi][pj];
          mqq[u] = Mc[qi][qj];
          jp[u] = Jc[i][pj];
          jq[u] = Jc[i][qj];
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int i = i0 + 8 * u;
          const float tp = __fmaf_rn(cpj, mpp[u], cqj * mpq[u]);
          const float tq = __fmaf_rn(cpj, mqp[u], cqj * mqq[u]);
          Mn[i][j] = __fmaf_rn(cpi[u], tp, cqi[u] * tq);
          Jn[i][j] = __fmaf_rn(cpj, jp[u], cqj * jq[u]);
        }
      }
      __syncthreads();
      float(*tm)[kBJP + 1] = Mc;
      Mc = Mn;
      Mn = tm;
      tm = Jc;
      Jc = Jn;
      Jn = tm;
    }
    if (Jc != sh.J) {
      for (int e = tid; e < kBJP * kBJP; e += blockDim.x) sh.J[e / kBJP][e % kBJP] = Jc[e / kBJP][e % kBJP];
    }
  }
}

// Rows of At (or Vt) belonging to the pair: local l -> global row, or -1.
QG_DEV int bj_row(int l, int I, int Jb, int k) {
  const int g = l < kBJW ? I * kBJW + l : Jb * kBJW + (l - kBJW);
  return g < k ? g : -1;
}

// Loads columns [c0, c0 + kBJChunk) of the pair's rows into X (0 outside).
QG_DEV void bj_load(BJShared& sh, const float* Mat, int64_t ld, int I, int Jb, int k, int c0) {
  for (int e = threadIdx.x; e < kBJP * kBJChunk; e += blockDim.x) {
    const int l = e / kBJChunk, cc = e % kBJChunk;
    const int g = bj_row(l, I, Jb, k);
    sh.X[l][cc] = (g >= 0 && c0 + cc < k) ? __ldcg(Mat + static_cast<int64_t>(g) * ld + c0 + cc) : 0.f;
  }
}

// rows <- J^T rows for the pair's rows of Mat (new row i = sum_l J[l][i] row_l).
QG_DEV void bj_apply(BJShared& sh, float* Mat, int64_t ld, int I, int Jb, int k) {
  const int cc = threadIdx.x % kBJChunk, ig = threadIdx.x / kBJChunk;  // 2 groups of 16 rows (256 threads)
  for (int c0 = 0; c0 < k; c0 += kBJChunk) {
    __syncthreads();
    bj_load(sh, Mat, ld, I, Jb, k, c0);
    __syncthreads();
    float out[kBJP / 2];
#pragma unroll
    for (int u = 0; u < kBJP / 2; ++u) out[u] = 0.f;
#pragma unroll 4
    for (int l = 0; l < kBJP; ++l) {
      const float x = sh.X[l][cc];
#pragma unroll
      for (int u = 0; u < kBJP / 2; ++u) out[u] = __fmaf_rn(sh.J[l][ig * (kBJP / 2) + u], x, out[u]);
    }
    if (c0 + cc < k) {
#pragma unroll
      for (int u = 0; u < kBJP / 2; ++u) {
        const int g = bj_row(ig * (kBJP / 2) + u, I, Jb, k);
        if (g >= 0) __stcg(Mat + static_cast<int64_t>(g) * ld + c0 + cc, out[u]);
      }
    }
  }
}

// ---- resident variant: the pair's 2 kBJW rows live in shared memory (one
// asynchronous load per pass), for k up to kBJResidentMaxK.
constexpr int kBJResidentMaxK = 1536;

// Row stride (floats) of the resident tile: a multiple of 4 that is 4 mod 32, so
// that 16-byte reads of the same column by rows 0..31 spread over all banks.
__host__ __device__ inline int bj_resident_stride(int k) {
  int kp = (k + 3) / 4 * 4;
  return kp + ((4 - kp % 32) + 32) % 32;  // kp = 4 mod 32, so kp / 4 is odd
}

QG_DEV void cp_async16(void* smem, const void* gmem, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem), "r"(src_bytes)
               : "memory");
}
QG_DEV void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// X (2 kBJW rows x kp) <- the pair's rows of Mat, zero outside the matrix.
QG_DEV void bj_load_resident(float* X, int kp, const float* Mat, int64_t ld, int I, int Jb, int k) {
  const int quads = kp / 4;
  for (int e = threadIdx.x; e < kBJP * quads; e += blockDim.x) {
    const int l = e / quads, c = (e % quads) * 4;
    const int g = bj_row(l, I, Jb, k);
    const int valid = (g >= 0 && c < k) ? min(4, k - c) : 0;
    const float* src = Mat + (g >= 0 ? static_cast<int64_t>(g) * ld : 0) + (valid ? c : 0);
    cp_async16(X + l * kp + c, src, valid * 4);
  }
  cp_async_wait_all();
  __syncthreads();
}

// rows of Mat <- J^T X (new row i = sum_l J[l][i] X[l]), 4 columns x 8 rows per
// thread and pass.
QG_DEV void bj_apply_resident(const BJShared& sh, const float* X, int kp, float* Mat, int64_t ld, int I, int Jb,
                              int k) {
  constexpr int kRows = kBJP / 4;
  static_assert(kRows == 8, "two 16-byte reads of J per row");
  const int quads = kp / 4;
  const int ig = threadIdx.x / 64, cq0 = threadIdx.x % 64;
  for (int cq = cq0; cq < quads; cq += 64) {
    const int c = cq * 4;
    if (c >= k) break;
    float4 out[kRows];
#pragma unroll
    for (int u = 0; u < kRows; ++u) out[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int l = 0; l < kBJP; ++l) {
      const float4 x = *reinterpret_cast<const float4*>(X + l * kp + c);
      const float4 ja = *reinterpret_cast<const float4*>(&sh.Jv[l][ig * kRows]);
      const float4 jb = *reinterpret_cast<const float4*>(&sh.Jv[l][ig * kRows + 4]);
      const float jr[kRows] = {ja.x, ja.y, ja.z, ja.w, jb.x, jb.y, jb.z, jb.w};
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const float j = jr[u];
        out[u].x = __fmaf_rn(j, x.x, out[u].x);
        out[u].y = __fmaf_rn(j, x.y, out[u].y);
        out[u].z = __fmaf_rn(j, x.z, out[u].z);
        out[u].w = __fmaf_rn(j, x.w, out[u].w);
      }
    }
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int g = bj_row(ig * kRows + u, I, Jb, k);
      if (g < 0) continue;
      float* dst = Mat + static_cast<int64_t>(g) * ld + c;
      if (c + 4 <= k) {
        __stcg(reinterpret_cast<float4*>(dst), out[u]);
      } else {
        __stcg(dst, out[u].x);
        if (c + 1 < k) __stcg(dst + 1, out[u].y);
        if (c + 2 < k) __stcg(dst + 2, out[u].z);
      }
    }
  }
}

template <bool kResident>
__global__ void __launch_bounds__(256) jacobi_kernel(float* At, float* Vt, int64_t ld, int k, int max_sweeps,
                                                     float tol, unsigned* bar, int* sweeps_out, uint32_t* status) {
  __shared__ BJShared sh;
  extern __shared__ float4 dyn_smem[];
  float* Xr = reinterpret_cast<float*>(dyn_smem);
  const int kp = bj_resident_stride(k);
  const int tid = threadIdx.x;
  const int nblk = (k + kBJW - 1) / kBJW;
  const int nb = nblk + (nblk & 1);
  const int npairs = nb / 2;
  unsigned* rot = bar + 3;
  int sweep = 0;
  for (; sweep < max_sweeps; ++sweep) {
    for (int round = 0; round < nb - 1; ++round) {
      for (int pidx = blockIdx.x; pidx < npairs; pidx += gridDim.x) {
        const int a = pidx, b = nb - 1 - pidx;
        const int I = (a == 0) ? 0 : ((a - 1 + round) % (nb - 1)) + 1;
        const int Jb = ((b - 1 + round) % (nb - 1)) + 1;
        if (I >= nblk || Jb >= nblk) continue;  // paired with the dummy player
        // ---- Gram matrix of the pair's columns (2 x 2 outputs per thread)
        const int ty = tid >> 4, tx = tid & 15;
        float g00 = 0.f, g01 = 0.f, g10 = 0.f, g11 = 0.f;
        if (kResident) {
          __syncthreads();
          bj_load_resident(Xr, kp, At, ld, I, Jb, k);
          // rows ty, ty + 16 against tx, tx + 16: with kp / 4 odd, sixteen
          // consecutive rows fall on eight different 16-byte bank groups
          const float* ra0 = Xr + ty * kp;
          const float* ra1 = ra0 + 16 * kp;
          const float* rb0 = Xr + tx * kp;
          const float* rb1 = rb0 + 16 * kp;
          // four partial sums per entry (one per float4 lane): shorter rounding
          // chains keep the Gram's noise below the convergence test
          float4 s00 = make_float4(0.f, 0.f, 0.f, 0.f), s01 = s00, s10 = s00, s11 = s00;
#pragma unroll 4
          for (int c = 0; c < kp; c += 4) {
            const float4 a0 = *reinterpret_cast<const float4*>(ra0 + c), a1 = *reinterpret_cast<const float4*>(ra1 + c);
            const float4 b0 = *reinterpret_cast<const float4*>(rb0 + c), b1 = *reinterpret_cast<const float4*>(rb1 + c);
            s00.x = __fmaf_rn(a0.x, b0.x, s00.x); s00.y = __fmaf_rn(a0.y, b0.y, s00.y);
            s00.z = __fmaf_rn(a0.z, b0.z, s00.z); s00.w = __fmaf_rn(a0.w, b0.w, s00.w);
            s01.x = __fmaf_rn(a0.x, b1.x, s01.x); s01.y = __fmaf_rn(a0.y, b1.y, s01.y);
            s01.z = __fmaf_rn(a0.z, b1.z, s01.z); s01.w = __fmaf_rn(a0.w, b1.w, s01.w);
            s10.x = __fmaf_rn(a1.x, b0.x, s10.x); s10.y = __fmaf_rn(a1.y, b0.y, s10.y);
            s10.z = __fmaf_rn(a1.z, b0.z, s10.z); s10.w = __fmaf_rn(a1.w, b0.w, s10.w);
            s11.x = __fmaf_rn(a1.x, b1.x, s11.x); s11.y = __fmaf_rn(a1.y, b1.y, s11.y);
            s11.z = __fmaf_rn(a1.z, b1.z, s11.z); s11.w = __fmaf_rn(a1.w, b1.w, s11.w);
          }
          g00 = (s00.x + s00.y) + (s00.z + s00.w);
          g01 = (s01.x + s01.y) + (s01.z + s01.w);
          g10 = (s10.x + s10.y) + (s10.z + s10.w);
          g11 = (s11.x + s11.y) + (s11.z + s11.w);
        }
        for (int c0 = 0; !kResident && c0 < k; c0 += kBJChunk) {
          __syncthreads();
          bj_load(sh, At, ld, I, Jb, k, c0);
          __syncthreads();
#pragma unroll 8
          for (int cc = 0; cc < kBJChunk; ++cc) {
            const float a0 = sh.X[2 * ty][cc], a1 = sh.X[2 * ty + 1][cc];
            const float b0 = sh.X[2 * tx][cc], b1 = sh.X[2 * tx + 1][cc];
            g00 = __fmaf_rn(a0, b0, g00);
            g01 = __fmaf_rn(a0, b1, g01);
            g10 = __fmaf_rn(a1, b0, g10);
            g11 = __fmaf_rn(a1, b1, g11);
          }
        }
        if (kResident) {
          sh.M[ty][tx] = g00;
          sh.M[ty][tx + 16] = g01;
          sh.M[ty + 16][tx] = g10;
          sh.M[ty + 16][tx + 16] = g11;
        } else {
          sh.M[2 * ty][2 * tx] = g00;
          sh.M[2 * ty][2 * tx + 1] = g01;
          sh.M[2 * ty + 1][2 * tx] = g10;
          sh.M[2 * ty + 1][2 * tx + 1] = g11;
        }
        if (tid == 0) sh.rotate = 0;
        __syncthreads();
        // ---- already orthogonal to tol?  (also the sweep's largest relative
        // off-diagonal entry, for the stopping rule)
        {
          float worst = 0.f;
          for (int e = tid; e < kBJP * kBJP; e += blockDim.x) {
            const int p = e / kBJP, q = e % kBJP;
            if (p < q) {
              const float dd = sh.M[p][p] * sh.M[q][q];
              const float rel = dd > 0.f ? fabsf(sh.M[p][q]) * rsqrtf(sh.M[p][p]) * rsqrtf(sh.M[q][q]) : 0.f;
              if (rel > tol) sh.rotate = 1;
              worst = fmaxf(worst, rel);
            }
          }
          for (int o = 16; o > 0; o >>= 1) worst = fmaxf(worst, __shfl_xor_sync(0xFFFFFFFFu, worst, o));
          if ((tid & 31) == 0 && worst > 0.f) atomicMax(bar + 4, __float_as_uint(worst));
        }
        __syncthreads();
        if (!sh.rotate) continue;
        bj_inner_sweep(sh);
        bj_reorthogonalize(sh);
        // ---- the pair's columns (and V's) become A J
        if (kResident) {
          bj_apply_resident(sh, Xr, kp, At, ld, I, Jb, k);
          if (Vt) {
            __syncthreads();
            bj_load_resident(Xr, kp, Vt, ld, I, Jb, k);
            bj_apply_resident(sh, Xr, kp, Vt, ld, I, Jb, k);
          }
        } else {
          bj_apply(sh, At, ld, I, Jb, k);
          if (Vt) bj_apply(sh, Vt, ld, I, Jb, k);
        }
        if (tid == 0) atomicAdd(rot, 1u);
      }
      if (!grid_barrier(bar, gridDim.x, status)) return;
    }
    const unsigned rotations = *reinterpret_cast<volatile unsigned*>(rot);
    const float worst = __uint_as_float(*reinterpret_cast<volatile unsigned*>(bar + 4));
    if (!grid_barrier(bar, gridDim.x, status)) return;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      atomicExch(rot, 0u);
      atomicExch(bar + 4, 0u);
    }
    if (!grid_barrier(bar, gridDim.x, status)) return;
    // done after a sweep without rotation, or once every pair met in this sweep
    // was within kBJStopTol (the rotations of this sweep leave the columns
    // orthogonal to about tol; float32 rounding keeps a few pairs from ever
    // passing tol exactly)
    if (rotations == 0 || worst <= kBJStopTol) {
      ++sweep;
      break;
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && sweeps_out) *sweeps_out = sweep;
}

// ---- split variant: each block pair is shared by kBJSplit CTAs, each holding
// the pair's 2 kBJW rows over one slice of the k columns (the slices are
// multiples of 4 columns).  The CTAs exchange their partial Gram matrices
// through global memory (double-buffered by the slot's exchange parity, so that
// the next exchange never overwrites partials another CTA of the pair still
// reads), sum them in one fixed order (every CTA gets the same M bit for bit),
// and then run the same inner sweep and Newton-Schulz step, so that all hold the
// same J; each applies it to its own slice.  Four times the SMs of the one-CTA
// form work on each round's Gram matrices and updates.
constexpr int kBJSplit = 4;

__host__ __device__ inline int bj_split_width(int k) { return ((k + kBJSplit - 1) / kBJSplit + 3) / 4 * 4; }

// X (2 kBJW rows x kps) <- columns [c_lo, c_lo + cw) of the pair's rows of Mat,
// zero outside the matrix and beyond cw.
QG_DEV void bj_load_slice(float* X, int kps, const float* Mat, int64_t ld, int I, int Jb, int k, int c_lo, int cw) {
  const int quads = kps / 4;
  for (int e = threadIdx.x; e < kBJP * quads; e += blockDim.x) {
    const int l = e / quads, c = (e % quads) * 4;
    const int g = bj_row(l, I, Jb, k);
    const int gc = c_lo + c;
    const int valid = (g >= 0 && c < cw && gc < k) ? min(4, k - gc) : 0;
    const float* src = Mat + (valid ? static_cast<int64_t>(g) * ld + gc : 0);
    cp_async16(X + l * kps + c, src, valid * 4);
  }
  cp_async_wait_all();
  __syncthreads();
}

// The slice's columns of the pair's rows of Mat <- J^T X.
QG_DEV void bj_apply_slice(const BJShared& sh, const float* X, int kps, float* Mat, int64_t ld, int I, int Jb, int k,
                           int c_lo, int cw) {
  constexpr int kRows = kBJP / 4;
  const int ig = threadIdx.x / 64, cq0 = threadIdx.x % 64;
  for (int cq = cq0; cq < cw / 4; cq += 64) {
    const int c = cq * 4, gc = c_lo + c;
    if (gc >= k) break;
    float4 out[kRows];
#pragma unroll
    for (int u = 0; u < kRows; ++u) out[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int l = 0; l < kBJP; ++l) {
      const float4 x = *reinterpret_cast<const float4*>(X + l * kps + c);
      const float4 ja = *reinterpret_cast<const float4*>(&sh.Jv[l][ig * kRows]);
      const float4 jb = *reinterpret_cast<const float4*>(&sh.Jv[l][ig * kRows + 4]);
      const float jr[kRows] = {ja.x, ja.y, ja.z, ja.w, jb.x, jb.y, jb.z, jb.w};
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const float j = jr[u];
        out[u].x = __fmaf_rn(j, x.x, out[u].x);
        out[u].y = __fmaf_rn(j, x.y, out[u].y);
        out[u].z = __fmaf_rn(j, x.z, out[u].z);
        out[u].w = __fmaf_rn(j, x.w, out[u].w);
      }
    }
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int g = bj_row(ig * kRows + u, I, Jb, k);
      if (g < 0) continue;
      float* dst = Mat + static_cast<int64_t>(g) * ld + gc;
      if (gc + 4 <= k) {
        __stcg(reinterpret_cast<float4*>(dst), out[u]);
      } else {
        __stcg(dst, out[u].x);
        if (gc + 1 < k) __stcg(dst + 1, out[u].y);
        if (gc + 2 < k) __stcg(dst + 2, out[u].z);
      }
    }
  }
}

// The same Jacobi as jacobi_kernel, gridDim.x = kBJSplit x slots.  pair_ctr
// (one counter per slot, zero at launch) and gx (slots x 2 x kBJSplit x kBJP^2
// floats) carry the Gram exchange.
__global__ void __launch_bounds__(256) jacobi_split_kernel(float* At, float* Vt, int64_t ld, int k, int max_sweeps,
                                                           float tol, unsigned* bar, unsigned* pair_ctr, float* gx,
                                                           int* sweeps_out, uint32_t* status) {
  __shared__ BJShared sh;
  __shared__ int ok_s;
  extern __shared__ float4 dyn_smem[];
  float* Xr = reinterpret_cast<float*>(dyn_smem);
  const int cw = bj_split_width(k);
  const int kps = bj_resident_stride(cw);
  const int tid = threadIdx.x;
  const int sub = blockIdx.x % kBJSplit, slot = blockIdx.x / kBJSplit, nslots = gridDim.x / kBJSplit;
  const int c_lo = sub * cw;
  const int nblk = (k + kBJW - 1) / kBJW;
  const int nb = nblk + (nblk & 1);
  const int npairs = nb / 2;
  unsigned* rot = bar + 3;
  unsigned nex = 0;  // exchanges of this slot so far (the same in its kBJSplit CTAs)
  int sweep = 0;
  for (; sweep < max_sweeps; ++sweep) {
    for (int round = 0; round < nb - 1; ++round) {
      for (int pidx = slot; pidx < npairs; pidx += nslots) {
        const int a = pidx, b = nb - 1 - pidx;
        const int I = (a == 0) ? 0 : ((a - 1 + round) % (nb - 1)) + 1;
        const int Jb = ((b - 1 + round) % (nb - 1)) + 1;
        if (I >= nblk || Jb >= nblk) continue;  // paired with the dummy player
        // ---- partial Gram matrix over this CTA's slice (2 x 2 outputs per thread)
        const int ty = tid >> 4, tx = tid & 15;
        __syncthreads();
        bj_load_slice(Xr, kps, At, ld, I, Jb, k, c_lo, cw);
        {
          const float* ra0 = Xr + ty * kps;
          const float* ra1 = ra0 + 16 * kps;
          const float* rb0 = Xr + tx * kps;
          const float* rb1 = rb0 + 16 * kps;
          float4 s00 = make_float4(0.f, 0.f, 0.f, 0.f), s01 = s00, s10 = s00, s11 = s00;
#pragma unroll 4
          for (int c = 0; c < kps; c += 4) {
            const float4 a0 = *reinterpret_cast<const float4*>(ra0 + c), a1 = *reinterpret_cast<const float4*>(ra1 + c);
            const float4 b0 = *reinterpret_cast<const float4*>(rb0 + c), b1 = *reinterpret_cast<const float4*>(rb1 + c);
            s00.x = __fmaf_rn(a0.x, b0.x, s00.x); s00.y = __fmaf_rn(a0.y, b0.y, s00.y);
            s00.z = __fmaf_rn(a0.z, b0.z, s00.z); s00.w = __fmaf_rn(a0.w, b0.w, s00.w);
            s01.x = __fmaf_rn(a0.x, b1.x, s01.x); s01.y = __fmaf_rn(a0.y, b1.y, s01.y);
            s01.z = __fmaf_rn(a0.z, b1.z, s01.z); s01.w = __fmaf_rn(a0.w, b1.w, s01.w);
            s10.x = __fmaf_rn(a1.x, b0.x, s10.x); s10.y = __fmaf_rn(a1.y, b0.y, s10.y);
            s10.z = __fmaf_rn(a1.z, b0.z, s10.z); s10.w = __fmaf_rn(a1.w, b0.w, s10.w);
            s11.x = __fmaf_rn(a1.x, b1.x, s11.x); s11.y = __fmaf_rn(a1.y, b1.y, s11.y);
            s11.z = __fmaf_rn(a1.z, b1.z, s11.z); s11.w = __fmaf_rn(a1.w, b1.w, s11.w);
          }
          float* mine = gx + ((static_cast<size_t>(slot) * 2 + (nex & 1u)) * kBJSplit + sub) * (kBJP * kBJP);
          __stcg(mine + ty * kBJP + tx, (s00.x + s00.y) + (s00.z + s00.w));
          __stcg(mine + ty * kBJP + tx + 16, (s01.x + s01.y) + (s01.z + s01.w));
          __stcg(mine + (ty + 16) * kBJP + tx, (s10.x + s10.y) + (s10.z + s10.w));
          __stcg(mine + (ty + 16) * kBJP + tx + 16, (s11.x + s11.y) + (s11.z + s11.w));
        }
        // ---- the pair's kBJSplit partials meet (bounded wait)
        __syncthreads();
        ++nex;
        if (tid == 0) {
          __threadfence();
          atomicAdd(pair_ctr + slot, 1u);
          const unsigned target = kBJSplit * nex;
          volatile unsigned* ctr = pair_ctr + slot;
          volatile unsigned* bad = bar + 2;
          int ok = 1;
          const uint64_t t0 = globaltimer();
          while (*ctr < target) {
            if (*bad || globaltimer() - t0 > kWaitLimitNs) {
              ok = 0;
              atomicExch(bar + 2, 1u);
              if (status) atomicOr(status, kErrTimeout);
              break;
            }
          }
          __threadfence();
          ok_s = ok;
        }
        __syncthreads();
        if (!ok_s) return;
        {
          const float* base = gx + (static_cast<size_t>(slot) * 2 + ((nex - 1u) & 1u)) * kBJSplit * (kBJP * kBJP);
          for (int e = tid; e < kBJP * kBJP; e += blockDim.x) {
            float v = __ldcg(base + e);
#pragma unroll
            for (int q = 1; q < kBJSplit; ++q) v += __ldcg(base + q * (kBJP * kBJP) + e);
            sh.M[e / kBJP][e % kBJP] = v;
          }
        }
        if (tid == 0) sh.rotate = 0;
        __syncthreads();
        // ---- already orthogonal to tol?  (and the sweep's largest relative
        // off-diagonal entry, for the stopping rule)
        {
          float worst = 0.f;
          for (int e = tid; e < kBJP * kBJP; e += blockDim.x) {
            const int p = e / kBJP, q = e % kBJP;
            if (p < q) {
              const float dd = sh.M[p][p] * sh.M[q][q];
              const float rel = dd > 0.f ? fabsf(sh.M[p][q]) * rsqrtf(sh.M[p][p]) * rsqrtf(sh.M[q][q]) : 0.f;
              if (rel > tol) sh.rotate = 1;
              worst = fmaxf(worst, rel);
            }
          }
          for (int o = 16; o > 0; o >>= 1) worst = fmaxf(worst, __shfl_xor_sync(0xFFFFFFFFu, worst, o));
          if (sub == 0 && (tid & 31) == 0 && worst > 0.f) atomicMax(bar + 4, __float_as_uint(worst));
        }
        __syncthreads();
        if (!sh.rotate) continue;
        bj_inner_sweep(sh);
        bj_reorthogonalize(sh);
        // ---- this slice of the pair's columns (and V's) becomes A J
        bj_apply_slice(sh, Xr, kps, At, ld, I, Jb, k, c_lo, cw);
        if (Vt) {
          __syncthreads();
          bj_load_slice(Xr, kps, Vt, ld, I, Jb, k, c_lo, cw);
          bj_apply_slice(sh, Xr, kps, Vt, ld, I, Jb, k, c_lo, cw);
        }
        if (sub == 0 && tid == 0) atomicAdd(rot, 1u);
      }
      if (!grid_barrier(bar, gridDim.x, status)) return;
    }
    const unsigned rotations = *reinterpret_cast<volatile unsigned*>(rot);
    const float worst = __uint_as_float(*reinterpret_cast<volatile unsigned*>(bar + 4));
    if (!grid_barrier(bar, gridDim.x, status)) return;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      atomicExch(rot, 0u);
      atomicExch(bar + 4, 0u);
    }
    if (!grid_barrier(bar, gridDim.x, status)) return;
    if (rotations == 0 || worst <= kBJStopTol) {
      ++sweep;
      break;
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && sweeps_out) *sweeps_out = sweep;
}

}  // namespace qg
