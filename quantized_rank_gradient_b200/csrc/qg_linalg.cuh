// Small dense linear algebra for the subspace refresh (float32, SIMT):
//   sgemm_kernel        C = op(A) op(B) (64 x 64 tiles, 4 x 4 outputs per thread)
//   potrf_diag_kernel   Cholesky of one 32 x 32 diagonal block + its inverse
//   trsm_panel_kernel   L[i, jb] = A[i, jb] * inv(L[jb, jb])^T below the block
//   syrk_update_kernel  trailing update A -= L[:, jb] L[:, jb]^T (lower tiles)
//   trsm_rows_kernel    X <- X L^-T for a tall X, 32 rows per CTA
//   jacobi_kernel       one-sided (Hestenes) Jacobi on the columns of a square
//                       matrix, round-robin pairs, one warp per pair, a bounded
//                       grid barrier between rounds (cooperative launch)
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

// ------------------------------------------------------------------ Cholesky

// Cholesky of the nb x nb diagonal block at (j0, j0) of the lower triangle of A
// (read from the lower triangle only), written back as L; its inverse (32 x 32,
// lower, identity-padded) goes to Linv.  A pivot that is not positive (the
// matrix is not numerically positive definite) raises *flag and is replaced by
// a tiny positive value so that the factorisation stays finite.
__global__ void __launch_bounds__(1024) potrf_diag_kernel(float* A, int64_t ld, int j0, int nb, float* Linv,
                                                          int* flag) {
  __shared__ float T[32][33];
  __shared__ float X[32][33];
  const int i = threadIdx.y, j = threadIdx.x;
  float v = (i == j) ? 1.f : 0.f;
  if (i < nb && j < nb && j <= i) v = A[static_cast<int64_t>(j0 + i) * ld + j0 + j];
  T[i][j] = (j <= i) ? v : 0.f;
  __syncthreads();
  for (int c = 0; c < 32; ++c) {
    if (i == c && j == c) {
      float d = T[c][c];
      if (!(d > 0.f)) {
        if (c < nb) atomicOr(flag, 1);
        d = 1e-30f;
      }
      T[c][c] = sqrtf(d);
    }
    __syncthreads();
    if (j == c && i > c) T[i][c] = T[i][c] / T[c][c];
    __syncthreads();
    if (i > c && j > c && j <= i) T[i][j] = T[i][j] - T[i][c] * T[j][c];
    __syncthreads();
  }
  if (i < nb && j < nb) A[static_cast<int64_t>(j0 + i) * ld + j0 + j] = (j <= i) ? T[i][j] : 0.f;
  // inverse: column j of inv(T) by forward substitution (thread row 0 of each column)
  if (i == 0) {
    for (int r = 0; r < 32; ++r) {
      float s = (r == j) ? 1.f : 0.f;
      for (int t = j; t < r; ++t) s -= T[r][t] * X[t][j];
      X[r][j] = (r >= j) ? s / T[r][r] : 0.f;
    }
  }
  __syncthreads();
  Linv[i * 32 + j] = X[i][j];
}

// L[i, j0 + c] = sum_c' A[i, j0 + c'] Linv[c][c'] for rows i >= j0 + 32.
__global__ void __launch_bounds__(1024) trsm_panel_kernel(float* A, int64_t ld, int j0, int n, const float* Linv) {
  __shared__ float R[32][33];
  __shared__ float Li[32][33];
  const int r = threadIdx.y, c = threadIdx.x;
  const int row = j0 + 32 + blockIdx.x * 32 + r;
  Li[r][c] = Linv[r * 32 + c];
  R[r][c] = (row < n && j0 + c < n) ? A[static_cast<int64_t>(row) * ld + j0 + c] : 0.f;
  __syncthreads();
  float s = 0.f;
  for (int t = 0; t <= c; ++t) s = __fmaf_rn(R[r][t], Li[c][t], s);
  if (row < n && j0 + c < n) A[static_cast<int64_t>(row) * ld + j0 + c] = s;
}

// A[i, l] -= sum_t L[i, j0 + t] L[l, j0 + t] over the lower tiles of the
// trailing matrix (rows and columns >= j0 + 32).
__global__ void __launch_bounds__(1024) syrk_update_kernel(float* A, int64_t ld, int j0, int n) {
  // blockIdx.x enumerates the lower tiles (ti >= tl) of the trailing part
  int t = blockIdx.x, ti = 0;
  while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
  const int tl = t - ti * (ti + 1) / 2;
  __shared__ float Li[32][33];
  __shared__ float Ll[32][33];
  const int r = threadIdx.y, c = threadIdx.x;
  const int base = j0 + 32;
  const int ri = base + ti * 32 + r, rl = base + tl * 32 + r;
  Li[r][c] = (ri < n) ? A[static_cast<int64_t>(ri) * ld + j0 + c] : 0.f;
  Ll[r][c] = (rl < n) ? A[static_cast<int64_t>(rl) * ld + j0 + c] : 0.f;
  __syncthreads();
  const int gi = base + ti * 32 + r, gl = base + tl * 32 + c;
  if (gi < n && gl < n && gl <= gi) {
    float s = 0.f;
    for (int q = 0; q < 32; ++q) s = __fmaf_rn(Li[r][q], Ll[c][q], s);
    float* a = A + static_cast<int64_t>(gi) * ld + gl;
    *a = *a - s;
  }
}

// X (rows x k, row stride ldx) <- X L^-T, i.e. solves Y L^T = X row by row, with
// L the lower Cholesky factor (k x k, stride ldl) and Linv the inverses of its
// 32 x 32 diagonal blocks.  Each CTA owns 32 rows kept in shared memory; also
// writes a bf16 copy (stride ldb) when Xb is non-null and, when Xlo is
// non-null, the bf16 rounding of the residual X - Xb (so that Xb + Xlo carries
// about 16 significant bits).
__global__ void __launch_bounds__(256) trsm_rows_kernel(float* X, int64_t ldx, uint16_t* Xb, uint16_t* Xlo,
                                                        int64_t ldb, int rows, int k, const float* L, int64_t ldl,
                                                        const float* Linv) {
  extern __shared__ float Ys[];  // 32 x (k + 1)
  const int kp = k + 1;
  const int r0 = blockIdx.x * 32;
  const int tid = threadIdx.x;
  for (int e = tid; e < 32 * k; e += 256) {
    const int i = e / k, c = e % k;
    Ys[i * kp + c] = (r0 + i < rows) ? X[static_cast<int64_t>(r0 + i) * ldx + c] : 0.f;
  }
  __syncthreads();
  __shared__ float acc_s[32][33];
  const int i = tid & 31;        // row in the CTA
  const int cg = tid >> 5;       // 4 columns: cg*4 .. cg*4+3 of the block
  const int nblk = (k + 31) / 32;
  for (int jb = 0; jb < nblk; ++jb) {
    const int c0 = jb * 32;
    float acc[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + cg * 4 + u;
      float s = (c < k) ? Ys[i * kp + c] : 0.f;
      if (c < k) {
        const float* lrow = L + static_cast<int64_t>(c) * ldl;
        for (int t = 0; t < c0; ++t) s = __fmaf_rn(-Ys[i * kp + t], lrow[t], s);
      }
      acc[u] = s;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) acc_s[i][cg * 4 + u] = acc[u];
    __syncthreads();
    const float* li = Linv + static_cast<int64_t>(jb) * 1024;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int cl = cg * 4 + u, c = c0 + cl;
      float s = 0.f;
      for (int t = 0; t <= cl; ++t) s = __fmaf_rn(acc_s[i][t], li[cl * 32 + t], s);
      if (c < k) Ys[i * kp + c] = s;
    }
    __syncthreads();
  }
  for (int e = tid; e < 32 * k; e += 256) {
    const int ii = e / k, c = e % k;
    if (r0 + ii < rows) {
      const float y = Ys[ii * kp + c];
      X[static_cast<int64_t>(r0 + ii) * ldx + c] = y;
      if (Xb) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(y);
        Xb[static_cast<int64_t>(r0 + ii) * ldb + c] = __bfloat16_as_ushort(hi);
        if (Xlo)
          Xlo[static_cast<int64_t>(r0 + ii) * ldb + c] =
              __bfloat16_as_ushort(__float2bfloat16_rn(__fsub_rn(y, __bfloat162float(hi))));
      }
    }
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

// One-sided Jacobi: rotates pairs of columns of A (k x k, stored transposed:
// row p of At is column p of A, stride ld) until every pair is orthogonal to
// |a_p . a_q| <= tol * |a_p| |a_q|; applies the same rotations to V (rows of
// Vt) when Vt is non-null.  Round-robin pairing (player 0 fixed, the others
// rotate): every pair meets once per sweep of kk - 1 rounds (kk = k rounded up
// to even; the dummy player pairs with nobody).  bar[3] counts the rotations of
// the current sweep.  Stops after a sweep with no rotation or max_sweeps.
__global__ void __launch_bounds__(256) jacobi_kernel(float* At, float* Vt, int64_t ld, int k, int max_sweeps,
                                                     float tol, unsigned* bar, int* sweeps_out, uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int warps_per_block = blockDim.x >> 5;
  const int gwarp = blockIdx.x * warps_per_block + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * warps_per_block;
  const int kk = (k + 1) & ~1;
  unsigned* rot = bar + 3;
  int sweep = 0;
  for (; sweep < max_sweeps; ++sweep) {
    for (int round = 0; round < kk - 1; ++round) {
      for (int idx = gwarp; idx < kk / 2; idx += nwarps) {
        const int a = idx, b = kk - 1 - idx;
        const int p = (a == 0) ? 0 : ((a - 1 + round) % (kk - 1)) + 1;
        const int q = ((b - 1 + round) % (kk - 1)) + 1;
        if (p >= k || q >= k) continue;
        float* ap = At + static_cast<int64_t>(p) * ld;
        float* aq = At + static_cast<int64_t>(q) * ld;
        float al = 0.f, be = 0.f, ga = 0.f;
        // columns are rewritten by other SMs between rounds: bypass L1
        for (int t = lane; t < k; t += 32) {
          const float x = __ldcg(ap + t), y = __ldcg(aq + t);
          al = __fmaf_rn(x, x, al);
          be = __fmaf_rn(y, y, be);
          ga = __fmaf_rn(x, y, ga);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          al += __shfl_xor_sync(0xFFFFFFFFu, al, o);
          be += __shfl_xor_sync(0xFFFFFFFFu, be, o);
          ga += __shfl_xor_sync(0xFFFFFFFFu, ga, o);
        }
        if (!(fabsf(ga) > tol * sqrtf(al) * sqrtf(be))) continue;
        const float zeta = (be - al) / (2.f * ga);
        const float tt = fabsf(zeta) < 1e18f ? copysignf(1.f, zeta) / (fabsf(zeta) + sqrtf(1.f + zeta * zeta))
                                             : 0.5f / zeta;
        const float c = 1.f / sqrtf(1.f + tt * tt);
        const float s = c * tt;
        for (int t = lane; t < k; t += 32) {
          const float x = __ldcg(ap + t), y = __ldcg(aq + t);
          __stcg(ap + t, c * x - s * y);
          __stcg(aq + t, s * x + c * y);
        }
        if (Vt) {
          float* vp = Vt + static_cast<int64_t>(p) * ld;
          float* vq = Vt + static_cast<int64_t>(q) * ld;
          for (int t = lane; t < k; t += 32) {
            const float x = __ldcg(vp + t), y = __ldcg(vq + t);
            __stcg(vp + t, c * x - s * y);
            __stcg(vq + t, s * x + c * y);
          }
        }
        if (lane == 0) atomicAdd(rot, 1u);
      }
      if (!grid_barrier(bar, gridDim.x, status)) return;
    }
    const unsigned rotations = *reinterpret_cast<volatile unsigned*>(rot);
    if (!grid_barrier(bar, gridDim.x, status)) return;
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicExch(rot, 0u);
    if (!grid_barrier(bar, gridDim.x, status)) return;
    if (rotations == 0) {
      ++sweep;
      break;
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && sweeps_out) *sweeps_out = sweep;
}

}  // namespace qg
