// Subspace refresh on sm_100a: INT4 quantization of a projection (being
// extended to the full randomized top-r SVD and CosSim).
#include "qg_device.cuh"
#include "qg_internal.h"
#include "qg_refresh.h"

namespace qg {

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
  const bool live = amax >= 7.52316384526264e-37f;
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

size_t refresh_scratch_bytes(int32_t, int32_t, int32_t, int32_t) { return 256; }
size_t cossim_scratch_bytes(int32_t, int32_t) { return 256; }

qg_status run_refresh(const RefreshArgs&, uint8_t*, size_t, cudaStream_t, float*) { return QG_ESHAPE; }

qg_status run_cossim(const float*, const float*, int32_t, int32_t, int64_t, float*, uint8_t*, cudaStream_t) {
  return QG_ESHAPE;
}

}  // namespace qg
