// Internal interface between the C ABI (qg_api.cu) and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace qg {

// Everything one matrix's step a1..a5 reads and writes (device pointers).
struct StepProblem {
  const uint8_t* Pq;    // m*r/2 packed INT4 codes
  const float* sP;      // m*r/64 scales
  const void* G;        // m x ldg bf16
  int64_t ldg;
  int8_t* Mq;           // R's shape (r x n, or m x r for the right side), row stride ld_mom
  int8_t* Vq;
  float* sM;            // r x nblk
  float* sV;
  int64_t ld_mom;
  int32_t nblk;
  int8_t* W;            // m x ldw
  int64_t ldw;
  float* sW;            // ceil(m*n/256); grows in place where w_rescale = 1
  uint16_t* Pbf;        // scratch: P~ (m x r bf16, or n x r for the right side)
  uint16_t* Nbuf;       // scratch: N (R's shape, bf16, row stride ldN)
  int64_t ldN;
  int32_t m, n, r;
  int32_t side;         // 0: P m x r, R = P^T G (r x n); 1: P n x r, R = G P (m x r)
  int32_t w_rescale;    // 1: a weight group leaving the INT8 grid is re-scaled (n % 256 == 0)
  float beta1, beta2, om1, om2, c1, c2, eps, alpha;  // c1 = -lr/(1-b1^t), c2 = 1/sqrt(1-b2^t)
  uint32_t t, layer_id;
  uint64_t seed;
  uint32_t* status;
};

// Scratch layout of one step: P~ (m x r bf16) then N (r x ldN bf16), each
// starting on a 256-byte boundary.
int64_t step_ldN(int32_t n);
size_t step_scratch_bytes(int32_t m, int32_t n, int32_t r, int32_t side);

// Enqueues a1..a5 for `count` problems on `stream`.  Returns cudaSuccess or the
// first launch / set-up error.
cudaError_t launch_step(const StepProblem* probs, int count, cudaStream_t stream);

cudaError_t launch_dequant_projection(const uint8_t* Pq, const float* sP, int64_t total,
                                      uint16_t* out, cudaStream_t stream);
cudaError_t launch_philox(const uint32_t* c0, const uint32_t* c1, const uint32_t* c2,
                          const uint32_t* c3, int64_t count, uint32_t k0, uint32_t k1, uint32_t* out,
                          cudaStream_t stream);
// D = A B (or D += A B when accumulate), bf16 operands on the tcgen05 core.
cudaError_t launch_gemm_f32(const void* A, int64_t lda, bool a_trans, const void* B, int64_t ldb,
                            bool b_trans, float* D, int64_t ldd, int M, int N, int K,
                            cudaStream_t stream, bool accumulate = false);

// Tensor-map encoder (driver entry point, resolved once).  Returns false when
// the driver refuses the map.
bool encode_map_bf16(void* map, const void* base, uint64_t inner, uint64_t outer, uint64_t ld_elems,
                     uint32_t box_inner, uint32_t box_outer);

int sm_count();

// Launch accounting (qg_profile.cu): returns a token for profile_end, or -1
// when accounting is off.  `kind` is a qg_kernel_kind.
int profile_begin(cudaStream_t s, int kind, double flops, double bytes);
void profile_end(cudaStream_t s, int token);

cudaError_t launch_quantize_projection(const float* P, int64_t ld, int32_t m, int32_t r, uint8_t* Pq, float* sP,
                                       cudaStream_t stream);

}  // namespace qg
