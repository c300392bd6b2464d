// Internal interface of the subspace refresh (randomized top-r SVD, INT4
// quantization of the new projection, CosSim against the previous one).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qgalore.h"

namespace qg {

constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusNonFinite = 2u;

struct RefreshArgs {
  const void* G;  // m x ldg bf16
  int64_t ldg;
  int32_t m, n, r, oversample, power_iters;
  uint64_t seed;
  uint32_t refresh_idx, layer_id;
  uint8_t* Pq;  // out: new INT4 projection (current slot of the state)
  float* sP;
  uint8_t* Pq_prev;  // the previous projection is moved here when has_prev
  float* sP_prev;
  int32_t has_prev;
  uint32_t* status;
  // the layer's INT8 moments, for cfg.mom_refresh (0 keep, 1 reset, 2 rotate)
  int32_t mom_refresh;
  int8_t* Mq;
  int8_t* Vq;
  float* sM;
  float* sV;
  int64_t ld_mom;
  int32_t nblk;
  int32_t mom_rows, mom_cols;  // the moments' shape (that of R)
  // 1 for the right-side projection: m and n above are then the rows of P
  // (the layer's n) and the layer's m, and the refresh works on G^T
  int32_t transpose_g;
};

size_t refresh_scratch_bytes(int32_t m, int32_t n, int32_t r, int32_t oversample);
size_t cossim_scratch_bytes(int32_t m, int32_t r);

// Enqueues the refresh on `stream`; when has_prev, also CosSim, and waits for
// the stream to read it into *cossim.
qg_status run_refresh(const RefreshArgs& a, uint8_t* ws, size_t ws_bytes, cudaStream_t stream, float* cossim);

// CosSim of two float32 m x r matrices (row stride ld) into d_out[0].
qg_status run_cossim(const float* Pa, const float* Pb, int32_t m, int32_t r, int64_t ld, float* d_out, uint8_t* ws,
                     cudaStream_t stream);

}  // namespace qg
