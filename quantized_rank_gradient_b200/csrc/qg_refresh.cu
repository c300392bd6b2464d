// Subspace refresh on sm_100a (being built).
#include "qg_refresh.h"
#include "qg_internal.h"

namespace qg {

size_t refresh_scratch_bytes(int32_t, int32_t, int32_t, int32_t) { return 256; }
size_t cossim_scratch_bytes(int32_t, int32_t) { return 256; }

qg_status run_refresh(const RefreshArgs&, uint8_t*, size_t, cudaStream_t, float*) { return QG_ESHAPE; }

qg_status run_cossim(const float*, const float*, int32_t, int32_t, int64_t, float*, uint8_t*, cudaStream_t) {
  return QG_ESHAPE;
}

}  // namespace qg
