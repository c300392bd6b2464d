// Device-time accounting of the library's own launches (qg_profile_enable /
// qg_profile_collect): CUDA events recorded on the launch stream around each
// kernel, summed per kernel kind when collected.
#include <mutex>
#include <vector>

#include "../../include/qgalore.h"
#include "qg_internal.h"

namespace qg {

namespace {

struct Record {
  int kind;
  cudaEvent_t start, stop;
  double flops, bytes;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Record> g_records;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

int profile_begin(cudaStream_t s, int kind, double flops, double bytes) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on) return -1;
  Record r{kind, take_event(), take_event(), flops, bytes};
  if (!r.start || !r.stop) return -1;
  cudaEventRecord(r.start, s);
  g_records.push_back(r);
  return static_cast<int>(g_records.size()) - 1;
}

void profile_end(cudaStream_t s, int token) {
  if (token < 0) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (token < static_cast<int>(g_records.size())) cudaEventRecord(g_records[token].stop, s);
}

}  // namespace qg

extern "C" {

qg_status qg_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(qg::g_mu);
  for (auto& r : qg::g_records) {
    qg::g_pool.push_back(r.start);
    qg::g_pool.push_back(r.stop);
  }
  qg::g_records.clear();
  qg::g_on = on != 0;
  return QG_OK;
}

qg_status qg_profile_collect(qg_kernel_times* out, int32_t kinds) {
  if (!out || kinds <= 0) return QG_EINVAL;
  for (int k = 0; k < kinds; ++k) out[k] = qg_kernel_times{0, 0.0, 0.0, 0.0};
  std::lock_guard<std::mutex> lk(qg::g_mu);
  for (auto& r : qg::g_records) {
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return QG_ECUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) return QG_ECUDA;
    if (r.kind < 0 || r.kind >= kinds) continue;
    out[r.kind].launches += 1;
    out[r.kind].device_ms += ms;
    out[r.kind].flops += r.flops;
    out[r.kind].bytes += r.bytes;
  }
  return QG_OK;
}

}  // extern "C"
