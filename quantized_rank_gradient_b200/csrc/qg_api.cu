// C ABI of the library (declared in include/qgalore.h): argument validation,
// carving of the caller's state buffer, the host side of the layer-adaptive
// schedule, and the launches.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "../../include/qgalore.h"
#include "qg_internal.h"
#include "qg_refresh.h"

using qg::StepProblem;

struct qg_layer {
  qg_config cfg;
  uint8_t* state;
  size_t state_bytes;
  int8_t* W;
  int64_t ldw;
  float* sW;
  qg_layer_views v;
  qg_sched sched;
};

namespace {

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct StateLayout {
  size_t status, Pq, sP, Pq_prev, sP_prev, Mq, Vq, sM, sV, total;
  int64_t ld_mom;
  int32_t nblk;
  int32_t p_rows, mom_rows, mom_cols;
};

// Rows of P, and the moments' shape (that of R): P m x r and R r x n for the
// left projection; P n x r and R m x r for the right one.
void proj_dims(const qg_config& c, int32_t* p_rows, int32_t* rows, int32_t* cols) {
  *p_rows = c.proj_side ? c.n : c.m;
  *rows = c.proj_side ? c.m : c.r;
  *cols = c.proj_side ? c.r : c.n;
}

StateLayout state_layout(const qg_config& c) {
  StateLayout L;
  proj_dims(c, &L.p_rows, &L.mom_rows, &L.mom_cols);
  const size_t mr = static_cast<size_t>(L.p_rows) * c.r;
  const size_t pq = (mr + 1) / 2;
  const size_t ps = ((mr + 63) / 64) * sizeof(float);
  L.ld_mom = (static_cast<int64_t>(L.mom_cols) + 31) / 32 * 32;
  L.nblk = (L.mom_cols + 255) / 256;
  size_t off = 0;
  L.status = off;
  off += 256;
  L.Pq = off;
  off += round256(pq);
  L.sP = off;
  off += round256(ps);
  L.Pq_prev = off;
  off += round256(pq);
  L.sP_prev = off;
  off += round256(ps);
  L.Mq = off;
  off += round256(static_cast<size_t>(L.mom_rows) * L.ld_mom);
  L.Vq = off;
  off += round256(static_cast<size_t>(L.mom_rows) * L.ld_mom);
  L.sM = off;
  off += round256(static_cast<size_t>(L.mom_rows) * L.nblk * sizeof(float));
  L.sV = off;
  off += round256(static_cast<size_t>(L.mom_rows) * L.nblk * sizeof(float));
  L.total = off;
  return L;
}

qg_status check_config(const qg_config* c) {
  if (!c) return QG_EINVAL;
  if (c->m <= 0 || c->n <= 0 || c->r <= 0) return QG_ESHAPE;
  if (c->r % 32 != 0 || c->r > c->m || c->r > c->n) return QG_ESHAPE;
  if (static_cast<int64_t>(c->m) * c->n >= (int64_t(1) << 40)) return QG_ESHAPE;
  if (c->m >= (1 << 30) || c->n >= (1 << 30)) return QG_ESHAPE;
  // the projection's INT4 codes are indexed by 32-bit words (8 codes each)
  if (static_cast<int64_t>(c->m > c->n ? c->m : c->n) * c->r >= (int64_t(1) << 34)) return QG_ESHAPE;
  if (c->w_group != 256 || c->p_group != 64 || c->mom_block != 256) return QG_ESHAPE;
  if (!(c->beta1 >= 0.f && c->beta1 < 1.f) || !(c->beta2 >= 0.f && c->beta2 < 1.f)) return QG_EINVAL;
  if (!(c->eps > 0.f) || !isfinite(c->eps) || !isfinite(c->lr) || !isfinite(c->alpha)) return QG_EINVAL;
  if (!isfinite(c->gamma) || c->delta0 < 1 || c->oversample < 0 || c->power_iters < 0) return QG_EINVAL;
  if (c->mom_refresh < 0 || c->mom_refresh > 2) return QG_EINVAL;
  if (c->proj_side < 0 || c->proj_side > 1) return QG_EINVAL;
  if (c->w_rescale < 0 || c->w_rescale > 1) return QG_EINVAL;
  if (c->w_rescale && c->n % 256 != 0) return QG_ESHAPE;
  return QG_OK;
}

qg_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QG_OK : QG_ECUDA; }

void fill_step_problem(const qg_layer* L, const void* G, int64_t ldg, uint8_t* ws, int64_t t, StepProblem* s) {
  const qg_config& c = L->cfg;
  memset(s, 0, sizeof(*s));
  s->Pq = L->v.Pq;
  s->sP = L->v.sP;
  s->G = G;
  s->ldg = ldg;
  s->Mq = L->v.Mq;
  s->Vq = L->v.Vq;
  s->sM = L->v.sM;
  s->sV = L->v.sV;
  s->ld_mom = L->v.ld_mom;
  s->nblk = L->v.nblk;
  s->W = L->W;
  s->ldw = L->ldw;
  s->sW = L->sW;
  s->Pbf = reinterpret_cast<uint16_t*>(ws);
  s->Nbuf = reinterpret_cast<uint16_t*>(ws + round256(static_cast<size_t>(L->v.p_rows) * c.r * 2));
  s->ldN = qg::step_ldN(L->v.mom_cols);
  s->m = c.m;
  s->n = c.n;
  s->r = c.r;
  s->side = c.proj_side;
  s->w_rescale = c.w_rescale;
  const double b1 = static_cast<double>(c.beta1);
  const double b2 = static_cast<double>(c.beta2);
  s->beta1 = c.beta1;
  s->beta2 = c.beta2;
  s->om1 = static_cast<float>(1.0 - b1);
  s->om2 = static_cast<float>(1.0 - b2);
  s->c1 = static_cast<float>(-static_cast<double>(c.lr) / (1.0 - pow(b1, static_cast<double>(t))));
  s->c2 = static_cast<float>(1.0 / sqrt(1.0 - pow(b2, static_cast<double>(t))));
  s->eps = c.eps;
  s->alpha = c.alpha;
  s->t = static_cast<uint32_t>(t);
  s->layer_id = c.layer_id;
  s->seed = c.seed;
  s->status = L->v.status;
}

qg_status check_step_args(const qg_layer* L, const void* G, int64_t ldg) {
  if (!L || !G) return QG_EINVAL;
  if (!L->sched.has_projection) return QG_ESTATE;
  if (ldg < L->cfg.n || ldg % 8 != 0 || !aligned(G, 16)) return QG_EALIGN;
  if (L->sched.t + 1 >= (int64_t(1) << 32)) return QG_ESTATE;
  return QG_OK;
}

}  // namespace

namespace qg {
qg_status layer_config(const qg_layer* layer, qg_config* out) {
  if (!layer || !out) return QG_EINVAL;
  *out = layer->cfg;
  return QG_OK;
}
}  // namespace qg

extern "C" {

const char* qg_status_str(qg_status s) {
  switch (s) {
    case QG_OK: return "ok";
    case QG_EINVAL: return "invalid argument";
    case QG_ESHAPE: return "unsupported shape";
    case QG_EALIGN: return "misaligned pointer or leading dimension";
    case QG_ESTATE: return "buffer too small or layer not ready";
    case QG_ECUDA: return "CUDA error";
    case QG_ETIMEOUT: return "device wait timed out";
    case QG_ENONFINITE: return "non-finite value";
  }
  return "unknown status";
}

void qg_config_default(qg_config* c, int32_t m, int32_t n, int32_t r) {
  if (!c) return;
  memset(c, 0, sizeof(*c));
  c->m = m;
  c->n = n;
  c->r = r;
  c->w_group = 256;
  c->p_group = 64;
  c->mom_block = 256;
  c->beta1 = 0.9f;
  c->beta2 = 0.999f;
  c->eps = 1e-8f;
  c->lr = 1e-3f;
  c->alpha = 0.25f;
  c->gamma = 0.4f;
  c->delta0 = 200;
  c->oversample = 16;
  c->power_iters = 2;
  c->seed = 0;
  c->layer_id = 0;
}

size_t qg_state_bytes(const qg_config* cfg) {
  if (check_config(cfg) != QG_OK) return 0;
  return state_layout(*cfg).total;
}

size_t qg_step_workspace_bytes(const qg_config* cfg) {
  if (check_config(cfg) != QG_OK) return 0;
  return qg::step_scratch_bytes(cfg->m, cfg->n, cfg->r, cfg->proj_side);
}

size_t qg_refresh_workspace_bytes(const qg_config* cfg) {
  if (check_config(cfg) != QG_OK) return 0;
  const int32_t pm = cfg->proj_side ? cfg->n : cfg->m, pn = cfg->proj_side ? cfg->m : cfg->n;
  return qg::refresh_scratch_bytes(pm, pn, cfg->r, cfg->oversample);
}

qg_status qg_layer_init(qg_layer** out, const qg_config* cfg, void* d_state, size_t state_bytes, int8_t* d_W,
                        int64_t ldw, float* d_Wscale, void* stream) {
  if (!out) return QG_EINVAL;
  *out = nullptr;
  qg_status st = check_config(cfg);
  if (st != QG_OK) return st;
  if (!d_state || !d_W || !d_Wscale) return QG_EINVAL;
  if (!aligned(d_state, 256) || !aligned(d_W, 16) || !aligned(d_Wscale, 4)) return QG_EALIGN;
  if (ldw < cfg->n || ldw % 16 != 0) return QG_EALIGN;
  const StateLayout SL = state_layout(*cfg);
  if (state_bytes < SL.total) return QG_ESTATE;
  qg_layer* L = static_cast<qg_layer*>(calloc(1, sizeof(qg_layer)));
  if (!L) return QG_EINVAL;
  L->cfg = *cfg;
  L->state = static_cast<uint8_t*>(d_state);
  L->state_bytes = state_bytes;
  L->W = d_W;
  L->ldw = ldw;
  L->sW = d_Wscale;
  uint8_t* b = L->state;
  L->v.status = reinterpret_cast<uint32_t*>(b + SL.status);
  L->v.Pq = b + SL.Pq;
  L->v.sP = reinterpret_cast<float*>(b + SL.sP);
  L->v.Pq_prev = b + SL.Pq_prev;
  L->v.sP_prev = reinterpret_cast<float*>(b + SL.sP_prev);
  L->v.Mq = reinterpret_cast<int8_t*>(b + SL.Mq);
  L->v.Vq = reinterpret_cast<int8_t*>(b + SL.Vq);
  L->v.sM = reinterpret_cast<float*>(b + SL.sM);
  L->v.sV = reinterpret_cast<float*>(b + SL.sV);
  L->v.ld_mom = SL.ld_mom;
  L->v.nblk = SL.nblk;
  L->v.p_rows = SL.p_rows;
  L->v.mom_rows = SL.mom_rows;
  L->v.mom_cols = SL.mom_cols;
  L->sched.t = 0;
  L->sched.delta = cfg->delta0;
  L->sched.t_next = 0;
  L->sched.n_refresh = 0;
  L->sched.has_projection = 0;
  if (cudaMemsetAsync(d_state, 0, SL.total, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    free(L);
    return QG_ECUDA;
  }
  *out = L;
  return QG_OK;
}

qg_status qg_layer_destroy(qg_layer* L) {
  free(L);
  return QG_OK;
}

qg_status qg_layer_views_get(const qg_layer* L, qg_layer_views* v) {
  if (!L || !v) return QG_EINVAL;
  *v = L->v;
  return QG_OK;
}

qg_status qg_layer_sched_get(const qg_layer* L, qg_sched* s) {
  if (!L || !s) return QG_EINVAL;
  *s = L->sched;
  return QG_OK;
}

qg_status qg_layer_sched_set(qg_layer* L, const qg_sched* s) {
  if (!L || !s) return QG_EINVAL;
  if (s->t < 0 || s->delta < 1 || s->t_next < 0 || s->n_refresh < 0) return QG_EINVAL;
  L->sched = *s;
  return QG_OK;
}

qg_status qg_layer_set_projection(qg_layer* L, const uint8_t* d_Pq, const float* d_sP, int32_t keep_prev,
                                  void* stream) {
  if (!L || !d_Pq || !d_sP) return QG_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t mr = static_cast<size_t>(L->v.p_rows) * L->cfg.r;
  const size_t pq = (mr + 1) / 2, ps = ((mr + 63) / 64) * sizeof(float);
  if (keep_prev && L->sched.has_projection) {
    if (cudaMemcpyAsync(L->v.Pq_prev, L->v.Pq, pq, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return QG_ECUDA;
    if (cudaMemcpyAsync(L->v.sP_prev, L->v.sP, ps, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return QG_ECUDA;
  }
  if (cudaMemcpyAsync(L->v.Pq, d_Pq, pq, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return QG_ECUDA;
  if (cudaMemcpyAsync(L->v.sP, d_sP, ps, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return QG_ECUDA;
  L->sched.has_projection = 1;
  return QG_OK;
}

qg_status qg_step(qg_layer* L, const void* d_G, int64_t ldg, void* d_ws, size_t ws_bytes, void* stream) {
  qg_status st = check_step_args(L, d_G, ldg);
  if (st != QG_OK) return st;
  if (!d_ws) return QG_EINVAL;
  if (!aligned(d_ws, 256)) return QG_EALIGN;
  if (ws_bytes < qg::step_scratch_bytes(L->cfg.m, L->cfg.n, L->cfg.r, L->cfg.proj_side)) return QG_ESTATE;
  const int64_t t = L->sched.t + 1;
  StepProblem sp;
  fill_step_problem(L, d_G, ldg, static_cast<uint8_t*>(d_ws), t, &sp);
  st = cuda_status(qg::launch_step(&sp, 1, static_cast<cudaStream_t>(stream)));
  if (st == QG_OK) L->sched.t = t;
  return st;
}

// Batches and lanes.  The matrices go in batches of up to kBatch (three
// launches per batch: one dequantization grid, one persistent grid per GEMM
// stage).  Batches take turns among kLanes lanes, the caller's stream and
// kLanes - 1 streams the library keeps per device, and each lane reuses one
// workspace slot as large as the largest batch's scratch.  The lanes' kernels
// overlap, so the SMs that one batch's last wave of tiles leaves idle take
// tiles of another lane's batch.  The lanes fork from and join back to the
// caller's stream through events: the call is ordered on `stream` like a plain
// launch sequence and can be captured into a CUDA graph.
static constexpr int kBatch = 8;
// measured on the LLaMA stacks: three lanes 2 % (1B) and 0.5 % (7B) faster than
// two, four no faster than three
static constexpr int kLanes = 3;
static constexpr int kMaxDevices = 64;

struct Lane {
  cudaStream_t s[kLanes - 1] = {};
  cudaEvent_t fork = nullptr;
  cudaEvent_t join[kLanes - 1] = {};
};
static std::mutex g_lane_mu;  // guards g_lane and each fork / launch / join sequence
static Lane g_lane[kMaxDevices];

// The current device's extra lanes, created on first use.
static qg_status extra_lanes(Lane** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QG_ECUDA;
  Lane& L = g_lane[dev];
  if (!L.fork) {
    for (int i = 0; i < kLanes - 1; ++i) {
      if (cudaStreamCreateWithFlags(&L.s[i], cudaStreamNonBlocking) != cudaSuccess) return QG_ECUDA;
      if (cudaEventCreateWithFlags(&L.join[i], cudaEventDisableTiming) != cudaSuccess) return QG_ECUDA;
    }
    if (cudaEventCreateWithFlags(&L.fork, cudaEventDisableTiming) != cudaSuccess) return QG_ECUDA;
  }
  *out = &L;
  return QG_OK;
}

static size_t batch_slot_bytes(const int32_t* m, const int32_t* n, const int32_t* r, const int32_t* side,
                               int count) {
  size_t slot = 0;
  for (int b = 0; b * kBatch < count; ++b) {
    size_t sum = 0;
    for (int i = b * kBatch; i < count && i < (b + 1) * kBatch; ++i)
      sum += qg::step_scratch_bytes(m[i], n[i], r[i], side[i]);
    slot = std::max(slot, sum);
  }
  return slot;
}

static int batch_lanes(int count) { return std::min(kLanes, (count + kBatch - 1) / kBatch); }

size_t qg_step_batch_workspace_bytes(const qg_config* const* cfgs, int32_t count) {
  if (!cfgs || count < 0) return 0;
  std::vector<int32_t> m(count), n(count), r(count), side(count);
  for (int i = 0; i < count; ++i) {
    if (check_config(cfgs[i]) != QG_OK) return 0;
    m[i] = cfgs[i]->m, n[i] = cfgs[i]->n, r[i] = cfgs[i]->r, side[i] = cfgs[i]->proj_side;
  }
  return batch_slot_bytes(m.data(), n.data(), r.data(), side.data(), count) * batch_lanes(count);
}

qg_status qg_step_batch(qg_layer* const* layers, const void* const* d_G, const int64_t* ldg, int32_t count,
                        void* d_ws, size_t ws_bytes, void* stream) {
  if (count < 0 || (count > 0 && (!layers || !d_G || !ldg || !d_ws))) return QG_EINVAL;
  if (count == 0) return QG_OK;
  if (!aligned(d_ws, 256)) return QG_EALIGN;
  std::vector<int32_t> m(count), n(count), r(count), side(count);
  for (int i = 0; i < count; ++i) {
    qg_status st = check_step_args(layers[i], d_G[i], ldg[i]);
    if (st != QG_OK) return st;
    for (int j = 0; j < i; ++j)
      if (layers[j] == layers[i]) return QG_EINVAL;
    m[i] = layers[i]->cfg.m, n[i] = layers[i]->cfg.n, r[i] = layers[i]->cfg.r, side[i] = layers[i]->cfg.proj_side;
  }
  const size_t slot = batch_slot_bytes(m.data(), n.data(), r.data(), side.data(), count);
  const int lanes = batch_lanes(count);
  if (ws_bytes < slot * lanes) return QG_ESTATE;
  std::vector<StepProblem> probs(count);
  for (int b = 0; b * kBatch < count; ++b) {
    uint8_t* ws = static_cast<uint8_t*>(d_ws) + (b % lanes) * slot;
    for (int i = b * kBatch; i < count && i < (b + 1) * kBatch; ++i) {
      fill_step_problem(layers[i], d_G[i], ldg[i], ws, layers[i]->sched.t + 1, &probs[i]);
      ws += qg::step_scratch_bytes(m[i], n[i], r[i], side[i]);
    }
  }
  const cudaStream_t user = static_cast<cudaStream_t>(stream);
  qg_status st = QG_OK;
  if (lanes == 1) {
    st = cuda_status(qg::launch_step(probs.data(), count, user));
  } else {
    std::lock_guard<std::mutex> lock(g_lane_mu);
    Lane* L = nullptr;
    st = extra_lanes(&L);
    if (st != QG_OK) return st;
    if (cudaEventRecord(L->fork, user) != cudaSuccess) return QG_ECUDA;
    for (int i = 0; i < lanes - 1; ++i)
      if (cudaStreamWaitEvent(L->s[i], L->fork, 0) != cudaSuccess) return QG_ECUDA;
    for (int b = 0; st == QG_OK && b * kBatch < count; ++b) {
      const int cnt = std::min(kBatch, count - b * kBatch);
      const int lane = b % lanes;
      st = cuda_status(qg::launch_step(probs.data() + b * kBatch, cnt, lane ? L->s[lane - 1] : user));
    }
    // join even after a failed launch, so later work on `stream` stays ordered
    // after whatever the extra lanes hold
    for (int i = 0; i < lanes - 1; ++i)
      if (cudaEventRecord(L->join[i], L->s[i]) != cudaSuccess || cudaStreamWaitEvent(user, L->join[i], 0) != cudaSuccess)
        st = QG_ECUDA;
  }
  if (st == QG_OK)
    for (int i = 0; i < count; ++i) layers[i]->sched.t += 1;
  return st;
}

qg_status qg_sched_after_refresh(int64_t t, int32_t delta, int32_t has_cossim, float cossim, float gamma,
                                 int32_t* delta_out, int64_t* t_next_out) {
  if (!delta_out || !t_next_out || delta < 1 || t < 0) return QG_EINVAL;
  int64_t d = delta;
  if (has_cossim && cossim > gamma) d *= 2;
  if (d > INT32_MAX) d = INT32_MAX;
  *delta_out = static_cast<int32_t>(d);
  *t_next_out = t + d;
  return QG_OK;
}

qg_status qg_refresh(qg_layer* L, const void* d_G, int64_t ldg, int32_t force, void* d_ws, size_t ws_bytes,
                     qg_refresh_info* info, void* stream) {
  if (!L || !d_G) return QG_EINVAL;
  if (info) memset(info, 0, sizeof(*info));
  const bool due = force || L->sched.t == L->sched.t_next;
  if (!due) {
    if (info) {
      info->delta = L->sched.delta;
      info->t_next = L->sched.t_next;
      info->n_refresh = L->sched.n_refresh;
    }
    return QG_OK;
  }
  const qg_config& c = L->cfg;
  if (ldg < c.n || ldg % 8 != 0 || !aligned(d_G, 16)) return QG_EALIGN;
  if (!d_ws) return QG_EINVAL;
  if (!aligned(d_ws, 256)) return QG_EALIGN;
  // the right-side projection refreshes on G^T: P has n rows
  const int32_t pm = c.proj_side ? c.n : c.m, pn = c.proj_side ? c.m : c.n;
  if (ws_bytes < qg::refresh_scratch_bytes(pm, pn, c.r, c.oversample)) return QG_ESTATE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool has_prev = L->sched.has_projection != 0;
  qg::RefreshArgs ra;
  memset(&ra, 0, sizeof(ra));
  ra.G = d_G;
  ra.ldg = ldg;
  ra.m = pm;
  ra.n = pn;
  ra.transpose_g = c.proj_side;
  ra.r = c.r;
  ra.oversample = c.oversample;
  ra.power_iters = c.power_iters;
  ra.seed = c.seed;
  ra.refresh_idx = static_cast<uint32_t>(L->sched.n_refresh);
  ra.layer_id = c.layer_id;
  ra.Pq = L->v.Pq;
  ra.sP = L->v.sP;
  ra.Pq_prev = L->v.Pq_prev;
  ra.sP_prev = L->v.sP_prev;
  ra.has_prev = has_prev ? 1 : 0;
  ra.status = L->v.status;
  ra.mom_refresh = c.mom_refresh;
  ra.Mq = L->v.Mq;
  ra.Vq = L->v.Vq;
  ra.sM = L->v.sM;
  ra.sV = L->v.sV;
  ra.ld_mom = L->v.ld_mom;
  ra.nblk = L->v.nblk;
  ra.mom_rows = L->v.mom_rows;
  ra.mom_cols = L->v.mom_cols;
  float cs = 0.f;
  qg_status st = qg::run_refresh(ra, static_cast<uint8_t*>(d_ws), ws_bytes, s, &cs);
  if (st != QG_OK) return st;
  int32_t nd;
  int64_t tn;
  qg_sched_after_refresh(L->sched.t, L->sched.delta, has_prev ? 1 : 0, cs, c.gamma, &nd, &tn);
  L->sched.delta = nd;
  L->sched.t_next = tn;
  L->sched.n_refresh += 1;
  L->sched.has_projection = 1;
  if (info) {
    info->refreshed = 1;
    info->has_cossim = has_prev ? 1 : 0;
    info->cossim = cs;
    info->delta = nd;
    info->t_next = tn;
    info->n_refresh = L->sched.n_refresh;
  }
  return QG_OK;
}

size_t qg_cossim_workspace_bytes(int32_t m, int32_t r) {
  if (m <= 0 || r <= 0) return 0;
  return qg::cossim_scratch_bytes(m, r);
}

qg_status qg_cossim(const float* d_Pa, const float* d_Pb, int32_t m, int32_t r, int64_t ld, float* d_out,
                    void* d_ws, size_t ws_bytes, void* stream) {
  if (!d_Pa || !d_Pb || !d_out || !d_ws) return QG_EINVAL;
  if (m <= 0 || r <= 0 || ld < r) return QG_ESHAPE;
  if (!aligned(d_ws, 256)) return QG_EALIGN;
  if (ws_bytes < qg::cossim_scratch_bytes(m, r)) return QG_ESTATE;
  return qg::run_cossim(d_Pa, d_Pb, m, r, ld, d_out, static_cast<uint8_t*>(d_ws), static_cast<cudaStream_t>(stream));
}

qg_status qg_layer_status(qg_layer* L, void* stream) {
  if (!L) return QG_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return QG_ECUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, L->v.status, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return QG_ECUDA;
  if (word && cudaMemset(L->v.status, 0, sizeof(word)) != cudaSuccess) return QG_ECUDA;
  if (word & qg::kStatusTimeout) return QG_ETIMEOUT;
  if (word & qg::kStatusNonFinite) return QG_ENONFINITE;
  return QG_OK;
}

qg_status qg_philox4x32_10(const uint32_t* c0, const uint32_t* c1, const uint32_t* c2, const uint32_t* c3,
                           int64_t count, uint32_t k0, uint32_t k1, uint32_t* out, void* stream) {
  if (count < 0) return QG_EINVAL;
  if (count > 0 && (!c0 || !c1 || !c2 || !c3 || !out)) return QG_EINVAL;
  if (!aligned(out, 16)) return QG_EALIGN;
  return cuda_status(qg::launch_philox(c0, c1, c2, c3, count, k0, k1, out, static_cast<cudaStream_t>(stream)));
}

qg_status qg_dequant_projection(const uint8_t* d_Pq, const float* d_sP, int32_t m, int32_t r, void* d_out,
                                void* stream) {
  if (!d_Pq || !d_sP || !d_out) return QG_EINVAL;
  if (m <= 0 || r <= 0 || r % 32 != 0) return QG_ESHAPE;
  if (!aligned(d_Pq, 4) || !aligned(d_out, 16)) return QG_EALIGN;
  return cuda_status(qg::launch_dequant_projection(d_Pq, d_sP, static_cast<int64_t>(m) * r,
                                                   static_cast<uint16_t*>(d_out), static_cast<cudaStream_t>(stream)));
}

qg_status qg_quantize_projection(const float* d_P, int64_t ld, int32_t m, int32_t r, uint8_t* d_Pq, float* d_sP,
                                 void* stream) {
  if (!d_P || !d_Pq || !d_sP) return QG_EINVAL;
  if (m <= 0 || r <= 0 || ld < r) return QG_ESHAPE;
  if (!aligned(d_P, 4) || !aligned(d_sP, 4)) return QG_EALIGN;
  return cuda_status(qg::launch_quantize_projection(d_P, ld, m, r, d_Pq, d_sP, static_cast<cudaStream_t>(stream)));
}

qg_status qg_gemm_bf16(const void* d_A, int64_t lda, int32_t a_trans, const void* d_B, int64_t ldb,
                       int32_t b_trans, float* d_D, int64_t ldd, int32_t M, int32_t N, int32_t K, void* stream) {
  if (!d_A || !d_B || !d_D) return QG_EINVAL;
  if (M <= 0 || N <= 0 || K <= 0) return QG_ESHAPE;
  if (!aligned(d_A, 16) || !aligned(d_B, 16) || !aligned(d_D, 16)) return QG_EALIGN;
  if (lda % 8 || ldb % 8 || ldd % 4) return QG_EALIGN;
  if (lda < (a_trans ? M : K) || ldb < (b_trans ? K : N) || ldd < N) return QG_EALIGN;
  return cuda_status(qg::launch_gemm_f32(d_A, lda, a_trans != 0, d_B, ldb, b_trans != 0, d_D, ldd, M, N, K,
                                         static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
