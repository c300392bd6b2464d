// Persistent, warp-specialised tcgen05 GEMM core for sm_100a with a pluggable
// epilogue.  D (M x N) = A (M x K) * B (K x N), bf16 operands fed by TMA into a
// 4-stage shared-memory ring, fp32 accumulators in TMEM (two 128 x 256 buffers,
// so the epilogue of one tile overlaps the MMAs of the next).
//
//   warp 0      : TMA producer (one elected lane)
//   warp 1      : TMEM allocator + MMA issuer (one elected lane)
//   warps 2..9  : two epilogue warpgroups; warpgroup g drains TMEM buffer g, i.e.
//                 every other tile of the CTA, so two tiles' epilogues overlap
//                 each other and the MMAs.  Within a warpgroup each warp owns one
//                 TMEM lane quarter (row = quarter*32 + lane).
//
// A grid of at most one CTA per SM walks a flat list of tiles that spans up to
// kMaxProblems independent problems (a batch of weight matrices).  Within a
// problem, tiles are ordered N-block-major so that the CTAs running at the same
// time share the same B column strip through L2.
//
// Every wait is bounded: a wait that runs out raises the CTA's abort flag and
// the timeout bit of the status word; all roles then leave their loops, the
// producer waits (bounded) for its copies in flight, the MMA issuer for its
// tensor-core work, and TMEM is freed before the kernel returns.
#pragma once

#include "qg_device.cuh"

namespace qg {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int kStages = 4;
constexpr int kAStageBytes = BM * BK * 2;  // 16 KiB
constexpr int kBStageBytes = BN * BK * 2;  // 32 KiB
constexpr int kGemmThreads = 320;
constexpr int kMaxProblems = 8;
constexpr int kTmemCols = 2 * BN;  // 512: the whole TMEM of the SM
constexpr size_t kGemmSmemBytes = size_t(kStages) * (kAStageBytes + kBStageBytes) + 1024;

template <class Epi>
struct GemmProblem {
  CUtensorMap tmA;  // K-major A: box {64 (K), 128 (M)}; MN-major A: box {64 (M), 64 (K)}
  CUtensorMap tmB;  // MN-major B: box {64 (N), 64 (K)}; K-major B: box {64 (K), 256 (N)}
  int32_t M, N, K;
  int32_t tiles_m, tiles_n, tile_begin;
  uint32_t* status;  // the matrix's device status word (may be null)
  typename Epi::Args epi;
};

template <class Epi>
struct GemmParams {
  GemmProblem<Epi> prob[kMaxProblems];
  int32_t nprob;
  int32_t total_tiles;
};

struct TileRef {
  int prob, mb, nb;
};

template <class Epi>
QG_DEV TileRef locate_tile(const GemmParams<Epi>& p, int tile) {
  int pi = 0;
  while (pi + 1 < p.nprob && tile >= p.prob[pi + 1].tile_begin) ++pi;
  const int local = tile - p.prob[pi].tile_begin;
  const int tm = p.prob[pi].tiles_m;
  return TileRef{pi, local % tm, local / tm};
}

template <class Epi, bool kAMN, bool kBMN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ GemmParams<Epi> p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kAStageBytes;

  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full[2];
  __shared__ __align__(8) uint64_t acc_empty[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint32_t* const status = nullptr;  // timeouts are reported per matrix at exit

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < p.nprob; ++i) {
      tma_prefetch_map(&p.prob[i].tmA);
      tma_prefetch_map(&p.prob[i].tmB);
    }
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // per-stage bit masks
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x) {
        const TileRef tr = locate_tile(p, tile);
        const GemmProblem<Epi>& pr = p.prob[tr.prob];
        const int nkb = (pr.K + BK - 1) / BK;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_bar[stage], kAStageBytes + kBStageBytes);
          uint8_t* a_dst = sA + stage * kAStageBytes;
          uint8_t* b_dst = sB + stage * kBStageBytes;
          if (kAMN) {
            tma_load_2d(a_dst, &pr.tmA, &full_bar[stage], tr.mb * BM, kb * BK);
            tma_load_2d(a_dst + 8192, &pr.tmA, &full_bar[stage], tr.mb * BM + 64, kb * BK);
          } else {
            tma_load_2d(a_dst, &pr.tmA, &full_bar[stage], kb * BK, tr.mb * BM);
          }
          if (kBMN) {
#pragma unroll
            for (int h = 0; h < 4; ++h)
              tma_load_2d(b_dst + h * 8192, &pr.tmB, &full_bar[stage], tr.nb * BN + 64 * h, kb * BK);
          } else {
            tma_load_2d(b_dst, &pr.tmB, &full_bar[stage], kb * BK, tr.nb * BN);
          }
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (abort_flag) {
        for (int s = 0; s < kStages; ++s)
          if (armed & (1u << s)) mbar_wait_drain(&full_bar[s], (armed_parity >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, kAMN, kBMN);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x) {
        const TileRef tr = locate_tile(p, tile);
        const GemmProblem<Epi>& pr = p.prob[tr.prob];
        const int nkb = (pr.K + BK - 1) / BK;
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, &abort_flag, status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * kAStageBytes);
          const uint32_t b_base = smem_u32(sB + stage * kBStageBytes);
          const int kleft = pr.K - kb * BK;
          const int ksteps = kleft >= BK ? BK / 16 : (kleft + 15) / 16;
          for (int kk = 0; kk < ksteps; ++kk) {
            const uint64_t ad = kAMN ? sdesc_sw128(a_base + kk * 2048, 8192, 1024)
                                     : sdesc_sw128(a_base + kk * 32, 16, 1024);
            const uint64_t bd = kBMN ? sdesc_sw128(b_base + kk * 2048, 8192, 1024)
                                     : sdesc_sw128(b_base + kk * 32, 16, 1024);
            umma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (abort_flag) {
        umma_commit(&drain_bar);
        mbar_wait_drain(&drain_bar, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t eg = static_cast<uint32_t>(warp - 2) >> 2;  // warpgroup = TMEM buffer
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    uint32_t acc_phase = 0, it = 0;
    for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++it) {
      if ((it & 1u) != eg) continue;
      const TileRef tr = locate_tile(p, tile);
      const GemmProblem<Epi>& pr = p.prob[tr.prob];
      if (!mbar_wait(&acc_full[eg], acc_phase, &abort_flag, status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + eg * BN;
      Epi::apply(pr.epi, pr.M, pr.N, tr.mb, tr.nb, row, taddr, pr.status);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[eg]);
      acc_phase ^= 1u;
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && abort_flag) {
    for (int i = 0; i < p.nprob; ++i)
      if (p.prob[i].status) atomicOr(p.prob[i].status, kErrTimeout);
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace qg
