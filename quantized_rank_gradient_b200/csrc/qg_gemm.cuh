// Persistent, warp-specialised tcgen05 GEMM core for sm_100a with a pluggable
// epilogue.  D (M x N) = A (M x K) * B (K x N), bf16 operands fed by TMA into a
// 4-stage shared-memory ring, fp32 accumulators in TMEM (two 128 x 256 buffers,
// so the epilogue of one tile overlaps the MMAs of the next).
//
//   warp 0      : TMA producer (one elected lane)
//   warp 1      : TMEM allocator + MMA issuer (one elected lane)
//   warps 2..9  : two epilogue warpgroups that share every tile, each taking
//                 128 of its 256 columns; while they drain one TMEM buffer the
//                 MMAs fill the other.  Within a warpgroup each warp owns one TMEM
//                 lane quarter (row = quarter*32 + lane).
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
  CUtensorMap tmS[2];  // side operands of the epilogue (int8 tiles staged in shared memory)
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

// Every epilogue warpgroup works on every tile: of `groups` warpgroups, group g
// takes the tile's columns [g BN / groups, (g + 1) BN / groups).  Row-wise
// reductions over the whole tile width (the Adam block absmax) combine the
// groups' partial values through `xchg` ([group][BM] slots, one per row), guarded
// by a per-lane-quarter mbarrier that completes once per tile.
struct EpiPair {
  int group;
  int groups;
  float2* xchg;         // slot of group 0 for this warp's 32 rows; group g's is xchg + g * BM
  uint64_t* xbar;       // count `groups`: one arrival per warp holding these rows
  uint32_t xphase;
  volatile int* abort;
  uint32_t* status;
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
  static_assert(Epi::kSideBytes == 0, "the one-CTA kernel stages no side operands");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kAStageBytes;

  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full[2];
  __shared__ __align__(8) uint64_t acc_empty[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ __align__(8) uint64_t xbar[4];
  __shared__ float2 xchg[2][2][BM];  // [tile parity][half][row]
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
      mbar_init(&acc_empty[a], 8);  // all 8 epilogue warps
    }
    for (int q = 0; q < 4; ++q) mbar_init(&xbar[q], 2);
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
    const int half = (warp - 2) >> 2;  // warpgroup: which 128 columns of every tile
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++it) {
      const uint32_t buf = it & 1u, ph = (it >> 1) & 1u;
      const TileRef tr = locate_tile(p, tile);
      const GemmProblem<Epi>& pr = p.prob[tr.prob];
      if (!mbar_wait(&acc_full[buf], ph, &abort_flag, status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + buf * BN;
      EpiPair ep{half, 2, &xchg[it & 1u][0][quarter * 32], &xbar[quarter], it & 1u, &abort_flag, pr.status};
      Epi::apply(pr.epi, pr.M, pr.N, tr.mb, tr.nb, row, taddr, ep, nullptr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
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

// ---------------------------------------------------------------------------
// The same GEMM on CTA pairs (clusters of 2, tcgen05 cta_group::2): a 256 x 256
// tile per pair, each CTA loading its 128 rows of A and 128 columns of B (half
// the B traffic per SM of the one-CTA kernel), a ring of 32 KiB stages per
// CTA, one MMA issuer in the even CTA (M = 256, N = 256, K = 16), and each
// CTA's TMEM holding its 128 rows of the accumulator, drained by its own
// Epi::kPairGroups epilogue warpgroups (warps 2 .. 4 kPairGroups + 1; warp 0
// loads, warp 1 issues the MMAs).  Four warpgroups give each SM sub-partition
// four epilogue warps to hide the epilogue's latencies behind one another.  Loads of both CTAs complete on the even CTA's
// full-barrier; the issuer's commits arrive on both CTAs' barriers; epilogues
// of both CTAs release an accumulator buffer on the even CTA's barrier.
// B is MN-major (two 64-column boxes per CTA) or K-major (one box of 64 K x 128 N).
//
// Side operands.  An epilogue may declare Epi::kSideBytes > 0: int8 tiles that
// belong to the output tile (the weight codes, the moment codes) are then
// staged in shared memory by TMA, Epi::kSideBufs buffers deep, so that the
// epilogue reads them at shared-memory latency.  One epilogue thread issues the
// loads of tile j + kSideBufs - 1 when the epilogue starts tile j, after every
// epilogue warp has released that buffer (side_empty, one arrival per warp);
// the loads complete on side_full.
// ---------------------------------------------------------------------------

// Epilogues of the pair kernel declare kPairBKMN, the K depth of a ring stage
// when both operands are MN-major (K is then the outer dimension of every TMA
// box, so any multiple of 16 works; a K-major operand's 128-byte swizzled rows
// hold exactly 64 bf16 of K, so with one the depth is 64), and kPairMaxStages,
// a cap on the ring's depth.  Smaller stages let more of them, and more bytes,
// stay in flight beside the side buffers.
template <class Epi, int kBK>
struct PairLayout {
  static constexpr int kGroups = Epi::kPairGroups;  // epilogue warpgroups per CTA
  static constexpr int kThreads = 64 + 128 * kGroups;
  static_assert(kGroups >= 2 && kGroups <= 4, "two to four epilogue warpgroups");
  static_assert(kBK % 16 == 0 && kBK >= 16 && kBK <= 64, "K depth of a stage");
  static constexpr int kHalfStageBytes = 128 * kBK * 2;  // 128 rows of A or 128 columns of B
  static constexpr int kChunkBytes = 64 * kBK * 2;       // one 64-wide M/N chunk of an MN-major stage
  static constexpr int kSideBytes = Epi::kSideBytes;
  static constexpr int kSideBufs = Epi::kSideBufs;
  static constexpr int kSideTotal = kSideBytes * kSideBufs;
  // shared memory a CTA may hold (227 KiB) less the static part: barriers and
  // flags, plus the row-maxima exchange when the epilogue uses it
  static constexpr int kBudget = 232448 - 512 - (Epi::kExchange ? int(sizeof(float2)) * 2 * kGroups * BM : 0) - 1024;
  // as many ring stages as fit beside the side buffers, at most kPairMaxStages
  static constexpr int kFit = (kBudget - kSideTotal) / (2 * kHalfStageBytes);
  static constexpr int kStages = kFit > Epi::kPairMaxStages ? Epi::kPairMaxStages : kFit;
  static constexpr size_t kSmemBytes = size_t(kStages) * 2 * kHalfStageBytes + kSideTotal + 1024;
  static_assert(kStages >= 3, "side buffers leave too few ring stages");
  static_assert(kStages <= 32, "stage bit masks are 32 bits wide");
  static_assert(kSideBytes % 1024 == 0, "side buffers keep 1024-byte alignment");
};

// The layout a pair-kernel instantiation uses.
template <class Epi, bool kAMN, bool kBMN>
struct PairCfg {
  static constexpr int kBK = (kAMN && kBMN) ? Epi::kPairBKMN : 64;
  using L = PairLayout<Epi, kBK>;
};

template <class Epi, bool kAMN, bool kBMN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<Epi, kAMN, kBMN>::L::kThreads, 1)
    gemm_tc_pair_kernel(const __grid_constant__ GemmParams<Epi> p) {
  using L = typename PairCfg<Epi, kAMN, kBMN>::L;
  constexpr int kBKp = PairCfg<Epi, kAMN, kBMN>::kBK;
  constexpr int kHalfStageBytes = L::kHalfStageBytes;
  constexpr int kChunk = L::kChunkBytes;
  constexpr int kGroups = L::kGroups;
  constexpr int kEpiWarps = 4 * kGroups;
  constexpr int kStagesP = L::kStages;
  constexpr int kSide = L::kSideBytes;
  constexpr int kSB = L::kSideBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStagesP * kHalfStageBytes;
  uint8_t* sSide = smem + 2 * kStagesP * kHalfStageBytes;

  __shared__ __align__(8) uint64_t full_bar[kStagesP];
  __shared__ __align__(8) uint64_t empty_bar[kStagesP];
  __shared__ __align__(8) uint64_t acc_full[2];
  __shared__ __align__(8) uint64_t acc_empty[2];
  __shared__ __align__(8) uint64_t side_full[2];
  __shared__ __align__(8) uint64_t side_empty[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ __align__(8) uint64_t xbar[4];
  __shared__ float2 xchg[Epi::kExchange ? 2 : 1][Epi::kExchange ? kGroups : 1][Epi::kExchange ? BM : 32];  // [tile parity][group][row]
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  uint32_t* const status = nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesP; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * kEpiWarps);  // every epilogue warp of both CTAs (used in the even CTA)
      mbar_init(&side_full[a], 1);
      mbar_init(&side_empty[a], kEpiWarps);  // this CTA's epilogue warps
    }
    for (int q = 0; q < 4; ++q) mbar_init(&xbar[q], kGroups);
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < p.nprob; ++i) {
      tma_prefetch_map(&p.prob[i].tmA);
      tma_prefetch_map(&p.prob[i].tmB);
      if (kSide > 0) {
        tma_prefetch_map(&p.prob[i].tmS[0]);
        tma_prefetch_map(&p.prob[i].tmS[1]);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(&tmem_base_sh, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;

  // tiles are 256 x 256 here: 128-row block index of this CTA = 2 * pair block + rank
  auto pair_tiles = [&](const GemmProblem<Epi>& pr) { return ((pr.M + 255) / 256) * pr.tiles_n; };
  auto locate = [&](int tile, int& pi, int& mb2, int& nb) {
    pi = 0;
    int begin = 0;
    while (pi + 1 < p.nprob && tile >= begin + pair_tiles(p.prob[pi])) {
      begin += pair_tiles(p.prob[pi]);
      ++pi;
    }
    const int local = tile - begin;
    const int tm = (p.prob[pi].M + 255) / 256;
    mb2 = local % tm;
    nb = local / tm;
  };
  int total = 0;
  for (int i = 0; i < p.nprob; ++i) total += pair_tiles(p.prob[i]);

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, armed = 0, armed_parity = 0;
      const uint32_t fb0 = mapa_shared(&full_bar[0], 0);  // the even CTA's full barriers, 8 bytes apart
      bool ok = true;
      for (int tile = cluster; ok && tile < total; tile += nclusters) {
        int pi, mb2, nb;
        locate(tile, pi, mb2, nb);
        const GemmProblem<Epi>& pr = p.prob[pi];
        const int nkb = (pr.K + kBKp - 1) / kBKp;
        const int row0 = mb2 * 256 + static_cast<int>(rank) * 128;
        const int col0 = nb * BN + static_cast<int>(rank) * 128;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag, status)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 4 * kHalfStageBytes);
          const uint32_t fb = fb0 + stage * 8u;
          uint8_t* a_dst = sA + stage * kHalfStageBytes;
          uint8_t* b_dst = sB + stage * kHalfStageBytes;
          if (kAMN) {
            tma_load_2d_pair(a_dst, &pr.tmA, fb, row0, kb * kBKp);
            tma_load_2d_pair(a_dst + kChunk, &pr.tmA, fb, row0 + 64, kb * kBKp);
          } else {
            tma_load_2d_pair(a_dst, &pr.tmA, fb, kb * kBKp, row0);
          }
          if (kBMN) {
            tma_load_2d_pair(b_dst, &pr.tmB, fb, col0, kb * kBKp);
            tma_load_2d_pair(b_dst + kChunk, &pr.tmB, fb, col0 + 64, kb * kBKp);
          } else {
            tma_load_2d_pair(b_dst, &pr.tmB, fb, kb * kBKp, col0);
          }
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStagesP) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (abort_flag && rank == 0) {
        for (int s = 0; s < kStagesP; ++s)
          if (armed & (1u << s)) mbar_wait_drain(&full_bar[s], (armed_parity >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, 256, kAMN, kBMN);
      // Descriptors of stage 0; a stage or a K step moves only the 14-bit start
      // address field (16-byte units, shared addresses < 256 KiB), so the
      // descriptors of any stage and step are one 64-bit add away.  This keeps
      // the issuing thread's instruction stream short while the epilogue warps
      // share its scheduler.
      const uint64_t a_desc0 = kAMN ? sdesc_sw128(smem_u32(sA), kChunk, 1024) : sdesc_sw128(smem_u32(sA), 16, 1024);
      const uint64_t b_desc0 = kBMN ? sdesc_sw128(smem_u32(sB), kChunk, 1024) : sdesc_sw128(smem_u32(sB), 16, 1024);
      constexpr uint64_t kStageStep = kHalfStageBytes >> 4;
      constexpr uint64_t kAStep = kAMN ? (2048 >> 4) : (32 >> 4);  // one K step of 16
      constexpr uint64_t kBStep = kBMN ? (2048 >> 4) : (32 >> 4);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < total; tile += nclusters) {
        int pi, mb2, nb;
        locate(tile, pi, mb2, nb);
        const int K = p.prob[pi].K;
        const int nkb = (K + kBKp - 1) / kBKp;
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, &abort_flag, status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = a_desc0 + stage * kStageStep;
          const uint64_t bd = b_desc0 + stage * kStageStep;
          const int kleft = K - kb * kBKp;
          if (kleft >= kBKp) {
            umma_bf16_pair(d_tmem, ad, bd, idesc, kb != 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 1; kk < kBKp / 16; ++kk) umma_bf16_pair(d_tmem, ad + kk * kAStep, bd + kk * kBStep, idesc, 1u);
          } else {
            const int ksteps = (kleft + 15) / 16;
            for (int kk = 0; kk < ksteps; ++kk)
              umma_bf16_pair(d_tmem, ad + kk * kAStep, bd + kk * kBStep, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair_mc(&empty_bar[stage], 0x3);
          if (++stage == kStagesP) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_mc(&acc_full[acc], 0x3);
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (abort_flag) {
        umma_commit_pair(&drain_bar);
        mbar_wait_drain(&drain_bar, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int group = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const bool side_issuer = kSide > 0 && warp == 2 && lane == 0;
    uint32_t side_armed = 0, side_parity = 0;  // per-buffer bit masks (issuer only)
    bool ok = true;
    // side loads of local tile j (the CTA's j-th tile) into buffer j % kSB;
    // returns false when the wait for the buffer's release ran out
    auto issue_side = [&](int j) -> bool {
      const int tile = cluster + j * nclusters;
      if (tile >= total) return true;
      const int b = j % kSB;
      if (j >= kSB && !mbar_wait(&side_empty[b], static_cast<uint32_t>(j / kSB - 1) & 1u, &abort_flag, status))
        return false;
      int pi, mb2, nb;
      locate(tile, pi, mb2, nb);
      fence_proxy_async_shared();
      mbar_arrive_expect_tx(&side_full[b], kSide);
      Epi::issue_side(p.prob[pi].tmS, mb2 * 2 + static_cast<int>(rank), nb, sSide + b * kSide, &side_full[b]);
      side_armed |= 1u << b;
      side_parity = (side_parity & ~(1u << b)) | ((static_cast<uint32_t>(j / kSB) & 1u) << b);
      return true;
    };
    if (side_issuer)
      for (int j = 0; j + 1 < kSB; ++j) ok = ok && issue_side(j);
    uint32_t it = 0;
    for (int tile = cluster; ok && tile < total; tile += nclusters, ++it) {
      if (side_issuer && !issue_side(static_cast<int>(it) + kSB - 1)) break;
      const uint32_t buf = it & 1u, ph = (it >> 1) & 1u;
      int pi, mb2, nb;
      locate(tile, pi, mb2, nb);
      const GemmProblem<Epi>& pr = p.prob[pi];
      if (!mbar_wait(&acc_full[buf], ph, &abort_flag, status)) break;
      const uint8_t* side = nullptr;
      if (kSide > 0) {
        const uint32_t sb = it % kSB;
        if (!mbar_wait(&side_full[sb], (it / kSB) & 1u, &abort_flag, status)) break;
        side = sSide + sb * kSide;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + buf * BN;
      float2* xs = Epi::kExchange ? &xchg[it & 1u][0][quarter * 32] : nullptr;
      EpiPair ep{group, kGroups, xs, &xbar[quarter], it & 1u, &abort_flag, pr.status};
      Epi::apply(pr.epi, pr.M, pr.N, mb2 * 2 + static_cast<int>(rank), nb, row, taddr, ep, side);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (kSide > 0) mbar_arrive(&side_empty[it % kSB]);
        mbar_arrive_cluster(mapa_shared(&acc_empty[buf], 0));
      }
    }
    if (side_issuer && abort_flag) {
      for (int b = 0; b < kSB; ++b)
        if (side_armed & (1u << b)) mbar_wait_drain(&side_full[b], (side_parity >> b) & 1u);
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && abort_flag) {
    for (int i = 0; i < p.nprob; ++i)
      if (p.prob[i].status) atomicOr(p.prob[i].status, kErrTimeout);
  }
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace qg
