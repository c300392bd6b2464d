/*
 * qgalore.h - C ABI of the B200 (sm_100a) Q-GaLore optimizer-step library.
 *
 * The method (sources: the paper-index record "Q-GaLore: Quantized GaLore with
 * INT4 Projection and Layer-Adaptive Low-Rank Gradients", abstract; the AIMech
 * curated page on Q-GaLore, mechanisms "layer-adaptive subspace cosine
 * schedule" (paper section 3.1, Eq. (5)) and "INT4 projection and INT8
 * stochastic rounding" (paper section 3.2)):
 *
 *   per weight matrix W (m x n, INT8 codes with float32 group scales, fixed
 *   unless w_rescale lets a group grow)
 *     a1  P~ = bf16(dequant(P^Q))             P^Q: m x r INT4, one scale / 64
 *     a2  R  = P~^T G                          G: m x n bf16 gradient
 *     a3  Adam on (M^Q, V^Q), r x n INT8 with per-row-block scales -> N (bf16)
 *     a4  U  = P~ N
 *     a5  W^Q <- W^Q + xi(alpha U / s_W)       xi: unbiased stochastic rounding
 *   beside it, when due: top-r randomized SVD of G -> new P^Q; CosSim against
 *   the previous P^Q; the refresh interval doubles when CosSim > gamma.
 *
 * Conventions for every entry point:
 *   - Arrays are row-major.  Pointers named d_* are DEVICE pointers; they are
 *     owned by the caller, who allocates and frees them (e.g. with PyTorch).
 *     The library owns only the opaque host handle qg_layer.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously on it; only qg_refresh (when a
 *     refresh runs) and qg_layer_status wait for the device.
 *   - A handle must not be used from two streams at once.
 *   - Argument errors are reported before anything is enqueued: nothing is
 *     launched and the state is unchanged.  Launch failures return QG_ECUDA.
 *     Errors found by kernels (a device wait that ran out, a non-finite
 *     gradient projection) set bits of the layer's device status word, read
 *     and cleared by qg_layer_status.
 *   - bf16 arrays are passed as void* (16-bit patterns).
 *   - Nothing here allocates device memory.
 */
#ifndef QGALORE_H
#define QGALORE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QG_OK = 0,
  QG_EINVAL = 1,      /* null pointer or hyper-parameter out of range */
  QG_ESHAPE = 2,      /* unsupported sizes */
  QG_EALIGN = 3,      /* pointer or leading dimension not aligned as required */
  QG_ESTATE = 4,      /* buffer too small, or the layer has no projection yet */
  QG_ECUDA = 5,       /* CUDA runtime or driver error */
  QG_ETIMEOUT = 6,    /* a bounded device wait gave up (kernel returned early) */
  QG_ENONFINITE = 7   /* a non-finite value was met on the device */
} qg_status;

/* Hyper-parameters of one weight matrix.  qg_config_default fills the values
 * used by the paper's setting where the pages give one (gamma = 0.4) and the
 * plain readings elsewhere. */
typedef struct {
  int32_t m, n, r;          /* W is m x n, P is m x r; 32 <= r <= min(m, n), r % 32 == 0;
                               m, n < 2^30, m n < 2^40, max(m, n) r < 2^34 */
  int32_t w_group;          /* weight-scale group (consecutive elements), must be 256 */
  int32_t p_group;          /* INT4 projection group, must be 64 */
  int32_t mom_block;        /* moment block along a row, must be 256 */
  float beta1, beta2, eps;  /* Adam: 0.9, 0.999, 1e-8 */
  float lr;                 /* learning rate, 1e-3 */
  float alpha;              /* scale of the low-rank update, 0.25 */
  float gamma;              /* CosSim threshold, 0.4 */
  int32_t delta0;           /* initial refresh interval (steps), 200 */
  int32_t oversample;       /* randomized SVD oversampling p, 16 */
  int32_t power_iters;      /* randomized SVD power iterations q, 2 */
  uint64_t seed;            /* Philox key of the stochastic rounding and of Omega */
  uint32_t layer_id;        /* Philox counter word: distinguishes matrices */
  int32_t mom_refresh;      /* the low-rank moments at a refresh that replaces P: 0 keep them (default),
                               1 reset them to zero, 2 rotate them into the new basis with
                               C = P_new^T P_prev: m' = C m, v' = (C o C) v (element-wise square),
                               re-quantized on the step's grids */
  int32_t proj_side;        /* which side is projected: 0 (default) P is m x r and R = P^T G (r x n);
                               1 P is n x r, R = G P (m x r) and U = N P^T, the projection taken
                               from the top-r right singular vectors of G */
  int32_t w_rescale;        /* a weight group whose updated values would leave the INT8 grid: 0 (default)
                               the codes saturate at +-127; 1 the group's scale grows to
                               s' = s / rho, rho = (127 * 2^16) / max|T| with T = q * 2^16 + ceil(X)
                               the values in units of 2^-16 code (X = U * alpha / s * 2^16), and the
                               group is rounded stochastically again on the new grid
                               (code = floor((ceil(fl(T) rho) + draw) / 2^16)) with the same draws;
                               needs n % 256 == 0 (QG_ESHAPE otherwise) */
} qg_config;

typedef struct qg_layer qg_layer;

/* Device pointers into a layer's state (for inspection, checkpointing). */
typedef struct {
  uint32_t* status;         /* device status word (bits: 1 timeout, 2 non-finite) */
  uint8_t* Pq;              /* ceil(m*r/2) bytes: INT4 P, two nibbles per byte, even index low */
  float* sP;                /* ceil(m*r/64) float32 scales */
  uint8_t* Pq_prev;         /* previous projection (for CosSim) */
  float* sP_prev;
  int8_t* Mq;               /* r x ld_mom INT8 first moment (columns >= n unused) */
  int8_t* Vq;               /* r x ld_mom INT8 codes 0..127 of sqrt(v), v the second moment */
  float* sM;                /* r x nblk float32 */
  float* sV;                /* r x nblk float32 */
  int64_t ld_mom;           /* row stride of Mq, Vq in bytes: mom_cols rounded up to 32 */
  int32_t nblk;             /* ceil(mom_cols / 256) */
  int32_t p_rows;           /* rows of P: m (left projection) or n (right) */
  int32_t mom_rows, mom_cols; /* shape of the moments (that of R): r x n (left) or m x r (right) */
} qg_layer_views;

/* Schedule state of the layer-adaptive refresh (host side). */
typedef struct {
  int64_t t;                /* steps taken (the next step is t + 1) */
  int32_t delta;            /* current refresh interval */
  int64_t t_next;           /* a refresh is due when t == t_next */
  int32_t n_refresh;        /* refreshes done so far */
  int32_t has_projection;   /* a projection has been installed or computed */
} qg_sched;

typedef struct {
  int32_t refreshed;        /* 1 if a refresh ran in this call */
  int32_t has_cossim;       /* 1 if a previous projection existed */
  float cossim;             /* CosSim(P_new, P_prev), Eq. (5) of the paper */
  int32_t delta;            /* interval after the call */
  int64_t t_next;           /* next due step after the call */
  int32_t n_refresh;
} qg_refresh_info;

const char* qg_status_str(qg_status s);
void qg_config_default(qg_config* cfg, int32_t m, int32_t n, int32_t r);

/* Sizes of the caller-provided buffers (bytes).  The state holds what a layer
 * carries between steps; the workspace is scratch for one call and may be
 * shared by layers that run one after another on the same stream. */
size_t qg_state_bytes(const qg_config* cfg);
size_t qg_step_workspace_bytes(const qg_config* cfg);
size_t qg_refresh_workspace_bytes(const qg_config* cfg);

/* Create a layer handle over caller-owned device memory: the per-matrix state
 * of the AIMech Q-GaLore page, mechanism "INT4 projection and INT8 stochastic
 * rounding" (paper section 3.2) -- INT8 master weights with their scales, the
 * INT4 projection P_t and the previous one, and the INT8 low-rank moments
 * (M_t^Q, V_t^Q) -- plus the layer's refresh schedule of the mechanism
 * "layer-adaptive subspace cosine schedule" (paper section 3.1, Eq. (5)):
 * t = 0, interval delta0, first refresh due at t = 0.
 *   d_state : >= qg_state_bytes(cfg) bytes, 256-byte aligned; zero-initialised
 *             here (moments and scales start at zero) on `stream`.
 *   d_W     : m x ldw INT8 weight codes, 16-byte aligned, ldw >= n, ldw % 16 == 0;
 *             updated in place by qg_step.
 *   d_Wscale: ceil(m*n/256) float32 scales, group g covering logical elements
 *             [256 g, 256 g + 256) of the row-major m x n array; read only,
 *             except with cfg->w_rescale = 1, where qg_step enlarges in place
 *             the scale of a group that the update would carry off the grid.
 * Returns QG_EINVAL / QG_ESHAPE / QG_EALIGN / QG_ESTATE on bad arguments. */
qg_status qg_layer_init(qg_layer** out, const qg_config* cfg, void* d_state, size_t state_bytes,
                        int8_t* d_W, int64_t ldw, float* d_Wscale, void* stream);
qg_status qg_layer_destroy(qg_layer* layer);
qg_status qg_layer_views_get(const qg_layer* layer, qg_layer_views* views);
qg_status qg_layer_sched_get(const qg_layer* layer, qg_sched* sched);
qg_status qg_layer_sched_set(qg_layer* layer, const qg_sched* sched);

/* Install an INT4 projection (e.g. from a checkpoint): copies ceil(p*r/2)
 * packed bytes and ceil(p*r/64) scales device-to-device into the state, p the
 * rows of P (m, or n for the right-side projection).  The previous projection
 * is kept for CosSim only when keep_prev != 0. */
qg_status qg_layer_set_projection(qg_layer* layer, const uint8_t* d_Pq, const float* d_sP,
                                  int32_t keep_prev, void* stream);

/* One optimizer step a1..a5 (AIMech Q-GaLore page, mechanism "INT4 projection
 * and INT8 stochastic rounding", paper section 3.2) on one matrix.
 *   d_G : m x ldg bf16 gradient, 16-byte aligned, ldg >= n, ldg % 8 == 0.
 *   d_ws: >= qg_step_workspace_bytes(cfg) bytes, 256-byte aligned.
 * Never refreshes; QG_ESTATE if no projection is installed. */
qg_status qg_step(qg_layer* layer, const void* d_G, int64_t ldg, void* d_ws, size_t ws_bytes,
                  void* stream);

/* The step of the AIMech Q-GaLore page, mechanism "INT4 projection and INT8
 * stochastic rounding" (paper section 3.2), applied to `count` independent
 * matrices (every layer of a model carries its own W, P and moments and steps
 * on its own gradient): the same arithmetic as qg_step for each, in few
 * launches: batches of up to 8
 * matrices, three launches per batch (dequantize the batch's projections, then
 * one persistent tcgen05 grid per GEMM stage).  With more than one batch, the
 * batches take turns among three lanes: `stream` and two streams that the
 * library creates on the current device at its first such call and keeps until
 * the process exits; they fork from `stream` and join back to it through
 * events, so the call is ordered on `stream` (and may be captured into a CUDA
 * graph once those streams exist) and the lanes' kernels overlap.  Calls from
 * several host threads are serialised while they enqueue.
 * d_ws (256-byte aligned) must hold qg_step_batch_workspace_bytes of the same
 * configurations in the same order: one slot per lane in use (as many as there
 * are batches, at most three), each the largest batch's sum of
 * qg_step_workspace_bytes, reused by the lane's batches.  A smaller d_ws gives
 * QG_ESTATE before anything is launched. */
qg_status qg_step_batch(qg_layer* const* layers, const void* const* d_G, const int64_t* ldg,
                        int32_t count, void* d_ws, size_t ws_bytes, void* stream);
size_t qg_step_batch_workspace_bytes(const qg_config* const* cfgs, int32_t count);

/* qg_step without a workspace argument, for callers that cannot allocate
 * device memory (for instance a host program whose device memory belongs to
 * another allocator with a fixed budget, or a thread that must not take the
 * implicit synchronisation of cudaMalloc / cudaFree).  The paper has no
 * counterpart: this is a property of the library only.
 *   The scratch (P~ and N) lives in a static device array of
 *   QG_NOALLOC_SCRATCH_BYTES (32 MiB), held by every GPU that loads the library
 *   until the process exits; every LLaMA-7B-shaped matrix at r = 1024 fits.
 *   Larger matrices are refused with QG_ESHAPE before anything is launched.
 *   The first call in each CUDA context looks up the array's device address
 *   (cudaGetSymbolAddress) with the device current; make that first call
 *   before any stream capture.  The address is cached with the context, so a
 *   device reset (which builds a new context and loads the array anew) makes
 *   the next call look it up again.  All calls share the array and it keeps the
 *   previous call's contents (the step overwrites everything it reads), so
 *   calls whose GPU work overlaps, from other streams or threads, race.
 * Arguments, state handling and errors are otherwise those of qg_step. */
#define QG_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
qg_status qg_step_noalloc(qg_layer* layer, const void* d_G, int64_t ldg, void* stream);

/* Layer-adaptive subspace refresh (AIMech Q-GaLore page, mechanism
 * "layer-adaptive subspace cosine schedule", paper section 3.1, Eq. (5); the
 * SVD that finds the subspace: the paper-index record's abstract).  Runs when
 * force != 0 or the layer is due (t == t_next); otherwise returns QG_OK with
 * info->refreshed = 0 and touches nothing.  When it runs: randomized top-r SVD
 * of G -> new INT4 P; if a projection existed, CosSim(P_new, P_prev) on the
 * device; the interval doubles iff CosSim > gamma; t_next = t + delta.  This
 * call synchronises `stream` to read CosSim.  `info` may be NULL.
 *   d_ws: >= qg_refresh_workspace_bytes(cfg) bytes, 256-byte aligned.  After a
 *   refresh its first m*r*4 bytes hold the float32 projection (row-major m x r,
 *   orthonormal columns sorted by descending singular value, each column's
 *   largest-magnitude entry positive) from which the INT4 one was quantized.
 * Randomized SVD: k = min(r + oversample, m, n) columns, Rademacher test
 * matrix from Philox keyed by the seed and counted by (refresh index, layer_id),
 * power_iters power iterations, Rayleigh-Ritz on the k-dimensional range. */
qg_status qg_refresh(qg_layer* layer, const void* d_G, int64_t ldg, int32_t force, void* d_ws,
                     size_t ws_bytes, qg_refresh_info* info, void* stream);

/* CosSim(Pa, Pb) = (1/r) sum_i sigma_i(Pa^T Pb), the subspace similarity of the
 * AIMech Q-GaLore page, mechanism "layer-adaptive subspace cosine schedule"
 * (paper section 3.1, Eq. (5)), for float32 m x r matrices with row stride ld
 * (elements), result written to d_out[0] on the device.  The sum of the
 * singular values is taken as the nuclear norm of Pa^T Pb through its polar
 * factor (Newton-Schulz iteration), not by an SVD.
 * d_ws >= qg_cossim_workspace_bytes(m, r). */
size_t qg_cossim_workspace_bytes(int32_t m, int32_t r);
qg_status qg_cossim(const float* d_Pa, const float* d_Pb, int32_t m, int32_t r, int64_t ld,
                    float* d_out, void* d_ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, reads and clears the layer's device status word:
 * QG_OK, QG_ETIMEOUT or QG_ENONFINITE.  The pages define no error reporting;
 * the word records the two device-side failures of the step of the AIMech
 * Q-GaLore page, mechanism "INT4 projection and INT8 stochastic rounding"
 * (paper section 3.2): a bounded wait that ran out, and a non-finite projected
 * gradient R = P^T G (whose Adam update, and so the step's outputs, are then
 * unspecified). */
qg_status qg_layer_status(qg_layer* layer, void* stream);

/* Host-only rule of the paper's layer-adaptive schedule: after a refresh at
 * step t, delta doubles iff has_cossim and cossim > gamma; t_next = t + delta. */
qg_status qg_sched_after_refresh(int64_t t, int32_t delta, int32_t has_cossim, float cossim,
                                 float gamma, int32_t* delta_out, int64_t* t_next_out);

/* INT4 quantization of a float32 projection (refresh stage): m x r matrix with
 * row stride ld (elements) -> ceil(m*r/2) packed bytes (two's-complement
 * nibbles, even index in the low nibble) and ceil(m*r/64) scales; groups of 64
 * consecutive elements of the row-major m x r array, scale = absmax / 7,
 * code = clamp(rint(x * (7 / absmax)), -7, 7); a group whose absmax is below
 * 2^-120 gets scale 0 and codes 0. */
qg_status qg_quantize_projection(const float* d_P, int64_t ld, int32_t m, int32_t r, uint8_t* d_Pq,
                                 float* d_sP, void* stream);

/* ---- Device-time accounting of this library's own launches ----
 * While enabled, every kernel the library launches is bracketed by CUDA events
 * recorded on the launch stream.  qg_profile_collect synchronises those events
 * and returns, per kernel kind, the launch count, the summed device time, and
 * the algorithmic FLOPs and bytes of those launches. */
typedef enum {
  QG_KERNEL_DEQUANT = 0,      /* a1: INT4 P -> bf16 */
  QG_KERNEL_PROJECT_ADAM = 1, /* a2 + a3: tcgen05 P^T G with the moment epilogue */
  QG_KERNEL_BACKPROJECT_SR = 2, /* a4 + a5: tcgen05 P N with stochastic rounding */
  QG_KERNEL_OTHER = 3,        /* refresh and single-stage kernels */
  QG_KERNEL_LINEAR_DEQUANT = 4, /* INT8 W -> bf16 W~ for the linear-layer products */
  QG_KERNEL_LINEAR_GEMM = 5,  /* tcgen05 forward / backward products of a linear layer */
  QG_KERNEL_LINEAR_FUSED = 6, /* forward product for a few tokens, INT8 W read once */
  QG_KERNEL_KINDS = 7
} qg_kernel_kind;

typedef struct {
  int64_t launches;
  double device_ms;   /* sum over launches */
  double flops;       /* algorithmic: 2*m*n*r per GEMM problem */
  double bytes;       /* algorithmic HBM bytes (see the design notes) */
} qg_kernel_times;

qg_status qg_profile_enable(int32_t on);  /* on != 0 starts a new window */
qg_status qg_profile_collect(qg_kernel_times* out, int32_t kinds);

/* ---- Single-stage entry points (used by the tests to check each stage) ---- */

/* Philox-4x32-10 words for `count` counters given as four device arrays of
 * uint32 (c0[i], c1[i], c2[i], c3[i]); writes out[4*i + w]. */
qg_status qg_philox4x32_10(const uint32_t* d_c0, const uint32_t* d_c1, const uint32_t* d_c2,
                           const uint32_t* d_c3, int64_t count, uint32_t k0, uint32_t k1,
                           uint32_t* d_out, void* stream);

/* Stage a1: P~ (m x r bf16, row stride r) from packed INT4 codes and scales. */
qg_status qg_dequant_projection(const uint8_t* d_Pq, const float* d_sP, int32_t m, int32_t r,
                                void* d_out_bf16, void* stream);

/* D (M x N float32, row stride ldd) = A B on the tcgen05 tensor cores, bf16
 * operands, float32 accumulation.  A is M x K given as row-major M x K
 * (a_trans = 0, stride lda) or as row-major K x M (a_trans = 1); B is K x N
 * given as row-major K x N (b_trans = 0) or as row-major N x K (b_trans = 1).
 * Strides in elements, multiples of 8; pointers 16-byte aligned. */
qg_status qg_gemm_bf16(const void* d_A, int64_t lda, int32_t a_trans, const void* d_B, int64_t ldb,
                       int32_t b_trans, float* d_D, int64_t ldd, int32_t M, int32_t N, int32_t K,
                       void* stream);

/* Self-check of the branch-free correctly rounded float32 reciprocal, square
 * root and division that the Adam epilogue uses in place of the IEEE
 * intrinsics (the update of the AIMech Q-GaLore page, "INT8 optimizer states":
 * one square root and one division per element).
 *   op 0: reciprocal, every float in [2^-100, 2^100];
 *   op 1: square root, every float in [2^-100, 2^100] and +-0;
 *   op 2: division, n Philox-drawn pairs (seeded by `seed`) with b > 0 in
 *         [2^-100, 2^100], |a| in [2^-90, 2^90] or +-0, quotient in range.
 * d_out: 3 device uint64; [0] mismatches against __frcp_rn / __fsqrt_rn /
 * __fdiv_rn, [1] operands tested, [2] smallest failing (a bits << 32 | b bits)
 * (all ones if none).  Asynchronous on `stream`; QG_EINVAL for a bad op or a
 * null d_out. */
qg_status qg_selfcheck_exact_math(int32_t op, uint64_t n, uint64_t seed, unsigned long long* d_out,
                                  void* stream);

/* Self-check of the bounded device waits that every kernel of this library
 * uses (the failure-detection path; the pages have no counterpart): one
 * thread waits on an mbarrier that nothing arrives at, with a limit of
 * limit_ns (1 ns .. 10 s).  The wait must give up after the limit, set the
 * timeout bit (1, as in a layer's status word) in *d_status (device uint32,
 * OR-ed) and let the kernel return, leaving the context usable.
 * d_out: 2 device uint64, [0] = 1 when
 * the wait reported failure, [1] = nanoseconds spent.  Asynchronous on
 * `stream`; QG_EINVAL for null pointers or a limit out of range. */
qg_status qg_selfcheck_wait_timeout(uint64_t limit_ns, uint32_t* d_status, unsigned long long* d_out, void* stream);

/* ---- Linear layers with INT8 weights (simulated weight-only quantization) ----
 * The matrix products around the optimizer step (AIMech Q-GaLore page,
 * limitation "simulated weight-quantization throughput", paper section 3.2 and
 * section 4.4, Fig. 4: activations stay in 16-bit floating point and the INT8
 * weights are dequantized for the forward and backward products; Theorem 3.1,
 * paper section 3.1: the weight gradient of y = W x is G = (1/B) D_y X^T, the
 * 1/B folded into D_y here).  For a layer whose INT8 weight W is m x n (the
 * optimizer's W^Q with its flattened groups of 256 scales), a training step
 * dequantizes W once and runs the three products on the tcgen05 core (bf16
 * operands, float32 accumulation, bf16 results rounded to nearest even):
 *   qg_linear_dequant_weight   W~ = bf16(fp32(q_ij) * s_W[(i n + j) / 256])  (m x n)
 *   qg_linear_forward          Y  = X W~^T    X: T x n   ->  Y: T x m
 *   qg_linear_backward_data    dX = D_y W~    D_y: T x m ->  dX: T x n
 *   qg_linear_backward_weight  G  = D_y^T X   ->  G: m x n, the bf16 gradient
 *                              qg_step / qg_step_batch take
 * Every matrix is row-major and device-resident, owned by the caller; the
 * functions allocate nothing and are asynchronous on `stream`.  bf16 strides
 * (ld*) are in elements, at least the column count and a multiple of 8, and
 * bf16 bases are 16-byte aligned (tensor-memory-access tiles); the INT8 W has
 * ldw >= n, ldw % 16 == 0, a 16-byte aligned base (as qg_layer_init requires).
 * Errors launch nothing: QG_EINVAL for a null pointer where data is needed,
 * QG_ESHAPE for negative sizes or a bad stride, QG_EALIGN for a misaligned
 * base, QG_ECUDA when a launch fails.  T = 0 is a no-op, except that G = 0.
 * No output may overlap an input. */
qg_status qg_linear_dequant_weight(const int8_t* d_W, int64_t ldw, const float* d_sW, int32_t m, int32_t n,
                                   void* d_Wt, int64_t ldwt, void* stream);
qg_status qg_linear_forward(const void* d_X, int64_t ldx, const void* d_Wt, int64_t ldwt, int32_t T, int32_t m,
                            int32_t n, void* d_Y, int64_t ldy, void* stream);
/* The forward product for a few tokens straight from the INT8 weight:
 * Y = X W~^T with W~ = bf16(fp32(q_ij) * s_W[(i n + j) / 256]) formed in
 * registers, never stored (the same limitation passage of the AIMech Q-GaLore
 * page: the dequantization fused into the product).  For 1 <= T <= 64 tokens
 * the product is bound by reading the weight: this reads its INT8 codes once,
 * where qg_linear_dequant_weight and qg_linear_forward move five bytes per
 * weight.  X: T x n bf16 (ldx, 16-byte aligned); W: m x ldw INT8 and its group
 * scales as qg_layer_init takes them; Y: T x m bf16 (ldy).  float32
 * accumulation in another order than qg_linear_forward's, each output rounded
 * once to bf16; two calls give the same bits.  The kernel is launched with
 * programmatic stream serialization: its set-up may overlap the end of the
 * preceding kernel in the stream, and every read of X, W and the scales comes
 * after that kernel has finished.  T > 64 gives QG_ESHAPE (use the
 * dequantization and the tcgen05 product there); T = 0 is a no-op.  Other
 * errors as above. */
qg_status qg_linear_forward_int8(const void* d_X, int64_t ldx, const int8_t* d_W, int64_t ldw, const float* d_sW,
                                 int32_t T, int32_t m, int32_t n, void* d_Y, int64_t ldy, void* stream);
qg_status qg_linear_backward_data(const void* d_dY, int64_t lddy, const void* d_Wt, int64_t ldwt, int32_t T,
                                  int32_t m, int32_t n, void* d_dX, int64_t lddx, void* stream);
qg_status qg_linear_backward_weight(const void* d_dY, int64_t lddy, const void* d_X, int64_t ldx, int32_t T,
                                    int32_t m, int32_t n, void* d_G, int64_t ldg, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* QGALORE_H */
