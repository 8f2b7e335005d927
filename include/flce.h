/*
 * flce.h - C ABI of the B200 (sm_100a) fused linear cross-entropy library.
 *
 * The operation. "Liger Kernel: Efficient Triton Kernels for LLM Training"
 * (paper review, 提案手法; Figure 1 "Fused Linear Cross Entropy") describes a
 * chunked fusion of the lm_head projection with cross-entropy that never keeps
 * the logits over the whole vocabulary. "Liger-Kernel 項目詳細介紹"
 * (使用方法 > 3. 低級 API 方式) gives its call, loss_fn(weight, input, target),
 * with weight [V,H], input [BT,H] and an integer target [BT], and says under
 * 核心特性 > 技術實現 that nothing is approximated. So, exactly:
 *
 *     z = X W^T;  l_i = logsumexp(z_i) - z_{i,t_i} for rows with t_i != ignore_index;
 *     loss = sum_i l_i / N (FLCE_MEAN, N = non-ignored rows) or sum_i l_i (FLCE_SUM);
 *     dz_i = (softmax(z_i) - onehot(t_i)) * (1/N or 1), 0 for ignored rows;
 *     grad_X = dz W;  grad_W = dz^T X.
 *
 * The gradients are those of the loss for an upstream gradient of 1. N = 0
 * (every row ignored) gives loss 0 and zero gradients.
 *
 * Conventions shared by every entry point:
 *  - Pointers in flce_tensor are DEVICE pointers on the current CUDA device.
 *    The caller owns every tensor; the library never keeps a pointer after a
 *    call returns (work it enqueued still reads them until it completes).
 *  - Matrices are row-major: stride[1] == 1, stride[0] >= shape[1] (elements).
 *  - Work is enqueued on `stream` (a cudaStream_t / CUstream; NULL = legacy
 *    default stream). Nothing synchronises unless FLCE_FLAG_SYNC_CHECK is set.
 *  - A call returns FLCE_OK once its work is enqueued. Argument errors are
 *    found on the host before anything is enqueued and leave outputs untouched.
 *    Data errors found on the device (a target outside [0,V) that is not
 *    ignore_index) set a bit of the device error word, read with
 *    flce_get_device_error(); such rows are treated as ignored. Nothing traps.
 *  - No C++ exception crosses this interface.
 *  - Calls may come from several host threads at once: the library's own
 *    state (the per-device context and the phase-timing record) is guarded by
 *    a mutex, and each call takes its own workspace. A caller-provided
 *    workspace (flce_options.workspace) must not be shared by calls that may
 *    run on the GPU at the same time.
 */
#ifndef FLCE_H
#define FLCE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FLCE_VERSION 120 /* 1.2.0: flce_options.grad_w_ready_event; 1.1.0: flce_scale_grad,
                             flce_gemm_bf16_wait_test, FLCE_FLAG_RECOMPUTE, FLCE_FLAG_ROUTE_EVERY_CHUNK */

#if defined(__GNUC__)
#define FLCE_API __attribute__((visibility("default")))
#else
#define FLCE_API
#endif

struct CUstream_st;
typedef struct CUstream_st* flce_stream_t; /* the same handle as cudaStream_t */

typedef enum {
  FLCE_OK = 0,
  FLCE_ERR_INVALID_ARG = 1,        /* null pointer, bad shape, stride or alignment */
  FLCE_ERR_UNSUPPORTED_DTYPE = 2,  /* dtype combination not provided */
  FLCE_ERR_UNSUPPORTED_DEVICE = 3, /* current device is not sm_100 (B200); caller may fall back */
  FLCE_ERR_ALLOC = 4,              /* workspace allocation from the library's pool failed */
  FLCE_ERR_CUDA = 5,               /* a CUDA runtime call failed */
  FLCE_ERR_WORKSPACE_TOO_SMALL = 6 /* caller-provided workspace smaller than the plan needs */
} flce_status;

typedef enum { FLCE_F32 = 0, FLCE_BF16 = 1, FLCE_I64 = 2 } flce_dtype;
/* FLCE_NONE: `loss` is fp32 [BT] and receives the per-row losses (0 for ignored rows). */
typedef enum { FLCE_MEAN = 0, FLCE_SUM = 1, FLCE_NONE = 2 } flce_reduction;

/* Bits of the device error word. */
#define FLCE_DEVERR_TARGET_RANGE 0x1u /* a target outside [0,V) that is not ignore_index */
#define FLCE_DEVERR_TIMEOUT 0x2u      /* a bounded wait inside a kernel ran out; results invalid */

/* A dense tensor of rank 0, 1 or 2. */
typedef struct {
  void* data;        /* device pointer */
  int32_t dtype;     /* flce_dtype */
  int32_t ndim;      /* 0, 1 or 2 */
  int64_t shape[2];  /* shape[0..ndim-1] */
  int64_t stride[2]; /* in elements; the last stride must be 1 */
} flce_tensor;

/* How grad_W is accumulated across row chunks. */
typedef enum {
  FLCE_GRADW_ACCUM_OUTPUT = 0, /* fp32 sum per chunk, added into grad_W in its own dtype */
  FLCE_GRADW_ACCUM_FP32 = 1    /* fp32 V x H accumulator in the workspace, cast once */
} flce_gradw_accum;

#define FLCE_FLAG_SYNC_CHECK 0x1  /* synchronise and check for CUDA errors after each launch */
#define FLCE_FLAG_TIME_PHASES 0x2 /* record CUDA events around each phase (flce_phase_times) */
/* Two-phase use, for losses whose per-row upstream gradient is known only
 * after the forward pass (preference losses, reduction 'none' under autograd):
 *   KEEP_LOGITS: forward only. The whole batch is one chunk (BT <= 32768);
 *     its store of exp(z - m_tile), the per-tile maxima and the row lse stay in
 *     the caller's workspace (opt->workspace, sized by flce_plan with the same
 *     options). loss (and row_loss / lse) are written; grad_X and grad_W must
 *     be NULL.
 *   FROM_KEPT: gradients only, from what a KEEP_LOGITS call with the same X, W,
 *     target, ignore_index and workspace left there, with opt->row_grad and the
 *     reduction's scale applied now; the logits GEMM is not run again. loss is
 *     not written. Nothing may touch the workspace between the two calls.
 * Together they do 6*BT*H*V tensor FLOPs where a forward call followed by a
 * full call with row_grad does 8. The paper has no counterpart: its chunked
 * preference losses take each chunk's gradient in one pass over complete
 * pairs; keeping the batch's store is the general form of that on one chunk. */
#define FLCE_FLAG_KEEP_LOGITS 0x4
#define FLCE_FLAG_FROM_KEPT 0x8
/* grad_W shards (below): route every chunk's grad_W boxes to their owners
 * instead of only the last chunk's. No local [V, H] partial sum is kept, at the
 * price of n_chunks times the exchanged bytes. */
#define FLCE_FLAG_ROUTE_EVERY_CHUNK 0x10
/* The recompute schedule (bf16 only; not with the two-phase flags or grad_W
 * shards). The pages' chunked method (技術原理 > 分塊計算 of "Liger-Kernel
 * 項目詳細介紹") bounds memory by computing the logits a piece at a time; this
 * schedule takes the pieces over the vocabulary instead of the rows. A first
 * pass computes every row's logsumexp with nothing stored; a second pass, per
 * chunk of Vc vocabulary columns, rebuilds the logits of all rows over the
 * chunk by GEMM, writes dz into a [BT, Vc] bf16 store, adds dz W_c into grad_X
 * (in bf16, one rounding per chunk after the first) and writes the chunk's rows
 * of grad_W = dz^T X complete. 8 * BT * H * V tensor FLOPs instead of 6; in
 * exchange the store can be as small as BT * 256 * 2 bytes. With this flag,
 * chunk_rows (if > 0) is the vocabulary columns per chunk (rounded up to 256),
 * else Vc comes from workspace_limit_bytes (default 512 MiB) over BT rows; the
 * stats' chunk_rows / n_chunks then describe vocabulary chunks. grad_w_accum
 * has no effect: every grad_W row is produced once. */
#define FLCE_FLAG_RECOMPUTE 0x20

typedef struct {
  int64_t chunk_rows;            /* rows per chunk; 0 = the environment variable
                                    FLCE_CHUNK_ROWS if it holds a positive integer, else
                                    chosen from workspace_limit_bytes.
                                    Rounded up to a multiple of 128. */
  int64_t workspace_limit_bytes; /* chunk store budget; 0 = at most 512 MiB but at least 2048
                                    rows, and at most half the rows, so two or more chunks
                                    whenever BT > 128 */
  void* workspace;               /* optional caller-owned device workspace (256-byte aligned) */
  int64_t workspace_bytes;       /* its size in bytes */
  int32_t grad_w_accum;          /* flce_gradw_accum */
  int32_t flags;                 /* FLCE_FLAG_* */
  const int64_t* n_valid;        /* optional DEVICE pointer: the mean denominator N to use
                                    (e.g. the count over all data-parallel ranks, from
                                    flce_count_valid + an all-reduce). NULL = count locally. */
  float* row_loss;               /* optional DEVICE [BT] fp32: per-row losses l_i (0 if ignored) */
  float* lse;                    /* optional DEVICE [BT] fp32: per-row logsumexp of z_i */
  const float* row_grad;         /* optional DEVICE [BT] fp32: upstream gradient per row; the
                                    gradients are those of sum_i row_grad_i * l_i * (1/N or 1).
                                    NULL = all ones. */
  /* grad_W scattered to shards (data parallelism): shard k (< n_shards <= 8) owns grad_W rows
     [k * shard_rows, (k+1) * shard_rows), stored bf16 [rows, H] with row pitch grad_w_shard_ld
     at grad_w_shards[k] (a HOST array of device pointers; a shard may live on a peer GPU, mapped
     into this one). The chunks before the last accumulate grad_W locally, in a bf16 [V, H]
     region of the workspace (flce_plan counts it); the last chunk's grad_W GEMM adds each of its
     output boxes, plus the same box of that local sum, into the owner's shard as it is produced
     (a TMA reduce-add, done in the owner's L2, over NVLink for a peer). So each rank sends
     V * H * 2 bytes whatever the chunk count, (P - 1) / P of them to peers.
     FLCE_FLAG_ROUTE_EVERY_CHUNK routes every chunk's boxes instead (no local sum).
     The caller zeroes each shard and orders that before any rank's call, and orders every rank's
     call before reading a shard. Requires the bf16 path, grad_W == NULL, shard_rows % 32 == 0 and
     n_shards * shard_rows >= V. Additions from several callers land in unspecified order. */
  void* const* grad_w_shards;
  int32_t n_shards;
  int64_t shard_rows;
  int64_t grad_w_shard_ld;
  /* Optional cudaEvent_t (passed as void*), owned and created by the caller: recorded once on
     `stream`, right after the last launch that writes grad_W (or the shards). In the stored-chunk
     schedule the last chunk then launches its grad_W GEMM before its grad_X GEMM, so that work a
     caller queues on another stream behind this event (a data-parallel reduction of grad_W, as
     the pages' FSDP benchmark runs after the backward) overlaps the last grad_X GEMM, whose
     256 x 512 tiles leave SMs free. Elsewhere it is recorded at the end of the call. Library
     infrastructure for overlapping the data-parallel exchange; the pages define no such hook.
     NULL = none. Added in 1.2.0. */
  void* grad_w_ready_event;
} flce_options;

typedef struct {
  int64_t chunk_rows;                /* rows per chunk actually used */
  int64_t n_chunks;                  /* number of chunks */
  int64_t workspace_bytes;           /* peak extra device memory this call uses */
  int64_t materialized_logits_bytes; /* BT * V * 2: the logits a non-fused loss would hold */
  int32_t kernel_launches;           /* kernels this call enqueued */
  int32_t path;                      /* 0 = SIMT fp32 path, 1 = tcgen05 bf16 path */
} flce_stats;

/* Fill *opt with the defaults (all zero / NULL). Library infrastructure: no passage of the pages
 * defines it. */
FLCE_API void flce_options_init(flce_options* opt);

/*
 * Fused linear cross-entropy, forward and backward, in one call: the chunked fused
 * Linear + CrossEntropy of "Liger Kernel: Efficient Triton Kernels for LLM Training"
 * (paper review, 提案手法; Figure 1), with the call shape of the low-level API of
 * "Liger-Kernel 項目詳細介紹" (使用方法 > 3. 低級 API 方式): loss_fn(weight, input, target),
 * then loss.backward(). The operation is the one this header's preamble writes out.
 *   X       [BT,H]  bf16 or f32 (row-major)
 *   W       [V,H]   same dtype as X
 *   target  [BT]    int64; rows equal to ignore_index are ignored
 *   reduction       FLCE_MEAN, FLCE_SUM or FLCE_NONE
 *   loss    scalar  f32 (ndim 0, or ndim 1 with one element): written;
 *                   for FLCE_NONE, f32 [BT]: the per-row losses
 *   grad_X  [BT,H]  same dtype as X, or NULL to skip: fully overwritten
 *   grad_W  [V,H]   same dtype as W, or NULL to skip: fully overwritten
 * bf16 runs the tcgen05 tensor-core path (fp32 accumulation, bf16 results,
 * H % 8 == 0, 16-byte aligned rows); f32 runs an exact-fp32 SIMT path.
 * Unless opt->workspace is given, workspace is taken stream-ordered from a
 * library-owned memory pool (cudaMallocFromPoolAsync) and released to it at
 * the end; the pool keeps the memory mapped for the next call.
 */
FLCE_API flce_status flce_fwd_bwd(const flce_tensor* X, const flce_tensor* W, const flce_tensor* target,
                         int64_t ignore_index, int32_t reduction, flce_tensor* loss,
                         flce_tensor* grad_X, flce_tensor* grad_W, flce_stream_t stream);

/* As flce_fwd_bwd, with options (opt may be NULL) and statistics (stats may be NULL). */
FLCE_API flce_status flce_fwd_bwd_ex(const flce_tensor* X, const flce_tensor* W,
                            const flce_tensor* target, int64_t ignore_index, int32_t reduction,
                            flce_tensor* loss, flce_tensor* grad_X, flce_tensor* grad_W,
                            flce_stream_t stream, const flce_options* opt, flce_stats* stats);

/*
 * Host-only planning (the chunking of "Liger-Kernel 項目詳細介紹", 技術原理 > 分塊計算,
 * sized for a workspace budget): fills *out with the chunk rows, chunk count and
 * workspace bytes flce_fwd_bwd_ex would use for this shape. Touches no GPU.
 * dtype is FLCE_BF16 or FLCE_F32. want_grad_W selects whether a grad_W
 * accumulator (FLCE_GRADW_ACCUM_FP32) is counted.
 */
FLCE_API flce_status flce_plan(int64_t BT, int64_t H, int64_t V, int32_t dtype, int32_t want_grad_W,
                      const flce_options* opt, flce_stats* out);

/*
 * Library infrastructure (no passage defines it; it sizes the chunking's memory).
 * Host-only: the workspace bytes flce_fwd_bwd_ex would use for this shape and
 * options with grad_W requested (flce_plan's workspace_bytes), i.e. the size a
 * caller-provided opt->workspace needs. 0 for an empty batch; (size_t)-1 if
 * the arguments are invalid. Touches no GPU.
 */
FLCE_API size_t flce_workspace_bytes(int64_t BT, int64_t H, int64_t V, int32_t dtype, const flce_options* opt);

/*
 * The mean's denominator: N, the count of rows whose target is not ignore_index (the
 * ignore_index of the low-level API, "Liger-Kernel 項目詳細介紹", 使用方法 > 3), written as int64
 * to the DEVICE pointer n_valid_out on `stream`. Targets outside [0,V) that
 * are not ignore_index set FLCE_DEVERR_TARGET_RANGE and are not counted.
 * Used by data-parallel callers to all-reduce N before flce_fwd_bwd_ex.
 */
FLCE_API flce_status flce_count_valid(const flce_tensor* target, int64_t V, int64_t ignore_index,
                             int64_t* n_valid_out, flce_stream_t stream);

/*
 * Cross-entropy of given logits (the logits-given CrossEntropy of the paper
 * review's 主な発見: online softmax with in-place gradient replacement).
 *   logits [BT,V] bf16 or f32; target [BT] int64; loss scalar f32.
 *   grad_logits: same shape/dtype as logits, or NULL to skip. It may be the
 *   logits tensor itself (in-place gradient replacement).
 * opt may be NULL; only opt->n_valid, opt->row_loss, opt->lse and opt->row_grad are read.
 * FLCE_NONE as for flce_fwd_bwd (loss is f32 [BT]).
 * bf16 logits with V up to 16 * 32768 (8 * 32768 on a device that cannot hold
 * a 16-CTA cluster) take one pass: a thread-block cluster per row reads the
 * logits once and writes the gradient once, with a workspace of N and the
 * per-row losses only. Each CTA of the cluster stages its slice of the row in
 * shared memory: ceil(V / 25600) CTAs while that fits the device's largest
 * cluster, else slices of up to 32768 columns (FLCE_CE_SLICE=<columns> sets
 * the slice). f32 logits and longer rows take three passes (per-tile
 * partials, row combine, gradient) with a per-(row, 1024-column tile) partials
 * workspace. The workspace comes from the library's memory pool.
 */
FLCE_API flce_status flce_cross_entropy(const flce_tensor* logits, const flce_tensor* target,
                               int64_t ignore_index, int32_t reduction, flce_tensor* loss,
                               flce_tensor* grad_logits, flce_stream_t stream,
                               const flce_options* opt);

/*
 * flce_cross_entropy without any device allocation. The paper has no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory where they compute the loss (while a CUDA graph is being
 * captured around them, inside a host that owns all device memory through its
 * own allocator, or in a loop where an allocation and the synchronisation it
 * may bring are not allowed).
 *   Arguments and results are those of flce_cross_entropy, with two
 *   differences: opt is not taken (the mean uses this call's own count of
 *   non-ignored rows), and reduction must be FLCE_MEAN or FLCE_SUM (FLCE_NONE
 *   returns FLCE_ERR_INVALID_ARG: per-row losses come from flce_cross_entropy).
 *   The caller still provides logits, target, loss and grad_logits (which may
 *   be the logits).
 *   Scratch comes from one fixed array of 8 MiB in device memory that every
 *   GPU loading the library holds until the process exits. It needs about
 *   8 * ceil(V / 1024) + 12 bytes per row (round BT up to a multiple of 32
 *   for the first term), e.g. up to ~8200 rows at V = 128256; larger problems
 *   return FLCE_ERR_WORKSPACE_TOO_SMALL before any GPU work.
 *   The first call on a device looks up the array's device address and loads
 *   every kernel the entry point launches (CUDA runtime queries, no allocation);
 *   make that first call before any stream capture. All calls share the array and it keeps the last call's contents;
 *   every value a call reads from it is written earlier in the same call.
 *   Calls that overlap on the GPU (on different streams, or from different
 *   threads without ordering) race on the array: order them.
 * Never calls cudaMalloc, cudaFree or any allocating routine.
 */
FLCE_API flce_status flce_cross_entropy_noalloc(const flce_tensor* logits, const flce_tensor* target,
                                                int64_t ignore_index, int32_t reduction, flce_tensor* loss,
                                                flce_tensor* grad_logits, flce_stream_t stream);

/*
 * Test hook; no passage defines it (the pages' method runs its contractions inside the
 * fused call). Plain bf16 GEMM on the library's tcgen05 engine, for testing that engine
 * on its own: C[M,N] (f32, row-major, ldc) = sum_k A(m,k) * B(n,k).
 * A is [M,K] row-major (a_mn_major = 0, lda >= K) or [K,M] row-major
 * (a_mn_major = 1, lda >= M); B likewise with N. Leading dimensions are in
 * elements and must be multiples of 8; pointers 16-byte aligned.
 */
FLCE_API flce_status flce_gemm_bf16(const void* A, const void* B, float* C, int64_t M, int64_t N,
                           int64_t K, int64_t lda, int64_t ldb, int64_t ldc, int32_t a_mn_major,
                           int32_t b_mn_major, flce_stream_t stream);

/*
 * Test of the engine's failure path; the paper has no counterpart. The plain
 * GEMM of flce_gemm_bf16 (both operands K-major) on the CTA-pair engine, with
 * one change: every pair's MMA issuer, before its output tile number
 * stall_tile (0 = its first), waits on a barrier that nothing arrives on. That
 * wait is bounded like every wait in the library, so it runs out after the
 * library's wait limit (about 2 s): the kernel sets FLCE_DEVERR_TIMEOUT in the
 * device error word, abandons its remaining tiles, waits for the loads and
 * tensor-core work it has in flight, frees its tensor memory and returns. The
 * caller reads the status with flce_get_device_error; C is left partly written.
 * The context stays usable: later calls run normally. Returns FLCE_ERR_INVALID_ARG
 * for the arguments flce_gemm_bf16 refuses, a negative stall_tile, or when the
 * single-CTA engine is selected (FLCE_ENGINE=1sm).
 */
FLCE_API flce_status flce_gemm_bf16_wait_test(const void* A, const void* B, float* C, int64_t M, int64_t N,
                                              int64_t K, int64_t lda, int64_t ldb, int64_t ldc, int32_t stall_tile,
                                              flce_stream_t stream);

/*
 * Upstream gradient: t *= *scale in place, on `stream`. The loss module of
 * "Liger-Kernel 項目詳細介紹" (使用方法 > 3. 低級 API 方式) is used as
 * loss = loss_fn(weight, input, target); loss.backward(). The fused call has
 * already produced the gradients for an upstream gradient of 1 during the
 * forward pass; backward multiplies them by the upstream gradient, which lives
 * in device memory. So the comparison with 1 is made on the device: the host
 * never waits for the value, and when it is exactly 1 no element of t is read
 * or written.
 *   t      bf16 or f32, ndim 0, 1 or 2 (unit inner stride; row pitch stride[0]);
 *          DEVICE memory owned by the caller, modified in place
 *   scale  DEVICE pointer to one f32
 * Returns FLCE_ERR_INVALID_ARG for null pointers or a bad layout (nothing is
 * enqueued then) and FLCE_ERR_UNSUPPORTED_DTYPE for other dtypes.
 */
FLCE_API flce_status flce_scale_grad(flce_tensor* t, const float* scale, flce_stream_t stream);

/*
 * Library infrastructure (no passage defines it): device-side data errors and
 * wait timeouts are reported here instead of trapping.
 * Waits for `stream`, then returns the device error word of the current
 * device in *err (FLCE_DEVERR_* bits) and clears it. The word is shared by
 * every stream on the device.
 */
FLCE_API flce_status flce_get_device_error(flce_stream_t stream, uint32_t* err);

/*
 * Library infrastructure (no passage defines it).
 * Phase timing (calls made with FLCE_FLAG_TIME_PHASES): waits for the
 * recorded events and writes, for each phase p < n_phases, the summed
 * milliseconds to ms[p] and the number of timed launches to count[p] (either
 * may be NULL). reset != 0 clears the record afterwards. Phases:
 *   0 count valid rows, 1 logits GEMM + online-softmax epilogue (for
 *   flce_cross_entropy: the per-tile partials, or the one-pass row kernel),
 *   2 row combine + loss (or the factors of a FLCE_FLAG_FROM_KEPT call),
 *   3 in-place dlogits (flce_cross_entropy: the gradient pass),
 *   4 grad_X / grad_W GEMMs, 5 final loss reduction.
 */
#define FLCE_NUM_PHASES 6
FLCE_API flce_status flce_phase_times(double* ms, int32_t* count, int32_t n_phases, int32_t reset);

/* Static string for a status code. Library infrastructure: no passage defines it. */
FLCE_API const char* flce_status_string(int32_t status);

/* FLCE_VERSION of the built library. Library infrastructure: no passage defines it. */
FLCE_API int32_t flce_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FLCE_H */
