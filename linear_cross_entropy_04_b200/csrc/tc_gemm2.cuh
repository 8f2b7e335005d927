// Persistent tcgen05 GEMM engine over CTA pairs (cta_group::2), sm_100a.
//
// A cluster of two CTAs on the two SMs of a TPC computes one 256 x 256 output
// tile per step: each CTA stages its own 128 rows of A and its own 128 rows of
// B (N-half) per K-block, and the even CTA (the pair leader) issues
// tcgen05.mma.cta_group::2, M = 256, N = 256, K = 16, which reads A and B from
// both CTAs' shared memory and leaves rows 0-127 of the tile in the leader's
// tensor memory and rows 128-255 in the peer's. Compared with the one-CTA
// 128 x 256 tile, every SM loads and the tensor core reads half as much B per
// multiply, which lifts the shared-memory and L2 bandwidth ceilings.
//
// Roles per CTA (192 threads): warp 0 TMA producer, warp 1 MMA issuer (leader
// only; in both CTAs it owns the tensor-memory allocation), warps 2-5 epilogue
// on this CTA's accumulator rows.
//
// Barriers: the leader's full[s] expects the bytes of both CTAs (each CTA's
// loads complete on it); the leader's MMA commit releases empty[s] in both
// CTAs and signals tfull[a] in both CTAs; the leader's tempty[a] counts one
// arrival per epilogue warp of both CTAs. All waits are bounded (ptx.cuh).
// No load uses cluster multicast: each CTA fetches its own operand halves.
#pragma once

#include "tc_gemm.cuh"

namespace flce {

constexpr int T2_BM = 256;  // tile rows over the pair
constexpr int T2_BN = 256;
constexpr int T2_HALF = 128;  // rows of A, and of B, staged per CTA
constexpr int T2_BK = 64;
#ifndef FLCE_PAIR_STAGES
#define FLCE_PAIR_STAGES 6
#endif
#ifndef FLCE_PAIR_PREFETCH
#define FLCE_PAIR_PREFETCH 0
#endif
#ifndef FLCE_PAIR_KFENCE
#define FLCE_PAIR_KFENCE 1  // tcgen05 fence after each operand-stage wait
#endif
#ifndef FLCE_EPI_BACKOFF_NS
#define FLCE_EPI_BACKOFF_NS 0  // sleep between the epilogue's accumulator polls
#endif
// 256 x 256 tiles stage two consecutive 64-wide K-blocks together (T2_STAGES / 2
// stages of 64 KB): one operand wait, one commit and eight MMAs per stage. Against
// one K-block per 32 KB stage (same shared memory) the short-K launches (logits,
// grad_W) kept the tensor pipe busier per clock: the step ran 2.5% faster.
constexpr int T2_STAGES = FLCE_PAIR_STAGES;
static_assert(T2_STAGES % 2 == 0, "narrow stages hold two K-blocks");
// K-blocks between an L2 prefetch and the load of the same box (0: no prefetch)
constexpr int T2_PREFETCH = FLCE_PAIR_PREFETCH;
constexpr int T2_A_BYTES = T2_HALF * T2_BK * 2;  // 16 KB
constexpr int T2_B_BYTES = T2_HALF * T2_BK * 2;  // 16 KB
constexpr int T2_STAGE_BYTES = T2_A_BYTES + T2_B_BYTES;
constexpr int T2_STAGE_OUT_BYTES = 32 * 32 * 2;  // one 32 x 32 bf16 staging box
// Staging boxes per epilogue warp (a power of two): a box is reused once the
// TMA store (or L2 reduce-add) issued from it FLCE_OUT_BOXES stores ago has read
// it. Four instead of two cut the 16-chunk Llama-3-8B step by 0.5% (15 of its 16
// grad_W launches add into grad_W in L2); the 2-chunk step did not move.
#ifndef FLCE_OUT_BOXES
#define FLCE_OUT_BOXES 4
#endif
constexpr int T2_OUT_BOXES = FLCE_OUT_BOXES;
static_assert((T2_OUT_BOXES & (T2_OUT_BOXES - 1)) == 0, "a power of two");
constexpr int T2_OUT_BYTES = 4 * T2_OUT_BOXES * T2_STAGE_OUT_BYTES;
constexpr int T2_SMEM_BYTES = T2_STAGES * T2_STAGE_BYTES + T2_OUT_BYTES + 1024 + 256;

// Wide tiles (256 x 512 over the pair, for long-K problems such as grad_X):
// each CTA stages 128 rows of A and two 128-row N-halves of B per K-block, and
// the leader issues two N = 256 MMAs per K-step that share the A operand, into
// columns [0, 256) and [256, 512) of one accumulator that fills tensor memory.
// A is loaded once per 512 output columns instead of per 256, so L2-to-SM
// traffic per FLOP drops by a quarter, and a problem has half as many tiles
// (grad_X of a 2048-row chunk with H = 4096: 64 tiles, one wave on 74 pairs,
// so every operand byte is read from DRAM about once). The accumulator is not
// double-buffered: a tile's epilogue does not overlap the next tile's MMAs,
// which costs little when K is long.
#ifndef FLCE_WIDE_STAGES
#define FLCE_WIDE_STAGES 4
#endif
constexpr int T2W_STAGES = FLCE_WIDE_STAGES;
constexpr int T2W_BN = 512;
constexpr int T2W_B_BYTES = 2 * T2_B_BYTES;  // 32 KB
constexpr int T2W_STAGE_BYTES = T2_A_BYTES + T2W_B_BYTES;
constexpr int T2W_SMEM_BYTES = T2W_STAGES * T2W_STAGE_BYTES + T2_OUT_BYTES + 1024 + 256;

// Soft K-synchronisation of one-wave wide tiles (TcParams::kprog): at every
// KSYNC_EVERY-th K-block a pair adds one to that checkpoint's counter, then waits
// until every synchronised pair has passed the checkpoint FLCE_KSYNC_WINDOW K-blocks
// back (at most KSYNC_CAP_NS; after a wait that runs out the pair stops
// synchronising for the rest of the launch). One counter load per check.
constexpr int KSYNC_EVERY = 16;
#ifndef FLCE_KSYNC_WINDOW
#define FLCE_KSYNC_WINDOW 32
#endif
// checkpoints of lead allowed: 32 K-blocks keep the dz and W panels the pairs
// share to ~25 MB (at 64 K-blocks, ~50 MB, grad_X read 1.63 GB of DRAM against
// its 1.58 GB of operands on the same box; at 32 and 16, 1.58 GB)
constexpr int KSYNC_LAG = FLCE_KSYNC_WINDOW / KSYNC_EVERY;
constexpr int KSYNC_MAX_CKPT = 4096;                         // counters available (V up to 4M columns)
constexpr uint64_t KSYNC_CAP_NS = 20000;

__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// The epilogue of the first half of a wide tile hands nothing back yet.
struct NoRelease {
  __device__ __forceinline__ void operator()() const {}
};

// bf16 output tile through shared memory and TMA: each epilogue warp writes its
// 32 rows in 32-column boxes, alternating two staging boxes, and one lane
// stores (store = true) or adds (store = false, the add done in L2) each box.
// Rows and columns outside the tensor map's extent are clipped by the TMA.
// Output maps of grad_W shards (data parallelism): shard k owns rows
// [k * shard_rows, (k+1) * shard_rows) and may live on a peer GPU.
constexpr int MAX_SHARDS = 8;
struct ShardMaps {
  CUtensorMap m[MAX_SHARDS];
};
// The plain kernel takes this placeholder instead: carrying the 1 KB of shard
// maps as a kernel parameter measurably slowed every launch (14% per step),
// so only the sharded instantiation has them.
struct NoShards {
  int unused;
};

// With `local` (shard routing of the last row chunk), each box is first rounded
// to bf16, then this thread's row of the earlier chunks' bf16 partial sum is
// added to it and the sum rounded again: the same two roundings as the L2
// reduce-add that accumulates the unsharded grad_W, so one rank's shard equals
// the unsharded result bit for bit.
template <typename Release>
__device__ __forceinline__ void epi_bf16_tma(const CUtensorMap* tmC, bool store, int64_t M, int64_t N,
                                             int64_t rwarp, int tn, uint32_t taddr, uint8_t* boxes,
                                             uint32_t& issued, const Release& release,
                                             const ShardMaps* shards = nullptr, int64_t shard_rows = 0,
                                             const __nv_bfloat16* local = nullptr, int64_t ld_local = 0) {
  const int lane = threadIdx.x & 31;
  const int n0 = tn * 256;
  uint32_t v[32];
#pragma unroll 1
  for (int c = 0; c < 8; ++c) {
    __syncwarp();
    tmem_ld_32x32(taddr + c * 32, v);
    tmem_ld_wait();
    if (c == 7) release();
    if (rwarp >= M || n0 + c * 32 >= N) continue;  // whole box outside: warp-uniform
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
    if (local != nullptr && rwarp + lane < M) {
      // N % 8 == 0: each 8-column vector lies wholly inside or outside the matrix
      const __nv_bfloat16* src = local + (rwarp + lane) * ld_local + n0 + c * 32;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (n0 + c * 32 + 8 * q >= N) continue;
        const uint4 o = *reinterpret_cast<const uint4*>(src + 8 * q);
        const uint32_t w[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 a = unpack_bf16x2(pk[4 * q + k]), b = unpack_bf16x2(w[k]);
          pk[4 * q + k] = pack_bf16x2(a.x + b.x, a.y + b.y);
        }
      }
    }
    uint8_t* box = boxes + (issued & (T2_OUT_BOXES - 1)) * T2_STAGE_OUT_BYTES;
    if (issued >= (uint32_t)T2_OUT_BOXES) {
      if (lane == 0) bulk_wait_group_read<T2_OUT_BOXES - 1>();  // the box written two stores ago is free again
      __syncwarp();
    }
    uint4* dst = reinterpret_cast<uint4*>(box + lane * 64);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (shards) {
        // the box's 32 rows lie in one shard (shard_rows is a multiple of 32)
        const int owner = (int)(rwarp / shard_rows);
        tma_reduce_add_2d(&shards->m[owner], box, n0 + c * 32, (int32_t)(rwarp - owner * shard_rows));
      } else if (store) {
        tma_store_2d(tmC, box, n0 + c * 32, (int32_t)rwarp);
      } else {
        tma_reduce_add_2d(tmC, box, n0 + c * 32, (int32_t)rwarp);
      }
      bulk_commit_group();
    }
    ++issued;
  }
}

// Logits epilogue of the pair engine: as epi_logits (tile max, then e = exp(z - max),
// its sum and the target logit per row), but the bf16 e tile leaves through
// shared memory and TMA stores instead of per-row global stores.
template <typename Release>
__device__ __forceinline__ void epi_logits_tma(const TcParams& p, const TcProblem& P, const CUtensorMap* tmE,
                                               int64_t r_base, int q, int tn, int row, uint32_t taddr,
                                               uint8_t* boxes, uint32_t& issued, const Release& release) {
  const LogitsArgs& g = p.lg;
  const int lane = threadIdx.x & 31;
  const int64_t r = r_base + row;
  const int64_t rwarp = r_base + q * 32;
  const bool row_ok = r < P.M;
  const int64_t n0 = (int64_t)tn * TC_BN;
  const int ncols = (int)((g.V - n0) < TC_BN ? (g.V - n0) : TC_BN);
  int tcol = -1;
  if (row_ok) {
    const int64_t t = g.target[r];
    if (t != g.ignore_index && t >= n0 && t < n0 + ncols) tcol = (int)(t - n0);
  }
  uint32_t v[32];
  float mx = -INFINITY;
#pragma unroll 1
  for (int c = 0; c < TC_BN / 32; ++c) {
    __syncwarp();
    tmem_ld_32x32(taddr + c * 32, v);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (c * 32 + j < ncols) mx = fmaxf(mx, __uint_as_float(v[j]));
  }
  const float ms = mx * LOG2E_F;
  float s = 0.f, ztv = 0.f;
#pragma unroll 1
  for (int c = 0; c < TC_BN / 32; ++c) {
    __syncwarp();
    tmem_ld_32x32(taddr + c * 32, v);
    tmem_ld_wait();
    if (c == TC_BN / 32 - 1) release();
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const int col = c * 32 + j;
      const float z0 = __uint_as_float(v[j]), z1 = __uint_as_float(v[j + 1]);
      const float e0 = col < ncols ? ex2_approx(fmaf(z0, LOG2E_F, -ms)) : 0.f;
      const float e1 = col + 1 < ncols ? ex2_approx(fmaf(z1, LOG2E_F, -ms)) : 0.f;
      s += e0 + e1;
      if (col == tcol) ztv = z0;
      if (col + 1 == tcol) ztv = z1;
      pk[j / 2] = pack_bf16x2(e0, e1);
    }
    if (!g.store || rwarp >= P.M || c * 32 >= ncols) continue;  // no store / box wholly outside: warp-uniform
    uint8_t* box = boxes + (issued & (T2_OUT_BOXES - 1)) * T2_STAGE_OUT_BYTES;
    if (issued >= (uint32_t)T2_OUT_BOXES) {
      if (lane == 0) bulk_wait_group_read<T2_OUT_BOXES - 1>();
      __syncwarp();
    }
    uint4* dst = reinterpret_cast<uint4*>(box + lane * 64);
#pragma unroll
    for (int k = 0; k < 4; ++k) dst[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      // the store is read back only after the whole launch (525 MB later): first out of L2,
      // ahead of the W panels that the chunk's other row tiles are about to read
      tma_store_2d_hint(tmE, box, (int32_t)(n0 + c * 32), (int32_t)rwarp, l2_policy_evict_first());
      bulk_commit_group();
    }
    ++issued;
  }
  if (row_ok) {
    g.part_m[(int64_t)tn * g.ldp + r] = mx;
    g.part_s[(int64_t)tn * g.ldp + r] = s;
    if (tcol >= 0) g.zt[r] = ztv;
  }
}

// dlogits epilogue of the recompute schedule: the logits tile was just rebuilt
// by the GEMM, and the row's logsumexp is known from the first pass, so the
// gradient is written directly: dz = exp(z - lse) * s - [column = target] * s,
// s = row_grad * (1/N or 1), 0 for ignored rows; bf16 boxes leave by TMA store.
template <typename Release>
__device__ __forceinline__ void epi_dlogits_tma(const TcParams& p, const TcProblem& P, const CUtensorMap* tmE,
                                                int64_t r_base, int q, int tn, int row, uint32_t taddr,
                                                uint8_t* boxes, uint32_t& issued, const Release& release) {
  const LogitsArgs& g = p.lg;
  const int lane = threadIdx.x & 31;
  const int64_t r = r_base + row;
  const int64_t rwarp = r_base + q * 32;
  const int64_t n0 = (int64_t)tn * T2_BN;
  const int ncols = (int)((P.N - n0) < T2_BN ? (P.N - n0) : T2_BN);
  int tcol = -1;
  float sg = 0.f, ls = 0.f;
  if (r < P.M) {
    const int64_t t = g.target[r];
    if (t != g.ignore_index && t >= 0 && t < g.V) {
      float s = 1.f;
      if (g.reduction == 0) {
        const int64_t n = *g.n_valid;
        s = n > 0 ? 1.f / (float)n : 0.f;
      }
      sg = g.row_grad ? s * g.row_grad[r] : s;
      ls = g.lse[r] * LOG2E_F;
      const int64_t tc = t - g.v0 - n0;
      if (tc >= 0 && tc < ncols) tcol = (int)tc;
    }
  }
  uint32_t v[32];
#pragma unroll 1
  for (int c = 0; c < T2_BN / 32; ++c) {
    __syncwarp();
    tmem_ld_32x32(taddr + c * 32, v);
    tmem_ld_wait();
    if (c == T2_BN / 32 - 1) release();
    if (rwarp >= P.M || c * 32 >= ncols) continue;  // box wholly outside: warp-uniform
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const int col = c * 32 + j;
      float d0 = ex2_approx(fmaf(__uint_as_float(v[j]), LOG2E_F, -ls)) * sg;
      float d1 = ex2_approx(fmaf(__uint_as_float(v[j + 1]), LOG2E_F, -ls)) * sg;
      if (col == tcol) d0 -= sg;
      if (col + 1 == tcol) d1 -= sg;
      pk[j / 2] = pack_bf16x2(d0, d1);
    }
    uint8_t* box = boxes + (issued & (T2_OUT_BOXES - 1)) * T2_STAGE_OUT_BYTES;
    if (issued >= (uint32_t)T2_OUT_BOXES) {
      if (lane == 0) bulk_wait_group_read<T2_OUT_BOXES - 1>();
      __syncwarp();
    }
    uint4* dst = reinterpret_cast<uint4*>(box + lane * 64);
#pragma unroll
    for (int k = 0; k < 4; ++k) dst[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmE, box, (int32_t)(n0 + c * 32), (int32_t)rwarp);
      bulk_commit_group();
    }
    ++issued;
  }
}

struct ReleasePair {  // 2-CTA engine: one arrival per epilogue warp on the leader's barrier
  uint32_t leader_bar;  // shared::cluster address
  __device__ __forceinline__ void operator()() const {
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive_cluster(leader_bar);
  }
};

// kWide: 256 x 512 tiles (see T2W_*); used only with bf16 TMA-store epilogues
// (EPI_STORE_BF16, or EPI_GRADW in a bf16 store / add mode) and one problem.
template <typename ShardArg, bool kWide = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(TC_THREADS, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                        const __grid_constant__ CUtensorMap tmC0, const __grid_constant__ CUtensorMap tmC1,
                        const __grid_constant__ ShardArg shard_maps, const __grid_constant__ TcParams p) {
  constexpr bool kShards = sizeof(ShardArg) == sizeof(ShardMaps);
  // narrow tiles: each stage holds KSUB consecutive 64-wide K-blocks (one wait and one commit per KSUB)
  constexpr int KSUB = kWide ? 1 : 2;
  constexpr int SUB_BYTES = kWide ? T2W_STAGE_BYTES : T2_STAGE_BYTES;
  constexpr int STAGES = kWide ? T2W_STAGES : T2_STAGES / KSUB;
  constexpr int STAGE_BYTES = KSUB * SUB_BYTES;
  constexpr int TILE_N = kWide ? T2W_BN : T2_BN;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* out_boxes = smem + STAGES * STAGE_BYTES;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(out_boxes + T2_OUT_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* mma_done_bar = tempty_bar + 2;
  uint64_t* stall_bar = mma_done_bar + 1;  // failure-path test: never arrived on
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(stall_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, G = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 2 * 4);
    }
    mbar_init(mma_done_bar, 1);
    mbar_init(stall_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmB0);
    if (p.nprob > 1) {
      tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmB1);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, TC_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // both CTAs' barriers must be initialised before any remote arrive or load
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const TileSched sched = make_sched(p, pair, G);
  const int ntiles = sched_count(sched);

  if (warp == 0) {
    // ---------------------------------------------------------- producer (both CTAs)
    if (lane == 0) {
      uint32_t kit = 0;
      bool ok = true;
      // the leader's producer keeps its pair in step (the peer's follows through the MMA commits)
      bool ksync = kWide && leader && p.kprog != nullptr && pair < p.ksync_pairs &&
                   p.prob[0].kblocks / KSYNC_EVERY < KSYNC_MAX_CKPT;
      for (int i = 0; i < ntiles && ok; ++i) {
        const Tile T = sched_tile(p, sched, pair, G, i);
        const int pi = T.prob, tm = T.tm, tn = T.tn;
        const TcProblem& P = p.prob[pi];
        const CUtensorMap* tA = pi == 0 ? &tmA0 : &tmA1;
        const CUtensorMap* tB = pi == 0 ? &tmB0 : &tmB1;
        const int am0 = tm * T2_BM + (int)rank * T2_HALF;  // this CTA's rows of A
        const int bn0 = tn * TILE_N + (int)rank * T2_HALF;  // this CTA's rows of B (wide: and bn0 + 256)
        for (int kb = T.kb0; kb < T.kb1; kb += KSUB, ++kit) {
          const int nsub = T.kb1 - kb < KSUB ? T.kb1 - kb : KSUB;
          if (kWide && ksync && (kb % KSYNC_EVERY) == 0) {
            // arrive at this checkpoint, then hold back while a pair is still KSYNC_LAG checkpoints behind
            const int c = kb / KSYNC_EVERY;
            atomicAdd(p.kprog + c, 1u);
            if (c >= KSYNC_LAG) {
              const uint32_t* behind = p.kprog + (c - KSYNC_LAG);
              const uint64_t t0 = globaltimer_ns();
              while (ld_relaxed_gpu(behind) < (uint32_t)p.ksync_pairs) {
                if (globaltimer_ns() - t0 > KSYNC_CAP_NS || *abort_flag) {
                  ksync = false;
                  break;
                }
                __nanosleep(256);
              }
            }
          }
          const int stage = kit % STAGES;
          const uint32_t phase = (kit / STAGES) & 1;
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.err)) { ok = false; break; }
          // every box is issued (out-of-range parts read as zero), so each
          // CTA contributes exactly nsub sub-blocks' bytes
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * nsub * SUB_BYTES);
          const uint32_t fb = mapa_shared(smem_u32(&full_bar[stage]), 0);
          for (int j = 0; j < nsub; ++j) {
            uint8_t* sA = smem + stage * STAGE_BYTES + j * SUB_BYTES;
            uint8_t* sB = sA + T2_A_BYTES;
            const int k0 = (kb + j) * T2_BK;
            if (!P.a_mn) {
              tma_load_2d_pair(sA, tA, fb, k0, am0);
            } else {
              tma_load_2d_pair(sA, tA, fb, am0, k0);
              tma_load_2d_pair(sA + 8192, tA, fb, am0 + 64, k0);
            }
            if (!P.b_mn) {
              tma_load_2d_pair(sB, tB, fb, k0, bn0);
              if (kWide) tma_load_2d_pair(sB + T2_B_BYTES, tB, fb, k0, bn0 + 256);
            } else {
              tma_load_2d_pair(sB, tB, fb, bn0, k0);
              tma_load_2d_pair(sB + 8192, tB, fb, bn0 + 64, k0);
              if (kWide) {
                tma_load_2d_pair(sB + T2_B_BYTES, tB, fb, bn0 + 256, k0);
                tma_load_2d_pair(sB + T2_B_BYTES + 8192, tB, fb, bn0 + 320, k0);
              }
            }
          }
          const int k0 = kb * T2_BK;
          // warm L2 for a later K-block so the load above it finds its data there
          if (!kWide && T2_PREFETCH > 0 && kb + T2_PREFETCH < T.kb1) {
            const int kp = k0 + T2_PREFETCH * T2_BK;
            if (!P.a_mn) {
              tma_prefetch_2d(tA, kp, am0);
            } else {
              tma_prefetch_2d(tA, am0, kp);
              tma_prefetch_2d(tA, am0 + 64, kp);
            }
            if (!P.b_mn) {
              tma_prefetch_2d(tB, kp, bn0);
            } else {
              tma_prefetch_2d(tB, bn0, kp);
              tma_prefetch_2d(tB, bn0 + 64, kp);
            }
          }
        }
      }
      if (!ok && leader) {
        // drain: the leader's full barriers also count the peer's bytes
        volatile int no_abort = 0;
        for (uint32_t j = kit > (uint32_t)STAGES ? kit - STAGES : 0; j < kit; ++j)
          mbar_wait(&full_bar[j % STAGES], (j / STAGES) & 1, &no_abort, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      uint32_t kit = 0;
      bool ok = true;
      for (int i = 0; i < ntiles && ok; ++i) {
        const Tile T = sched_tile(p, sched, pair, G, i);
        const TcProblem& P = p.prob[T.prob];
        // narrow: accumulators alternate; wide: one accumulator of all 512 columns
        const int acc = kWide ? 0 : (i & 1);
        const uint32_t aph = kWide ? (i & 1) : ((i >> 1) & 1);
        if (!mbar_wait(&tempty_bar[acc], aph ^ 1, abort_flag, p.err)) { ok = false; break; }
        // failure-path test: this wait can only run out (after the wait limit)
        if (p.test_stall > 0 && i == p.test_stall - 1 && !mbar_wait(stall_bar, 0, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * T2_BN;
        const uint32_t idesc = idesc_bf16_f32(P.a_mn, P.b_mn, T2_BM, T2_BN);
        for (int kb = T.kb0; kb < T.kb1; kb += KSUB, ++kit) {
          const int nsub = T.kb1 - kb < KSUB ? T.kb1 - kb : KSUB;
          const int stage = kit % STAGES;
          const uint32_t phase = (kit / STAGES) & 1;
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.err)) { ok = false; break; }
          if (FLCE_PAIR_KFENCE) tc_fence_after();
#pragma unroll
          for (int j = 0; j < KSUB; ++j) {
            if (j >= nsub) break;
            const uint32_t a_base = smem_u32(smem + stage * STAGE_BYTES + j * SUB_BYTES);
            const uint32_t b_base = a_base + T2_A_BYTES;
#pragma unroll
            for (int k = 0; k < T2_BK / 16; ++k) {
              const uint64_t ad = P.a_mn ? smem_desc_sw128(a_base + k * 2048, 8192, 1024)
                                         : smem_desc_sw128(a_base + k * 32, 16, 1024);
              const uint64_t bd = P.b_mn ? smem_desc_sw128(b_base + k * 2048, 8192, 1024)
                                         : smem_desc_sw128(b_base + k * 32, 16, 1024);
              tc_mma_bf16_pair(d_tmem, ad, bd, idesc, (kb != T.kb0) || (j != 0) || (k != 0));
              if (kWide) {
                // the second N-half of the tile, same A: columns [256, 512) of the accumulator
                const uint32_t b2 = b_base + T2_B_BYTES;
                const uint64_t bd2 = P.b_mn ? smem_desc_sw128(b2 + k * 2048, 8192, 1024)
                                            : smem_desc_sw128(b2 + k * 32, 16, 1024);
                tc_mma_bf16_pair(d_tmem + T2_BN, ad, bd2, idesc, (kb != T.kb0) || (j != 0) || (k != 0));
              }
            }
          }
          tc_commit_pair_mc(&empty_bar[stage], 0x3);
        }
        if (ok) tc_commit_pair_mc(&tfull_bar[acc], 0x3);
      }
      if (kit > 0) {
        tc_commit_pair_mc(mma_done_bar, 0x1);
        volatile int no_abort = 0;
        mbar_wait(mma_done_bar, 0, &no_abort, p.err);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    uint8_t* my_boxes = out_boxes + (warp - 2) * T2_OUT_BOXES * T2_STAGE_OUT_BYTES;
    uint32_t issued = 0;  // TMA output boxes this warp has issued
    for (int i = 0; i < ntiles; ++i) {
      const Tile T = sched_tile(p, sched, pair, G, i);
      const TcProblem& P = p.prob[T.prob];
      const int tm = T.tm, tn = T.tn;
      const int acc = kWide ? 0 : (i & 1);
      const uint32_t aph = kWide ? (i & 1) : ((i >> 1) & 1);
      const bool ok = mbar_wait(&tfull_bar[acc], aph, abort_flag, p.err, FLCE_EPI_BACKOFF_NS);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * T2_BN;
      const ReleasePair rel{mapa_shared(smem_u32(&tempty_bar[acc]), 0)};
      const int64_t r_base = (int64_t)tm * T2_BM + rank * T2_HALF;
      const bool tma_out = P.epi == EPI_STORE_BF16 ||
                           (P.epi == EPI_GRADW && (P.gw_mode == GW_STORE_BF16 || P.gw_mode == GW_ADD_BF16));
      if constexpr (kWide) {
        // the two 256-column halves in turn; the accumulator goes back after the second
        const CUtensorMap* tC = T.prob == 0 ? &tmC0 : &tmC1;
        const bool store = P.epi == EPI_STORE_BF16 || P.gw_mode == GW_STORE_BF16;
        epi_bf16_tma(tC, store, P.M, P.N, r_base + q * 32, 2 * tn, taddr, my_boxes, issued, NoRelease{});
        epi_bf16_tma(tC, store, P.M, P.N, r_base + q * 32, 2 * tn + 1, taddr + T2_BN, my_boxes, issued, rel);
      } else if (P.epi == EPI_LOGITS)
        epi_logits_tma(p, P, &tmC0, r_base, q, tn, row, taddr, my_boxes, issued, rel);
      else if (P.epi == EPI_DLOGITS)
        epi_dlogits_tma(p, P, &tmC0, r_base, q, tn, row, taddr, my_boxes, issued, rel);
      else if (kShards && P.epi == EPI_GRADW && P.n_shards > 0)
        epi_bf16_tma(nullptr, false, P.M, P.N, r_base + q * 32, tn, taddr, my_boxes, issued, rel,
                     reinterpret_cast<const ShardMaps*>(&shard_maps), P.shard_rows,
                     static_cast<const __nv_bfloat16*>(P.gw_local), P.ld_local);
      else if (tma_out)
        epi_bf16_tma(T.prob == 0 ? &tmC0 : &tmC1, P.epi == EPI_STORE_BF16 || P.gw_mode == GW_STORE_BF16, P.M, P.N,
                     r_base + q * 32, tn, taddr, my_boxes, issued, rel);
      else
        epi_store(P, r_base, tn, T.split, row, taddr, rel);
    }
    // every output box must be written before the CTA exits
    if (lane == 0 && issued > 0) bulk_wait_group_all();
    __syncwarp();
  }

  tc_fence_before();
  // neither CTA may leave while the pair's MMAs, loads or arrivals can still touch it
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TC_TMEM_COLS);
  }
}

}  // namespace flce
