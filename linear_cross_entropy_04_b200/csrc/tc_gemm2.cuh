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
constexpr int T2_STAGES = FLCE_PAIR_STAGES;
// K-blocks between an L2 prefetch and the load of the same box (0: no prefetch)
constexpr int T2_PREFETCH = FLCE_PAIR_PREFETCH;
constexpr int T2_A_BYTES = T2_HALF * T2_BK * 2;  // 16 KB
constexpr int T2_B_BYTES = T2_HALF * T2_BK * 2;  // 16 KB
constexpr int T2_STAGE_BYTES = T2_A_BYTES + T2_B_BYTES;
constexpr int T2_STAGE_OUT_BYTES = 32 * 32 * 2;  // one 32 x 32 bf16 staging box
constexpr int T2_OUT_BYTES = 4 * 2 * T2_STAGE_OUT_BYTES;  // 4 epilogue warps x 2 boxes
constexpr int T2_SMEM_BYTES = T2_STAGES * T2_STAGE_BYTES + T2_OUT_BYTES + 1024 + 256;

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

template <typename Release>
__device__ __forceinline__ void epi_bf16_tma(const CUtensorMap* tmC, bool store, int64_t M, int64_t N,
                                             int64_t rwarp, int tn, uint32_t taddr, uint8_t* boxes,
                                             uint32_t& issued, const Release& release,
                                             const ShardMaps* shards = nullptr, int64_t shard_rows = 0) {
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
    uint8_t* box = boxes + (issued & 1) * T2_STAGE_OUT_BYTES;
    if (issued >= 2) {
      if (lane == 0) bulk_wait_group_read<1>();  // the box written two stores ago is free again
      __syncwarp();
    }
    uint4* dst = reinterpret_cast<uint4*>(box + lane * 64);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      dst[q] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                          pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                          pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                          pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
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
      const float e0 = col < ncols ? exp2f(fmaf(z0, LOG2E_F, -ms)) : 0.f;
      const float e1 = col + 1 < ncols ? exp2f(fmaf(z1, LOG2E_F, -ms)) : 0.f;
      s += e0 + e1;
      if (col == tcol) ztv = z0;
      if (col + 1 == tcol) ztv = z1;
      pk[j / 2] = pack_bf16x2(e0, e1);
    }
    if (rwarp >= P.M || c * 32 >= ncols) continue;  // box wholly outside: warp-uniform
    uint8_t* box = boxes + (issued & 1) * T2_STAGE_OUT_BYTES;
    if (issued >= 2) {
      if (lane == 0) bulk_wait_group_read<1>();
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
  if (row_ok) {
    g.part_m[(int64_t)tn * g.ldp + r] = mx;
    g.part_s[(int64_t)tn * g.ldp + r] = s;
    if (tcol >= 0) g.zt[r] = ztv;
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

template <typename ShardArg>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(TC_THREADS, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                        const __grid_constant__ CUtensorMap tmC0, const __grid_constant__ CUtensorMap tmC1,
                        const __grid_constant__ ShardArg shard_maps, const __grid_constant__ TcParams p) {
  constexpr bool kShards = sizeof(ShardArg) == sizeof(ShardMaps);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* out_boxes = smem + T2_STAGES * T2_STAGE_BYTES;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(out_boxes + T2_OUT_BYTES);
  uint64_t* empty_bar = full_bar + T2_STAGES;
  uint64_t* tfull_bar = empty_bar + T2_STAGES;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* mma_done_bar = tempty_bar + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, G = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T2_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 2 * 4);
    }
    mbar_init(mma_done_bar, 1);
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
      for (int i = 0; i < ntiles && ok; ++i) {
        const Tile T = sched_tile(p, sched, pair, G, i);
        const int pi = T.prob, tm = T.tm, tn = T.tn;
        const TcProblem& P = p.prob[pi];
        const CUtensorMap* tA = pi == 0 ? &tmA0 : &tmA1;
        const CUtensorMap* tB = pi == 0 ? &tmB0 : &tmB1;
        const int am0 = tm * T2_BM + (int)rank * T2_HALF;  // this CTA's rows of A
        const int bn0 = tn * T2_BN + (int)rank * T2_HALF;  // this CTA's rows of B
        for (int kb = T.kb0; kb < T.kb1; ++kb, ++kit) {
          const int stage = kit % T2_STAGES;
          const uint32_t phase = (kit / T2_STAGES) & 1;
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.err)) { ok = false; break; }
          uint8_t* sA = smem + stage * T2_STAGE_BYTES;
          uint8_t* sB = sA + T2_A_BYTES;
          // every box is issued (out-of-range parts read as zero), so each
          // CTA contributes exactly one stage's bytes
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * T2_STAGE_BYTES);
          const uint32_t fb = mapa_shared(smem_u32(&full_bar[stage]), 0);
          const int k0 = kb * T2_BK;
          if (!P.a_mn) {
            tma_load_2d_pair(sA, tA, fb, k0, am0);
          } else {
            tma_load_2d_pair(sA, tA, fb, am0, k0);
            tma_load_2d_pair(sA + 8192, tA, fb, am0 + 64, k0);
          }
          if (!P.b_mn) {
            tma_load_2d_pair(sB, tB, fb, k0, bn0);
          } else {
            tma_load_2d_pair(sB, tB, fb, bn0, k0);
            tma_load_2d_pair(sB + 8192, tB, fb, bn0 + 64, k0);
          }
          // warm L2 for a later K-block so the load above it finds its data there
          if (T2_PREFETCH > 0 && kb + T2_PREFETCH < T.kb1) {
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
        for (uint32_t j = kit > T2_STAGES ? kit - T2_STAGES : 0; j < kit; ++j)
          mbar_wait(&full_bar[j % T2_STAGES], (j / T2_STAGES) & 1, &no_abort, nullptr);
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
        const int acc = i & 1;
        const uint32_t aph = (i >> 1) & 1;
        if (!mbar_wait(&tempty_bar[acc], aph ^ 1, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * T2_BN;
        const uint32_t idesc = idesc_bf16_f32(P.a_mn, P.b_mn, T2_BM, T2_BN);
        for (int kb = T.kb0; kb < T.kb1; ++kb, ++kit) {
          const int stage = kit % T2_STAGES;
          const uint32_t phase = (kit / T2_STAGES) & 1;
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.err)) { ok = false; break; }
          if (FLCE_PAIR_KFENCE) tc_fence_after();
          const uint32_t a_base = smem_u32(smem + stage * T2_STAGE_BYTES);
          const uint32_t b_base = a_base + T2_A_BYTES;
#pragma unroll
          for (int k = 0; k < T2_BK / 16; ++k) {
            const uint64_t ad = P.a_mn ? smem_desc_sw128(a_base + k * 2048, 8192, 1024)
                                       : smem_desc_sw128(a_base + k * 32, 16, 1024);
            const uint64_t bd = P.b_mn ? smem_desc_sw128(b_base + k * 2048, 8192, 1024)
                                       : smem_desc_sw128(b_base + k * 32, 16, 1024);
            tc_mma_bf16_pair(d_tmem, ad, bd, idesc, (kb != T.kb0) || (k != 0));
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
    uint8_t* my_boxes = out_boxes + (warp - 2) * 2 * T2_STAGE_OUT_BYTES;
    uint32_t issued = 0;  // TMA output boxes this warp has issued
    for (int i = 0; i < ntiles; ++i) {
      const Tile T = sched_tile(p, sched, pair, G, i);
      const TcProblem& P = p.prob[T.prob];
      const int tm = T.tm, tn = T.tn;
      const int acc = i & 1;
      const uint32_t aph = (i >> 1) & 1;
      const bool ok = mbar_wait(&tfull_bar[acc], aph, abort_flag, p.err, FLCE_EPI_BACKOFF_NS);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * T2_BN;
      const ReleasePair rel{mapa_shared(smem_u32(&tempty_bar[acc]), 0)};
      const int64_t r_base = (int64_t)tm * T2_BM + rank * T2_HALF;
      const bool tma_out = P.epi == EPI_STORE_BF16 ||
                           (P.epi == EPI_GRADW && (P.gw_mode == GW_STORE_BF16 || P.gw_mode == GW_ADD_BF16));
      if (P.epi == EPI_LOGITS)
        epi_logits_tma(p, P, &tmC0, r_base, q, tn, row, taddr, my_boxes, issued, rel);
      else if (kShards && P.epi == EPI_GRADW && P.n_shards > 0)
        epi_bf16_tma(nullptr, false, P.M, P.N, r_base + q * 32, tn, taddr, my_boxes, issued, rel,
                     reinterpret_cast<const ShardMaps*>(&shard_maps), P.shard_rows);
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
