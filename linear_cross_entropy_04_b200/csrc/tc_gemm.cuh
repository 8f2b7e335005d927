// Persistent tcgen05 GEMM engine for sm_100a with fused epilogues.
//
// One CTA per SM, 192 threads in three roles:
//   warp 0      TMA producer: loads A and B tiles (K-block of 64) into a
//               4-stage shared-memory ring, 128-byte swizzled;
//   warp 1      MMA issuer: one thread issues tcgen05.mma (M=128, N=256, K=16)
//               into one of two 256-column fp32 accumulators in tensor memory;
//               it also owns the tensor-memory allocation;
//   warps 2-5   epilogue: each thread owns one accumulator row (tensor-memory
//               lane), reads it with tcgen05.ld and applies the epilogue while
//               the MMA warp already fills the other accumulator.
//
// A launch runs one problem, or two problems from one persistent tile list
// (grad_X and grad_W of a row chunk): the long grad_X tiles (K = V) are dealt
// round-robin and the short grad_W tiles (K = chunk rows) fill each CTA up to
// an even share of the K-blocks, so the SMs finish together.
//
// Operands are K-major ([rows, K] row-major, one TMA box of 64 x rows) or
// MN-major ([K, rows] row-major, boxes of 64 MN-elements x 64 K-rows), which
// lets grad_X = dz W and grad_W = dz^T X read dz, W and X where they lie.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace flce {

constexpr int TC_BM = 128;
constexpr int TC_BN = 256;
constexpr int TC_BK = 64;
constexpr int TC_STAGES = 4;
constexpr int TC_A_BYTES = TC_BM * TC_BK * 2;  // 16 KB
constexpr int TC_B_BYTES = TC_BN * TC_BK * 2;  // 32 KB
constexpr int TC_STAGE_BYTES = TC_A_BYTES + TC_B_BYTES;
constexpr int TC_THREADS = 192;
constexpr int TC_TMEM_COLS = 512;  // two 128 x 256 fp32 accumulators
constexpr int TC_SMEM_BYTES = TC_STAGES * TC_STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;


enum EpiKind : int {
  EPI_LOGITS = 0,  // online-softmax partials + stored exp(z - m_tile) (bf16)
  EPI_STORE_BF16 = 1,
  EPI_GRADW = 2,
  EPI_STORE_F32 = 3,
  EPI_DLOGITS = 4,  // recompute schedule: dz = (exp(z - lse) - onehot) * scale, stored bf16
};

enum GradWMode : int {
  GW_STORE_BF16 = 0,   // out = bf16(acc)
  GW_ADD_BF16 = 1,     // out = bf16(out + acc)
  GW_STORE_F32 = 2,    // facc = acc
  GW_ADD_F32 = 3,      // facc += acc
  GW_FINAL_F32 = 4,    // out = bf16(facc + acc)
};

struct TcProblem {
  int M, N, K;
  int tiles_m, tiles_n, kblocks;
  int a_mn, b_mn;      // 0 = K-major operand, 1 = MN-major operand
  int epi;             // EpiKind
  int m_fastest;       // tile order: 1 -> consecutive tiles step m, 0 -> step n
  void* out;           // output base (bf16 or f32)
  int64_t ldo;         // output leading dimension (elements)
  int gw_mode;         // GradWMode (EPI_GRADW)
  float* facc;         // fp32 grad_W accumulator (GW_*_F32 modes)
  int64_t ld_facc;
  int n_shards;        // EPI_GRADW: > 0 routes each output box to its owner shard (add)
  int64_t shard_rows;  // rows per shard (multiple of 32)
  const void* gw_local;  // EPI_GRADW with shards: bf16 [M, ld_local] partial sum of the earlier
  int64_t ld_local;      // chunks, added to this tile before it goes to the owner shard (or null)
  int group_m;         // > 0: tiles run in groups of group_m tile rows, m fastest inside a group
                       // (each B column tile is reused by the group's rows while they share L2)
  int ksplit;          // split-K factor (>= 1): tile t covers K-blocks of split t / (tiles_m*tiles_n)
  int kb_per_split;    // K-blocks per split
  int64_t split_stride;  // elements between the output slices of consecutive splits
};

// One unit of work: output tile (tm, tn) of problem `prob` over K-blocks [kb0, kb1).
struct Tile {
  int prob, tm, tn, kb0, kb1, split;
};

struct LogitsArgs {
  const int64_t* target;  // chunk row 0
  int64_t ignore_index;
  int64_t V;
  __nv_bfloat16* e_store;  // [rows, lde]: bf16(exp(z - m_tile))
  int64_t lde;
  float* part_m;           // [ntile, ldp]: per (tile, row) max of z
  float* part_s;           // [ntile, ldp]: per (tile, row) sum of exp(z - m_tile)
  int64_t ldp;
  float* zt;               // [rows]: z at the target column
  int store;               // EPI_LOGITS on the pair engine: 0 = partials only, no store
  // EPI_DLOGITS (recompute schedule): columns [0, N) of the launch are vocabulary
  // columns [v0, v0 + N); V above is the whole vocabulary (for target validity)
  const float* lse;        // [rows]: row logsumexp from the first pass
  const int64_t* n_valid;  // mean denominator N (device)
  int reduction;           // 0 mean (scale 1/N), 1 sum, 2 none
  const float* row_grad;   // [rows] upstream gradient per row, or null (all ones)
  int64_t v0;
};

struct TcParams {
  TcProblem prob[2];
  int nprob;
  LogitsArgs lg;
  uint32_t* err;
  // Test of the failure path (pair engine; 0 = off): the MMA issuer waits, before
  // its output tile number test_stall - 1, on a barrier nothing arrives on, so the
  // bounded wait runs out and the kernel takes its abort path.
  int test_stall;
  // Wide tiles in one wave: pairs [0, ksync_pairs) count their arrivals at every
  // KSYNC_EVERY-th K-block in kprog[checkpoint] (zeroed before the launch), and a
  // pair waits a bounded time at a checkpoint until every pair has passed the one
  // FLCE_KSYNC_WINDOW K-blocks back, so that the dz and W panels the tiles share stay
  // in L2 between their readers. 0 = off. A performance hint only: nothing
  // depends on it for correctness.
  uint32_t* kprog;
  int ksync_pairs;
};

// ------------------------------------------------------------ tile schedule
struct TileSched {
  int n0_mine;    // tiles of problem 0 owned by this CTA (round-robin)
  int p1_begin;   // [p1_begin, p1_end): contiguous tiles of problem 1
  int p1_end;
};

__device__ __forceinline__ int rr_count(int ntiles, int cta, int G) {
  return ntiles > cta ? (ntiles - 1 - cta) / G + 1 : 0;
}

__device__ TileSched make_sched(const TcParams& p, int cta, int G) {
  TileSched s;
  const TcProblem& P0 = p.prob[0];
  const int n0 = P0.tiles_m * P0.tiles_n * P0.ksplit;
  s.n0_mine = rr_count(n0, cta, G);
  s.p1_begin = s.p1_end = 0;
  if (p.nprob < 2) return s;
  const TcProblem& P1 = p.prob[1];
  const int64_t n1 = (int64_t)P1.tiles_m * P1.tiles_n * P1.ksplit;
  // per-tile cost in K-blocks, plus two for the epilogue and hand-offs
  const int64_t c0 = P0.kb_per_split + 2, c1 = P1.kb_per_split + 2;
  const int64_t target = ((int64_t)n0 * c0 + n1 * c1) / G;
  int64_t before = 0, total = 0, mine = 0;
  for (int j = 0; j < G; ++j) {
    int64_t d = target - (int64_t)rr_count(n0, j, G) * c0;
    d = d > 0 ? d : 0;
    if (j < cta) before += d;
    if (j == cta) mine = d;
    total += d;
  }
  if (total > 0) {
    s.p1_begin = (int)((n1 * before) / total);
    s.p1_end = (int)((n1 * (before + mine)) / total);
  } else if (cta == 0) {
    s.p1_begin = 0;
    s.p1_end = (int)n1;
  }
  return s;
}

__device__ __forceinline__ int sched_count(const TileSched& s) {
  return s.n0_mine + (s.p1_end - s.p1_begin);
}

__device__ __forceinline__ Tile sched_tile(const TcParams& p, const TileSched& s, int cta, int G, int i) {
  Tile T;
  int t;
  if (i < s.n0_mine) {
    T.prob = 0;
    t = cta + i * G;
  } else {
    T.prob = 1;
    t = s.p1_begin + (i - s.n0_mine);
  }
  const TcProblem& P = p.prob[T.prob];
  const int per_split = P.tiles_m * P.tiles_n;
  T.split = t / per_split;
  t -= T.split * per_split;
  if (P.group_m > 0) {
    const int per_group = P.group_m * P.tiles_n;
    const int grp = t / per_group;
    const int first_m = grp * P.group_m;
    const int gm = min(P.group_m, P.tiles_m - first_m);
    const int w = t - grp * per_group;
    T.tm = first_m + w % gm;
    T.tn = w / gm;
  } else if (P.m_fastest) {
    T.tm = t % P.tiles_m;
    T.tn = t / P.tiles_m;
  } else {
    T.tn = t % P.tiles_n;
    T.tm = t / P.tiles_n;
  }
  T.kb0 = T.split * P.kb_per_split;
  T.kb1 = min(P.kblocks, T.kb0 + P.kb_per_split);
  return T;
}

// ------------------------------------------------------------ epilogues
// Each thread holds accumulator row `row` (tile-local 0..127) of tile (tm, tn).
// taddr addresses column 0 of that row's 32-lane group in the ready accumulator.

// Hands the accumulator back to the MMA issuer once this thread's reads are done.
struct ReleaseLocal {  // 1-CTA engine: all 128 epilogue threads arrive
  uint64_t* bar;
  __device__ __forceinline__ void operator()() const {
    tc_fence_before();
    mbar_arrive(bar);
  }
};

template <typename Release>
__device__ __forceinline__ void epi_logits(const TcParams& p, const TcProblem& P, int64_t r_base, int tn,
                                           int row, uint32_t taddr, const Release& release) {
  const LogitsArgs& g = p.lg;
  const int64_t r = r_base + row;
  const bool row_ok = r < P.M;
  const int64_t n0 = (int64_t)tn * TC_BN;
  const int ncols = (int)((g.V - n0) < TC_BN ? (g.V - n0) : TC_BN);
  int tcol = -1;
  if (row_ok) {
    const int64_t t = g.target[r];
    if (t != g.ignore_index && t >= n0 && t < n0 + ncols) tcol = (int)(t - n0);
  }
  uint32_t v[32];
  // pass 1: the tile maximum of this row
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
  // pass 2: e = exp(z - mx), its sum, the target logit, and the bf16 store
  const float ms = mx * LOG2E_F;
  float s = 0.f, ztv = 0.f;
  __nv_bfloat16* erow = g.e_store + r * g.lde + n0;
#pragma unroll 1
  for (int c = 0; c < TC_BN / 32; ++c) {
    __syncwarp();
    tmem_ld_32x32(taddr + c * 32, v);
    tmem_ld_wait();
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
    if (row_ok && c * 32 < ncols) {
      if (c * 32 + 32 <= ncols) {
        uint4* dst = reinterpret_cast<uint4*>(erow + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      } else {
        unsigned short* dst = reinterpret_cast<unsigned short*>(erow + c * 32);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c * 32 + j < ncols) dst[j] = (unsigned short)((pk[j / 2] >> ((j & 1) * 16)) & 0xFFFFu);
      }
    }
  }
  // the accumulator is no longer needed: hand it back to the MMA warp
  release();
  if (row_ok) {
    g.part_m[(int64_t)tn * g.ldp + r] = mx;
    g.part_s[(int64_t)tn * g.ldp + r] = s;
    if (tcol >= 0) g.zt[r] = ztv;
  }
}

template <typename Release>
__device__ __forceinline__ void epi_store(const TcProblem& P, int64_t r_base, int tn, int split, int row,
                                          uint32_t taddr, const Release& release) {
  const int64_t r = r_base + row;
  const bool row_ok = r < P.M;
  const int64_t n0 = (int64_t)tn * TC_BN;
  const int ncols = (int)((P.N - n0) < TC_BN ? (P.N - n0) : TC_BN);
  uint32_t v[32];
#pragma unroll 1
  for (int c = 0; c < TC_BN / 32; ++c) {
    __syncwarp();
    tmem_ld_32x32(taddr + c * 32, v);
    tmem_ld_wait();
    if (c == TC_BN / 32 - 1) release();
    if (!row_ok || c * 32 >= ncols) continue;
    const bool full = c * 32 + 32 <= ncols;
    const int64_t col0 = n0 + c * 32;
    if (P.epi == EPI_STORE_F32) {
      float* dst = reinterpret_cast<float*>(P.out) + split * P.split_stride + r * P.ldo + col0;
      if (full) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          reinterpret_cast<uint4*>(dst)[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c * 32 + j < ncols) dst[j] = __uint_as_float(v[j]);
      }
      continue;
    }
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(P.out) + r * P.ldo + col0;
    float a[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) a[j] = __uint_as_float(v[j]);
    if (P.epi == EPI_GRADW) {
      const int mode = P.gw_mode;
      if (mode == GW_STORE_F32 || mode == GW_ADD_F32 || mode == GW_FINAL_F32) {
        float* fa = P.facc + r * P.ld_facc + col0;
        if (mode != GW_STORE_F32) {
          if (full) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 o = reinterpret_cast<const float4*>(fa)[q];
              a[4 * q] += o.x; a[4 * q + 1] += o.y; a[4 * q + 2] += o.z; a[4 * q + 3] += o.w;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c * 32 + j < ncols) a[j] += fa[j];
          }
        }
        if (mode != GW_FINAL_F32) {
          if (full) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              reinterpret_cast<float4*>(fa)[q] = make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c * 32 + j < ncols) fa[j] = a[j];
          }
          continue;
        }
      } else if (mode == GW_ADD_BF16) {
        if (full) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 o = reinterpret_cast<const uint4*>(dst)[q];
            const uint32_t w[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 f = unpack_bf16x2(w[k]);
              a[8 * q + 2 * k] += f.x;
              a[8 * q + 2 * k + 1] += f.y;
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c * 32 + j < ncols) a[j] += __bfloat162float(dst[j]);
        }
      }
    }
    if (full) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        reinterpret_cast<uint4*>(dst)[q] =
            make_uint4(pack_bf16x2(a[8 * q], a[8 * q + 1]), pack_bf16x2(a[8 * q + 2], a[8 * q + 3]),
                       pack_bf16x2(a[8 * q + 4], a[8 * q + 5]), pack_bf16x2(a[8 * q + 6], a[8 * q + 7]));
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (c * 32 + j < ncols) dst[j] = __float2bfloat16_rn(a[j]);
    }
  }
}

// ------------------------------------------------------------ the kernel
__global__ void __launch_bounds__(TC_THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + TC_STAGES * TC_STAGE_BYTES);
  uint64_t* empty_bar = full_bar + TC_STAGES;
  uint64_t* tfull_bar = empty_bar + TC_STAGES;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* mma_done_bar = tempty_bar + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x, G = gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 4 * 32);
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
    tmem_alloc(tmem_holder, TC_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const TileSched sched = make_sched(p, cta, G);
  const int ntiles = sched_count(sched);

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      uint32_t kit = 0;  // K-blocks issued so far: stage kit % STAGES, phase (kit / STAGES) & 1
      bool ok = true;
      for (int i = 0; i < ntiles && ok; ++i) {
        const Tile T = sched_tile(p, sched, cta, G, i);
        const int pi = T.prob, tm = T.tm, tn = T.tn;
        const TcProblem& P = p.prob[pi];
        const CUtensorMap* tA = pi == 0 ? &tmA0 : &tmA1;
        const CUtensorMap* tB = pi == 0 ? &tmB0 : &tmB1;
        const int m0 = tm * TC_BM, n0 = tn * TC_BN;
        // boxes lying wholly outside the M or N extent are skipped; the
        // accumulator rows/columns they would feed are never stored
        int a_boxes = 1, b_boxes = 1;
        if (P.a_mn) a_boxes = min(2, (P.M - m0 + 63) / 64);
        if (P.b_mn) b_boxes = min(4, (P.N - n0 + 63) / 64);
        const uint32_t bytes = (P.a_mn ? a_boxes * 8192 : TC_A_BYTES) + (P.b_mn ? b_boxes * 8192 : TC_B_BYTES);
        for (int kb = T.kb0; kb < T.kb1; ++kb, ++kit) {
          const int stage = kit % TC_STAGES;
          const uint32_t phase = (kit / TC_STAGES) & 1;
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.err)) { ok = false; break; }
          uint8_t* sA = smem + stage * TC_STAGE_BYTES;
          uint8_t* sB = sA + TC_A_BYTES;
          mbar_arrive_expect_tx(&full_bar[stage], bytes);
          const int k0 = kb * TC_BK;
          if (!P.a_mn) {
            tma_load_2d(sA, tA, &full_bar[stage], k0, m0);
          } else {
            for (int j = 0; j < a_boxes; ++j) tma_load_2d(sA + j * 8192, tA, &full_bar[stage], m0 + 64 * j, k0);
          }
          if (!P.b_mn) {
            tma_load_2d(sB, tB, &full_bar[stage], k0, n0);
          } else {
            for (int j = 0; j < b_boxes; ++j) tma_load_2d(sB + j * 8192, tB, &full_bar[stage], n0 + 64 * j, k0);
          }
        }
      }
      if (!ok) {
        // drain: the last load issued into each stage must land before the CTA exits
        volatile int no_abort = 0;
        for (uint32_t j = kit > TC_STAGES ? kit - TC_STAGES : 0; j < kit; ++j)
          mbar_wait(&full_bar[j % TC_STAGES], (j / TC_STAGES) & 1, &no_abort, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t kit = 0;
      bool ok = true;
      for (int i = 0; i < ntiles && ok; ++i) {
        const Tile T = sched_tile(p, sched, cta, G, i);
        const TcProblem& P = p.prob[T.prob];
        const int acc = i & 1;
        const uint32_t aph = (i >> 1) & 1;
        if (!mbar_wait(&tempty_bar[acc], aph ^ 1, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * TC_BN;
        const uint32_t idesc = idesc_bf16_f32(P.a_mn, P.b_mn, TC_BM, TC_BN);
        for (int kb = T.kb0; kb < T.kb1; ++kb, ++kit) {
          const int stage = kit % TC_STAGES;
          const uint32_t phase = (kit / TC_STAGES) & 1;
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + stage * TC_STAGE_BYTES);
          const uint32_t b_base = a_base + TC_A_BYTES;
#pragma unroll
          for (int k = 0; k < TC_BK / 16; ++k) {
            const uint64_t ad = P.a_mn ? smem_desc_sw128(a_base + k * 2048, 8192, 1024)
                                       : smem_desc_sw128(a_base + k * 32, 16, 1024);
            const uint64_t bd = P.b_mn ? smem_desc_sw128(b_base + k * 2048, 8192, 1024)
                                       : smem_desc_sw128(b_base + k * 32, 16, 1024);
            tc_mma_bf16(d_tmem, ad, bd, idesc, (kb != T.kb0) || (k != 0));
          }
          tc_commit(&empty_bar[stage]);
        }
        if (ok) tc_commit(&tfull_bar[acc]);
      }
      // every MMA this thread issued must be finished before TMEM is freed
      if (kit > 0) {
        tc_commit(mma_done_bar);
        volatile int no_abort = 0;
        mbar_wait(mma_done_bar, 0, &no_abort, p.err);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue
    const int q = warp & 3;  // tensor-memory lane quarter this warp may access
    const int row = q * 32 + lane;
    for (int i = 0; i < ntiles; ++i) {
      const Tile T = sched_tile(p, sched, cta, G, i);
      const TcProblem& P = p.prob[T.prob];
      const int tm = T.tm, tn = T.tn;
      const int acc = i & 1;
      const uint32_t aph = (i >> 1) & 1;
      const bool ok = mbar_wait(&tfull_bar[acc], aph, abort_flag, p.err);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * TC_BN;
      const ReleaseLocal rel{&tempty_bar[acc]};
      if (P.epi == EPI_LOGITS)
        epi_logits(p, P, (int64_t)tm * TC_BM, tn, row, taddr, rel);
      else
        epi_store(P, (int64_t)tm * TC_BM, tn, T.split, row, taddr, rel);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TC_TMEM_COLS);
  }
}

}  // namespace flce
