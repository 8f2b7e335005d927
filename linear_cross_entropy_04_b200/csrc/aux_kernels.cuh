// Memory-bound steps of fused linear cross-entropy and the exact-fp32 SIMT path.
//
//   count_valid_kernel   N = #rows whose target is not ignore_index (A0)
//   combine_kernel       per row: merge the per-tile (max, sum-exp) partials
//                        into lse, write l_i = lse - z_t, and turn each tile's
//                        max into the factor exp(m_tile - lse) * scale (A3)
//   dlogits_kernel       in place over the chunk store: e * factor - onehot*scale,
//                        0 for ignored rows (A4, "in-place gradient replacement"
//                        of the paper review's 主な発見)
//   factor_kernel        combine's factor step alone, for gradients taken from
//                        a kept forward pass (FLCE_FLAG_FROM_KEPT)
//   finalize_loss_kernel fixed-order sum of the per-row losses, times 1/N or 1
//   scale_grad_kernel    gradients from the forward pass times the upstream
//                        gradient (a device scalar), in place; no memory
//                        traffic when that scalar is 1
//   ce_row_cluster_kernel logits given, bf16: one cluster of CTAs per row, z
//                        read once and dz written once
//   ce_partials_kernel   logits given (f32, or rows too long for a cluster):
//                        per-(row, tile) partials read from z
//   ce_grad_kernel       logits given: dz from z and lse, optionally in place
//   simt_gemm_kernel     fp32 FMA GEMM with the same epilogues as the tcgen05
//                        engine, for fp32 inputs where TF32 tensor cores would
//                        not meet an exact-fp32 tolerance
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace flce {

__device__ __forceinline__ bool target_valid(int64_t t, int64_t V, int64_t ignore_index) {
  return t != ignore_index && t >= 0 && t < V;
}

// 1/N for the mean reduction, 1 for sum and none.
__device__ __forceinline__ float mean_scale(const int64_t* n_valid, int reduction) {
  if (reduction != 0) return 1.f;
  const int64_t n = *n_valid;
  return n > 0 ? 1.f / (float)n : 0.f;
}

// ------------------------------------------------------------------ A0
// One block; integer counts, so the order of the reduction does not matter.
__global__ void count_valid_kernel(const int64_t* __restrict__ target, int64_t BT, int64_t V,
                                   int64_t ignore_index, int64_t* n_valid, uint32_t* err) {
  __shared__ unsigned long long part[32];
  unsigned long long c = 0;
  bool bad = false;
  for (int64_t i = threadIdx.x; i < BT; i += blockDim.x) {
    const int64_t t = target[i];
    if (t == ignore_index) continue;
    if (t >= 0 && t < V) ++c; else bad = true;
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(err, DEVERR_TARGET_RANGE);
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x < 32) {
    c = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0ull;
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (threadIdx.x == 0) *n_valid = (int64_t)c;
  }
}

// ------------------------------------------------------------------ A3
// Block = CB_THREADS threads = CB_WARPS warps over 32 rows: lane <-> row, warp
// w merges tiles w, w + CB_WARPS, ... so every partial load is a coalesced
// 128-byte read, and 32 warps per 32 rows keep enough loads in flight for a
// long row of tiles (a grid of only rows / 32 blocks).
constexpr int CB_WARPS = 32;
constexpr int CB_THREADS = CB_WARPS * 32;
struct CombineArgs {
  const int64_t* target;  // chunk row 0
  int64_t ignore_index, V;
  int rows;               // rows in this chunk
  int ntile;              // partial tiles per row
  int64_t ldp;
  float* part_m;          // in: tile max; out: exp(m_tile - lse) * scale (0 for ignored rows)
  const float* part_s;
  const float* zt;
  float* row_loss;        // [rows] at chunk row 0: l_i (0 for ignored rows)
  float* lse_out;         // optional [rows] at chunk row 0
  const int64_t* n_valid;
  int reduction;
  const float* row_grad;  // optional [rows] at chunk row 0: upstream gradient per row
  int skip_factors;       // 1: leave the tile maxima in part_m (factor_kernel turns them later)
};

__global__ void __launch_bounds__(CB_THREADS) combine_kernel(CombineArgs a) {
  __shared__ float sm_m[CB_WARPS][32], sm_s[CB_WARPS][32], sm_lse[32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int r = blockIdx.x * 32 + lane;
  const bool row_ok = r < a.rows;
  float M = -INFINITY, S = 0.f;
  if (row_ok) {
    for (int j = w; j < a.ntile; j += CB_WARPS) {
      const float m = a.part_m[(int64_t)j * a.ldp + r];
      const float s = a.part_s[(int64_t)j * a.ldp + r];
      if (m > M) {
        S = S * exp2f((M - m) * LOG2E_F) + s;
        M = m;
      } else {
        S += s * exp2f((m - M) * LOG2E_F);
      }
    }
  }
  sm_m[w][lane] = M;
  sm_s[w][lane] = S;
  __syncthreads();
  if (w == 0) {
    float Mt = -INFINITY;
    for (int k = 0; k < CB_WARPS; ++k) Mt = fmaxf(Mt, sm_m[k][lane]);
    float St = 0.f;
    for (int k = 0; k < CB_WARPS; ++k)
      if (sm_m[k][lane] != -INFINITY) St += sm_s[k][lane] * exp2f((sm_m[k][lane] - Mt) * LOG2E_F);
    const float lse = Mt + logf(St);
    sm_lse[lane] = lse;
    if (row_ok) {
      const int64_t t = a.target[r];
      const bool valid = target_valid(t, a.V, a.ignore_index);
      a.row_loss[r] = valid ? lse - a.zt[r] : 0.f;
      if (a.lse_out) a.lse_out[r] = lse;
    }
  }
  __syncthreads();
  if (row_ok && !a.skip_factors) {
    const bool valid = target_valid(a.target[r], a.V, a.ignore_index);
    const float scale = mean_scale(a.n_valid, a.reduction) * (a.row_grad ? a.row_grad[r] : 1.f);
    const float lse = sm_lse[lane];
    for (int j = w; j < a.ntile; j += CB_WARPS) {
      float* pm = a.part_m + (int64_t)j * a.ldp + r;
      *pm = valid ? exp2f((*pm - lse) * LOG2E_F) * scale : 0.f;
    }
  }
}

// The factor step of combine_kernel on its own, for gradients taken from a
// kept forward pass: part_m holds the tile maxima, lse the row lse.
struct FactorArgs {
  const int64_t* target;  // chunk row 0
  int64_t ignore_index, V;
  int rows, ntile;
  int64_t ldp;
  float* part_m;          // in: tile max; out: exp(m_tile - lse) * scale (0 for ignored rows)
  const float* lse;       // [rows]
  const int64_t* n_valid;
  int reduction;
  const float* row_grad;  // optional [rows]
};

__global__ void __launch_bounds__(CB_THREADS) factor_kernel(FactorArgs a) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int r = blockIdx.x * 32 + lane;
  if (r >= a.rows) return;
  const bool valid = target_valid(a.target[r], a.V, a.ignore_index);
  const float scale = mean_scale(a.n_valid, a.reduction) * (a.row_grad ? a.row_grad[r] : 1.f);
  const float lse = a.lse[r];
  for (int j = w; j < a.ntile; j += CB_WARPS) {
    float* pm = a.part_m + (int64_t)j * a.ldp + r;
    *pm = valid ? exp2f((*pm - lse) * LOG2E_F) * scale : 0.f;
  }
}

// ------------------------------------------------------------------ A4
// grid.y = chunk row, grid.x * blockDim.x covers the row in vectors of 8.
template <typename T>
struct Vec8;
template <>
struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&f)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 x = unpack_bf16x2(w[k]);
      f[2 * k] = x.x;
      f[2 * k + 1] = x.y;
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&f)[8]) {
    *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                              pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
  }
  static __device__ __forceinline__ float ld1(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void st1(__nv_bfloat16* p, float f) { *p = __float2bfloat16_rn(f); }
};
template <>
struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&f)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&f)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
  static __device__ __forceinline__ float ld1(const float* p) { return *p; }
  static __device__ __forceinline__ void st1(float* p, float f) { *p = f; }
};

template <typename T>
struct DlogitsArgs {
  T* e;                   // [rows, lde] in: exp(z - m_tile); out: dz
  int64_t lde;
  const T* src;           // where e is read from (== e for in place)
  int64_t lds;
  const int64_t* target;  // chunk row 0
  int64_t ignore_index, V;
  const float* factor;    // [ntile, ldp]
  int64_t ldp;
  int tile_shift;         // log2 of the partial tile width
  const int64_t* n_valid;
  int reduction;
  const float* row_grad;  // optional [rows] at chunk row 0
};

// Each thread owns DL_VECS groups of 8 columns, 2048 columns apart, and issues
// all their loads before any store; an ignored row is written as zeros without
// being read.
constexpr int DL_VECS = 4;
constexpr int DL_COLS = 256 * 8 * DL_VECS;  // columns per block
template <typename T>
__global__ void __launch_bounds__(256) dlogits_kernel(DlogitsArgs<T> a) {
  const int64_t r = blockIdx.y;
  const int64_t cb = (int64_t)blockIdx.x * DL_COLS + threadIdx.x * 8;
  const int64_t t = a.target[r];
  const bool valid = target_valid(t, a.V, a.ignore_index);
  T* d = a.e + r * a.lde;
  if (!valid) {
    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < DL_VECS; ++u) {
      const int64_t c0 = cb + u * 2048;
      if (c0 + 8 <= a.V) Vec8<T>::store(d + c0, z);
      else for (int k = 0; c0 + k < a.V && k < 8; ++k) Vec8<T>::st1(d + c0 + k, 0.f);
    }
    return;
  }
  const float scale = mean_scale(a.n_valid, a.reduction) * (a.row_grad ? a.row_grad[r] : 1.f);
  const T* s = a.src + r * a.lds;
  float v[DL_VECS][8];
#pragma unroll
  for (int u = 0; u < DL_VECS; ++u) {
    const int64_t c0 = cb + u * 2048;
    if (c0 + 8 <= a.V) {
      Vec8<T>::load(s + c0, v[u]);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[u][k] = c0 + k < a.V ? Vec8<T>::ld1(s + c0 + k) : 0.f;
    }
  }
#pragma unroll
  for (int u = 0; u < DL_VECS; ++u) {
    const int64_t c0 = cb + u * 2048;
    if (c0 >= a.V) break;
    const float f = a.factor[(c0 >> a.tile_shift) * a.ldp + r];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float x = v[u][k] * f;
      if (c0 + k == t) x -= scale;
      v[u][k] = x;
    }
    if (c0 + 8 <= a.V) Vec8<T>::store(d + c0, v[u]);
    else for (int k = 0; k < 8 && c0 + k < a.V; ++k) Vec8<T>::st1(d + c0 + k, v[u][k]);
  }
}

// Logits-given cross-entropy, pass 1: the per-(row, tile) (max, sum-exp)
// partials and the target logit, one warp per (row, tile of 1 << tile_shift).
template <typename T>
struct CePartialArgs {
  const T* z;
  int64_t ldz;
  const int64_t* target;
  int64_t ignore_index, V;
  float* part_m;
  float* part_s;
  int64_t ldp;
  float* zt;
  int rows, ntile, tile_shift;
};

template <typename T>
__global__ void __launch_bounds__(256) ce_partials_kernel(CePartialArgs<T> a) {
  // One warp per (row, tile of 1024 columns): each lane holds 32 values in
  // registers, read once as four 16-byte vectors when the tile is whole and
  // aligned (bf16), so the tile's max and sum-exp cost one pass over memory.
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t r = warp_global / a.ntile;
  const int j = (int)(warp_global % a.ntile);
  if (r >= a.rows) return;
  const int64_t n0 = (int64_t)j << a.tile_shift;
  const int64_t n1 = (n0 + (1 << a.tile_shift)) < a.V ? (n0 + (1 << a.tile_shift)) : a.V;
  const T* zr = a.z + r * a.ldz;
  float m = -INFINITY, s = 0.f;
  const bool vec = sizeof(T) == 2 && a.tile_shift == 10 && n1 - n0 == 1024;
  if (vec) {
    float x[32];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float f8[8];
      Vec8<T>::load(zr + n0 + (q * 32 + lane) * 8, f8);
#pragma unroll
      for (int k = 0; k < 8; ++k) x[q * 8 + k] = f8[k];
    }
#pragma unroll
    for (int k = 0; k < 32; ++k) m = fmaxf(m, x[k]);
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float ms = m * LOG2E_F;
#pragma unroll
    for (int k = 0; k < 32; ++k) s += exp2f(fmaf(x[k], LOG2E_F, -ms));
  } else {
    for (int64_t c = n0 + lane; c < n1; c += 32) m = fmaxf(m, Vec8<T>::ld1(zr + c));
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float ms = m * LOG2E_F;
    for (int64_t c = n0 + lane; c < n1; c += 32) s += exp2f(fmaf(Vec8<T>::ld1(zr + c), LOG2E_F, -ms));
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    a.part_m[(int64_t)j * a.ldp + r] = m;
    a.part_s[(int64_t)j * a.ldp + r] = s;
    const int64_t t = a.target[r];
    if (t != a.ignore_index && t >= n0 && t < n1) a.zt[r] = Vec8<T>::ld1(zr + t);
  }
}

// Logits-given cross-entropy, pass 2: dz = (exp(z - lse) - onehot) * scale,
// 0 for ignored rows; dst may be z itself (in-place gradient replacement).
template <typename T>
struct CeGradArgs {
  const T* z;
  int64_t ldz;
  T* dz;
  int64_t ldd;
  const int64_t* target;
  int64_t ignore_index, V;
  const float* lse;
  const int64_t* n_valid;
  int reduction;
  const float* row_grad;  // optional [rows] at row 0
};

// Each thread handles CEG_VECS 8-element vectors of one row, CEG_SPAN columns
// apart, issuing all loads before any store (two 16-byte loads in flight per
// thread keep this pass at copy bandwidth; one per thread is issue-bound).
constexpr int CEG_VECS = 2;
constexpr int CEG_SPAN = 256 * 8;
constexpr int CEG_BLOCK_COLS = CEG_SPAN * CEG_VECS;

template <typename T>
__global__ void __launch_bounds__(256) ce_grad_kernel(CeGradArgs<T> a) {
  const int64_t r = blockIdx.y;
  const int64_t cb = (int64_t)blockIdx.x * CEG_BLOCK_COLS + threadIdx.x * 8;
  const int64_t t = a.target[r];
  const bool valid = target_valid(t, a.V, a.ignore_index);
  const float scale = mean_scale(a.n_valid, a.reduction) * (a.row_grad ? a.row_grad[r] : 1.f);
  const float ls = a.lse[r] * LOG2E_F;
  const T* s = a.z + r * a.ldz;
  T* d = a.dz + r * a.ldd;
  float v[CEG_VECS][8];
#pragma unroll
  for (int i = 0; i < CEG_VECS; ++i) {
    const int64_t c0 = cb + i * CEG_SPAN;
    if (c0 >= a.V) continue;
    if (c0 + 8 <= a.V) {
      Vec8<T>::load(s + c0, v[i]);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[i][k] = c0 + k < a.V ? Vec8<T>::ld1(s + c0 + k) : 0.f;
    }
  }
#pragma unroll
  for (int i = 0; i < CEG_VECS; ++i) {
    const int64_t c0 = cb + i * CEG_SPAN;
    if (c0 >= a.V) continue;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float x = valid ? exp2f(fmaf(v[i][k], LOG2E_F, -ls)) * scale : 0.f;
      if (valid && c0 + k == t) x -= scale;
      v[i][k] = x;
    }
    if (c0 + 8 <= a.V) {
      Vec8<T>::store(d + c0, v[i]);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (c0 + k < a.V) Vec8<T>::st1(d + c0 + k, v[i][k]);
    }
  }
}

// Logits-given cross-entropy in one read and one write of z (bf16 rows).
// A thread-block cluster of C CTAs owns one row; CTA k of the cluster holds
// columns [k * slice, (k + 1) * slice) in registers as packed bf16 pairs
// (CER_VPT vectors of 8 per thread, all loads issued before any use). Each CTA
// reduces its slice to (max, sum exp(z - max)), keeping e = exp(z - max) in
// bf16 in place of z; the C pairs are exchanged through distributed shared
// memory and one cluster barrier, after which every CTA merges them in the same
// order into the row's lse and writes dz = e * exp(max - lse) * scale straight
// from its registers (one exponential per element), and the target column as
// exp(z_t - lse) * scale - scale from z_t itself. The merge is the online-softmax combination of the
// paper review's CrossEntropy kernel with the partial tiles held on chip
// instead of written out, so z crosses HBM once in and dz once out.
// 64 registers per thread let 4 CTAs share an SM; exponentials use the PTX
// ex2.approx.ftz instruction (results below 2^-126 flush to 0).
constexpr int CER_THREADS = 256;
#ifndef FLCE_CER_VPT
#define FLCE_CER_VPT 8
#endif
constexpr int CER_VPT = FLCE_CER_VPT;                   // 8-element vectors per thread
constexpr int CER_SLICE = CER_THREADS * CER_VPT * 8;    // max columns per CTA
constexpr int CER_MAX_CLUSTER = 16;
#ifndef FLCE_CER_MIN_BLOCKS
#define FLCE_CER_MIN_BLOCKS 4  // CTAs per SM the register budget is sized for
#endif

struct CeRowArgs {
  const __nv_bfloat16* z;
  int64_t ldz;
  __nv_bfloat16* dz;      // may be z (in place); null: loss only
  int64_t ldd;
  const int64_t* target;  // row 0 of this launch
  int64_t ignore_index, V;
  float* row_loss;        // [rows] at row 0: l_i, 0 for ignored rows
  float* lse_out;         // optional [rows] at row 0
  const int64_t* n_valid;
  int reduction;
  const float* row_grad;  // optional [rows] at row 0
  int slice;              // columns per CTA: a multiple of 8, at most CER_SLICE
};

__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

// Store two floats to a shared::cluster address (own or peer CTA).
__device__ __forceinline__ void st_cluster_f32x2(uint32_t cluster_addr, float a, float b) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(cluster_addr), "f"(a), "f"(b) : "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ float block_reduce_256(float v, bool is_max, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int o = 16; o > 0; o >>= 1) {
    const float u = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, u) : v + u;
  }
  __syncthreads();  // red[] is free (a previous reduction has been read)
  if (lane == 0) red[w] = v;
  __syncthreads();
  v = red[0];
#pragma unroll
  for (int k = 1; k < CER_THREADS / 32; ++k) v = is_max ? fmaxf(v, red[k]) : v + red[k];
  return v;
}

__global__ void __launch_bounds__(CER_THREADS, FLCE_CER_MIN_BLOCKS) ce_row_cluster_kernel(CeRowArgs a) {
  __shared__ float red[CER_THREADS / 32];
  __shared__ float2 parts[CER_MAX_CLUSTER];
  const uint32_t rank = cluster_ctarank(), csize = cluster_nctarank();
  const int r = blockIdx.y;
  // columns fit in 32 bits (V < 2^31 is checked on the host)
  const int base = (int)rank * a.slice;
  const int end = base + a.slice < (int)a.V ? base + a.slice : (int)a.V;
  const __nv_bfloat16* zr = a.z + (int64_t)r * a.ldz;
  const uint16_t* zbits = reinterpret_cast<const uint16_t*>(zr);
  const int64_t t64 = a.target[r];
  const bool valid = target_valid(t64, a.V, a.ignore_index);
  const int t = valid ? (int)t64 : -1;
  const bool owns_t = valid && t >= base && t < end;
  if (!valid && !a.lse_out) {
    // an ignored row needs neither its logits nor a cluster exchange: loss 0,
    // dz 0 (every CTA of the cluster takes this branch, as they share the row)
    if (threadIdx.x == 0 && rank == 0) a.row_loss[r] = 0.f;
    if (a.dz) {
      __nv_bfloat16* dr = a.dz + (int64_t)r * a.ldd;
      for (int c = base + (int)threadIdx.x * 8; c < end; c += CER_THREADS * 8) {
        if (c + 8 <= end) {
          *reinterpret_cast<uint4*>(dr + c) = make_uint4(0u, 0u, 0u, 0u);
        } else {
          for (int k = c; k < end; ++k) dr[k] = __float2bfloat16_rn(0.f);
        }
      }
    }
    return;
  }
  // z_t is read before the cluster barrier, ahead of any in-place store to it
  const float zt = (threadIdx.x == 0 && owns_t) ? __bfloat162float(zr[t]) : 0.f;
  constexpr uint32_t NEG_INF_BF16 = 0xff80u;
  uint32_t w[CER_VPT][4];
#pragma unroll
  for (int i = 0; i < CER_VPT; ++i) {
    const int c = base + ((int)threadIdx.x + i * CER_THREADS) * 8;
    if (c + 8 <= end) {
      const uint4 u = *reinterpret_cast<const uint4*>(zr + c);
      w[i][0] = u.x;
      w[i][1] = u.y;
      w[i][2] = u.z;
      w[i][3] = u.w;
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t lo = c + 2 * q < end ? zbits[c + 2 * q] : NEG_INF_BF16;
        const uint32_t hi = c + 2 * q + 1 < end ? zbits[c + 2 * q + 1] : NEG_INF_BF16;
        w[i][q] = lo | (hi << 16);
      }
    }
  }
  __nv_bfloat162 m2 = __floats2bfloat162_rn(-INFINITY, -INFINITY);
#pragma unroll
  for (int i = 0; i < CER_VPT; ++i)
#pragma unroll
    for (int q = 0; q < 4; ++q) m2 = __hmax2(m2, *reinterpret_cast<const __nv_bfloat162*>(&w[i][q]));
  float m = fmaxf(__low2float(m2), __high2float(m2));
  m = block_reduce_256(m, true, red);
  const float ms = m == -INFINITY ? 0.f : m * LOG2E_F;  // an all -inf slice sums to 0
  // e = exp(z - m) is summed and kept, rounded to bf16, in place of z: the
  // gradient pass then needs one multiply per element instead of a second exp
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < CER_VPT; ++i)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float e0 = ex2_approx(fmaf(bf16_lo(w[i][q]), LOG2E_F, -ms));
      const float e1 = ex2_approx(fmaf(bf16_hi(w[i][q]), LOG2E_F, -ms));
      s += e0 + e1;
      w[i][q] = pack_bf16x2(e0, e1);
    }
  s = block_reduce_256(s, false, red);
  if (threadIdx.x == 0) {
    const uint32_t slot = smem_u32(&parts[rank]);
    for (uint32_t q = 0; q < csize; ++q) st_cluster_f32x2(mapa_shared(slot, q), m, s);
  }
  cluster_sync();  // every CTA now holds all pairs; no CTA touches a peer after this
  float M = -INFINITY;
  for (uint32_t q = 0; q < csize; ++q) M = fmaxf(M, parts[q].x);
  float S = 0.f;
  for (uint32_t q = 0; q < csize; ++q)
    if (parts[q].x != -INFINITY) S += parts[q].y * exp2f((parts[q].x - M) * LOG2E_F);
  const float lse = M + logf(S);
  if (threadIdx.x == 0) {
    if (owns_t) a.row_loss[r] = lse - zt;
    if (!valid && rank == 0) a.row_loss[r] = 0.f;
    if (a.lse_out && rank == 0) a.lse_out[r] = lse;
  }
  if (!a.dz) return;
  // 0 for ignored rows: every dz of such a row is exp(.) * 0 = 0
  const float scale = valid ? mean_scale(a.n_valid, a.reduction) * (a.row_grad ? a.row_grad[r] : 1.f) : 0.f;
  const float ls = lse * LOG2E_F;
  const float f = ex2_approx(ms - ls) * scale;  // dz = e * exp(m - lse) * scale off the target
  __nv_bfloat16* dr = a.dz + (int64_t)r * a.ldd;
#pragma unroll
  for (int i = 0; i < CER_VPT; ++i) {
    const int c = base + ((int)threadIdx.x + i * CER_THREADS) * 8;
    if (c >= end) continue;
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) o[q] = pack_bf16x2(bf16_lo(w[i][q]) * f, bf16_hi(w[i][q]) * f);
    if (c + 8 <= end) {
      *reinterpret_cast<uint4*>(dr + c) = make_uint4(o[0], o[1], o[2], o[3]);
    } else {
      uint16_t* db = reinterpret_cast<uint16_t*>(dr);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (c + 2 * q < end) db[c + 2 * q] = (uint16_t)(o[q] & 0xffffu);
        if (c + 2 * q + 1 < end) db[c + 2 * q + 1] = (uint16_t)(o[q] >> 16);
      }
    }
  }
  if (owns_t) {
    __syncthreads();  // the vector store covering column t comes first
    if (threadIdx.x == 0) dr[t] = __float2bfloat16_rn(ex2_approx(fmaf(zt, LOG2E_F, -ls)) * scale - scale);
  }
}

// ------------------------------------------------------------------ one pass, staged in shared memory
// The same one-pass cross-entropy as ce_row_cluster_kernel (a cluster of C CTAs
// per row, each reducing its slice, the C (max, sum) pairs exchanged through
// distributed shared memory), with the slice staged in shared memory instead of
// registers: one thread moves it in with a single bulk copy (cp.async.bulk,
// completing on an mbarrier) and the gradient goes back out with another,
// written in place over the staged logits. The slice (up to 32768 bf16, 64 KB;
// about 21-26K columns by the host's rule) leaves the registers free, so 4-5
// CTAs share an SM instead of 4 at most, and the copies are issued by the
// bulk-copy engine rather than 256 threads' loads.
// Columns past the last 16-byte vector of a slice (V not a multiple of 8)
// move with plain loads and stores.
__device__ __forceinline__ void bulk_load_smem(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_store_global(void* gdst, const void* smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(smem_src)),
               "r"(bytes)
               : "memory");
}

__global__ void __launch_bounds__(CER_THREADS) ce_row_smem_kernel(CeRowArgs a, uint32_t* err) {
  extern __shared__ __align__(128) uint4 zs4[];  // the slice: (slice / 8) 16-byte vectors
  __shared__ float red[CER_THREADS / 32];
  __shared__ float2 parts[CER_MAX_CLUSTER];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int no_abort;
  const uint32_t rank = cluster_ctarank(), csize = cluster_nctarank();
  const int r = blockIdx.y;
  const int base = (int)rank * a.slice;
  const int end = base + a.slice < (int)a.V ? base + a.slice : (int)a.V;
  const int n = end - base;             // columns of this CTA (>= 1)
  const int nvec = n >> 3;              // whole 16-byte vectors
  const int tail = n - (nvec << 3);     // columns after them (< 8)
  const int nv_all = nvec + (tail ? 1 : 0);
  const __nv_bfloat16* zr = a.z + (int64_t)r * a.ldz;
  const int64_t t64 = a.target[r];
  const bool valid = target_valid(t64, a.V, a.ignore_index);
  const int t = valid ? (int)t64 : -1;
  const bool owns_t = valid && t >= base && t < end;
  if (!valid && !a.lse_out) {
    // an ignored row needs neither its logits nor a cluster exchange (every CTA of
    // the cluster takes this branch: they share the row)
    if (threadIdx.x == 0 && rank == 0) a.row_loss[r] = 0.f;
    if (a.dz) {
      __nv_bfloat16* dr = a.dz + (int64_t)r * a.ldd;
      for (int c = base + (int)threadIdx.x * 8; c < end; c += CER_THREADS * 8) {
        if (c + 8 <= end) {
          *reinterpret_cast<uint4*>(dr + c) = make_uint4(0u, 0u, 0u, 0u);
        } else {
          for (int k = c; k < end; ++k) dr[k] = __float2bfloat16_rn(0.f);
        }
      }
    }
    return;
  }
  uint16_t* zs = reinterpret_cast<uint16_t*>(zs4);
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    no_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar, (uint32_t)nvec * 16u);
    if (nvec > 0) bulk_load_smem(zs4, zr + base, (uint32_t)nvec * 16u, &bar);
  }
  // the tail, padded with -inf to a whole vector
  if (tail && (int)threadIdx.x < 8) {
    const int c = nvec * 8 + (int)threadIdx.x;
    zs[c] = c < n ? reinterpret_cast<const uint16_t*>(zr)[base + c] : (uint16_t)0xff80u;
  }
  if (!mbar_wait(&bar, 0, &no_abort, err)) {
    // the copy did not land within the wait limit: the error word says so; every
    // thread still takes every barrier below, so the cluster is not held up
  }
  __syncthreads();
  const float zt = (threadIdx.x == 0 && owns_t) ? __bfloat162float(__ushort_as_bfloat16(zs[t - base])) : 0.f;
  __nv_bfloat162 m2 = __floats2bfloat162_rn(-INFINITY, -INFINITY);
  for (int v = threadIdx.x; v < nv_all; v += CER_THREADS) {
    const uint4 u = zs4[v];
    m2 = __hmax2(m2, *reinterpret_cast<const __nv_bfloat162*>(&u.x));
    m2 = __hmax2(m2, *reinterpret_cast<const __nv_bfloat162*>(&u.y));
    m2 = __hmax2(m2, *reinterpret_cast<const __nv_bfloat162*>(&u.z));
    m2 = __hmax2(m2, *reinterpret_cast<const __nv_bfloat162*>(&u.w));
  }
  float m = fmaxf(__low2float(m2), __high2float(m2));
  m = block_reduce_256(m, true, red);
  const float ms = m == -INFINITY ? 0.f : m * LOG2E_F;  // an all -inf slice sums to 0
  // e = exp(z - m) is summed and written back, rounded to bf16, over z: the
  // gradient pass then needs one multiply per element instead of a second exp
  float s = 0.f;
  for (int v = threadIdx.x; v < nv_all; v += CER_THREADS) {
    const uint4 u = zs4[v];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float e0 = ex2_approx(fmaf(bf16_lo(w[q]), LOG2E_F, -ms));
      const float e1 = ex2_approx(fmaf(bf16_hi(w[q]), LOG2E_F, -ms));
      s += e0 + e1;
      o[q] = pack_bf16x2(e0, e1);
    }
    zs4[v] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  s = block_reduce_256(s, false, red);
  if (threadIdx.x == 0) {
    const uint32_t slot = smem_u32(&parts[rank]);
    for (uint32_t q = 0; q < csize; ++q) st_cluster_f32x2(mapa_shared(slot, q), m, s);
  }
  cluster_sync();  // every CTA now holds all pairs; no CTA touches a peer after this
  float M = -INFINITY;
  for (uint32_t q = 0; q < csize; ++q) M = fmaxf(M, parts[q].x);
  float S = 0.f;
  for (uint32_t q = 0; q < csize; ++q)
    if (parts[q].x != -INFINITY) S += parts[q].y * exp2f((parts[q].x - M) * LOG2E_F);
  const float lse = M + logf(S);
  if (threadIdx.x == 0) {
    if (owns_t) a.row_loss[r] = lse - zt;
    if (!valid && rank == 0) a.row_loss[r] = 0.f;
    if (a.lse_out && rank == 0) a.lse_out[r] = lse;
  }
  if (!a.dz) return;
  // 0 for ignored rows: every dz of such a row is exp(.) * 0 = 0
  const float scale = valid ? mean_scale(a.n_valid, a.reduction) * (a.row_grad ? a.row_grad[r] : 1.f) : 0.f;
  const float ls = lse * LOG2E_F;
  const float f = ex2_approx(ms - ls) * scale;  // dz = e * exp(m - lse) * scale off the target
  for (int v = threadIdx.x; v < nv_all; v += CER_THREADS) {
    const uint4 u = zs4[v];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) o[q] = pack_bf16x2(bf16_lo(w[q]) * f, bf16_hi(w[q]) * f);
    zs4[v] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (owns_t) {
    // the target column, from z_t itself: exp(z_t - lse) * scale - scale
    __syncthreads();  // the vector that holds it has been written
    if (threadIdx.x == 0)
      zs[t - base] = __bfloat16_as_ushort(__float2bfloat16_rn(ex2_approx(fmaf(zt, LOG2E_F, -ls)) * scale - scale));
  }
  __nv_bfloat16* dr = a.dz + (int64_t)r * a.ldd;
  fence_proxy_async_smem();  // this thread's writes, before the bulk copy reads them
  __syncthreads();
  if (tail && (int)threadIdx.x < tail) {
    const int c = nvec * 8 + (int)threadIdx.x;
    reinterpret_cast<uint16_t*>(dr)[base + c] = zs[c];
  }
  if (threadIdx.x == 0 && nvec > 0) {
    bulk_store_global(dr + base, zs4, (uint32_t)nvec * 16u);
    bulk_commit_group();
    bulk_wait_group_all();  // the shared memory it reads stays allocated until the copy is done
  }
}

// ------------------------------------------------------------------ loss
// One block, fixed order: thread k sums rows k, k+1024, ... in double, then a
// fixed shuffle tree. Deterministic for a given BT.
__global__ void __launch_bounds__(1024) finalize_loss_kernel(const float* __restrict__ row_loss,
                                                             int64_t BT, const int64_t* n_valid,
                                                             int reduction, float* loss) {
  __shared__ double part[32];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < BT; i += blockDim.x) acc += (double)row_loss[i];
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    acc = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (threadIdx.x == 0) {
      if (reduction == 0) {
        const int64_t n = *n_valid;
        *loss = n > 0 ? (float)(acc / (double)n) : 0.f;
      } else {
        *loss = (float)acc;
      }
    }
  }
}

// ------------------------------------------------------------------ upstream gradient
// p[r, c] *= *scale for a rows x cols matrix with row pitch ld (elements), in
// 16-byte vectors (VEC elements; cols, ld and p aligned to them) or, VEC = 1,
// one element at a time. The scale is read on the device, so the caller need
// not wait for it; when it is exactly 1 every block returns before touching p.
template <typename T, int VEC>
__global__ void __launch_bounds__(256) scale_grad_kernel(T* __restrict__ p, int64_t rows, int64_t cols, int64_t ld,
                                                         const float* __restrict__ scale) {
  const float f = *scale;
  if (f == 1.f) return;
  const int64_t vpr = cols / VEC;  // vectors per row
  const int64_t n = rows * vpr;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / vpr, c = (i - r * vpr) * VEC;
    T* q = p + r * ld + c;
    if constexpr (VEC == 1) {
      if constexpr (sizeof(T) == 2) *q = __float2bfloat16_rn(__bfloat162float(*q) * f);
      else *q = *q * f;
    } else if constexpr (sizeof(T) == 2) {
      uint4 v = *reinterpret_cast<const uint4*>(q);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 x = unpack_bf16x2(w[k]);
        w[k] = pack_bf16x2(x.x * f, x.y * f);
      }
      *reinterpret_cast<uint4*>(q) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
      float4 v = *reinterpret_cast<const float4*>(q);
      v.x *= f; v.y *= f; v.z *= f; v.w *= f;
      *reinterpret_cast<float4*>(q) = v;
    }
  }
}

// ------------------------------------------------------------------ split-K sum
// out[r, h] = bf16(sum over s = 0..S-1 of part[s * stride + r * H + h]), in
// that fixed order, so a split-K result does not depend on launch timing.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ part, int S,
                                                            int64_t stride, int rows, int H,
                                                            __nv_bfloat16* __restrict__ out, int64_t ldo) {
  const int64_t n4 = (int64_t)rows * H / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = i * 4;
    const int64_t r = e / H, h = e % H;
    float4 acc = reinterpret_cast<const float4*>(part + e)[0];
    for (int s = 1; s < S; ++s) {
      const float4 v = reinterpret_cast<const float4*>(part + s * stride + e)[0];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    uint2 o;
    o.x = pack_bf16x2(acc.x, acc.y);
    o.y = pack_bf16x2(acc.z, acc.w);
    *reinterpret_cast<uint2*>(out + r * ldo + h) = o;
  }
}

// ------------------------------------------------------------------ SIMT fp32
// C(m, n) = sum_k A(m, k) * B(n, k) with A(m, k) = A[m*sam + k*sak] and
// B(n, k) = B[n*sbn + k*sbk]. 64 x 64 tiles, 256 threads, 4 x 4 per thread.
constexpr int SG_BM = 64, SG_BN = 64, SG_BK = 16;

enum SimtEpi : int { SEPI_LOGITS = 0, SEPI_STORE = 1, SEPI_GRADW_STORE = 2, SEPI_GRADW_ADD = 3 };

struct SimtArgs {
  const float* A;
  int64_t sam, sak;
  const float* B;
  int64_t sbn, sbk;
  int M, N, K;
  int epi;
  float* out;
  int64_t ldo;
  // SEPI_LOGITS
  const int64_t* target;
  int64_t ignore_index;
  float* part_m;
  float* part_s;
  int64_t ldp;
  float* zt;
};

__global__ void __launch_bounds__(256) simt_gemm_kernel(SimtArgs a) {
  __shared__ float As[SG_BK][SG_BM + 4];
  __shared__ float Bs[SG_BK][SG_BN + 4];
  __shared__ float Cs[SG_BM][SG_BN + 1];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t m0 = (int64_t)blockIdx.y * SG_BM, n0 = (int64_t)blockIdx.x * SG_BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < a.K; k0 += SG_BK) {
    for (int i = tid; i < SG_BM * SG_BK; i += 256) {
      int mm, kk;
      if (a.sak == 1) { mm = i / SG_BK; kk = i % SG_BK; } else { kk = i / SG_BM; mm = i % SG_BM; }
      const int64_t gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < a.M && gk < a.K) ? a.A[gm * a.sam + gk * a.sak] : 0.f;
    }
    for (int i = tid; i < SG_BN * SG_BK; i += 256) {
      int nn, kk;
      if (a.sbk == 1) { nn = i / SG_BK; kk = i % SG_BK; } else { kk = i / SG_BN; nn = i % SG_BN; }
      const int64_t gn = n0 + nn, gk = k0 + kk;
      Bs[kk][nn] = (gn < a.N && gk < a.K) ? a.B[gn * a.sbn + gk * a.sbk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SG_BK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  if (a.epi != SEPI_LOGITS) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t gm = m0 + ty * 4 + i;
      if (gm >= a.M) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t gn = n0 + tx * 4 + j;
        if (gn >= a.N) continue;
        float* o = a.out + gm * a.ldo + gn;
        *o = a.epi == SEPI_GRADW_ADD ? *o + acc[i][j] : acc[i][j];
      }
    }
    return;
  }
  // online-softmax epilogue over this 64-column tile: one thread per row
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) Cs[ty * 4 + i][tx * 4 + j] = acc[i][j];
  __syncthreads();
  if (tid < SG_BM) {
    const int64_t r = m0 + tid;
    if (r >= a.M) return;
    const int ncols = (int)((a.N - n0) < SG_BN ? (a.N - n0) : SG_BN);
    float mx = -INFINITY;
    for (int j = 0; j < ncols; ++j) mx = fmaxf(mx, Cs[tid][j]);
    const float ms = mx * LOG2E_F;
    float s = 0.f;
    float* er = a.out + r * a.ldo + n0;
    for (int j = 0; j < ncols; ++j) {
      const float e = exp2f(fmaf(Cs[tid][j], LOG2E_F, -ms));
      s += e;
      er[j] = e;
    }
    const int64_t tile = blockIdx.x;
    a.part_m[tile * a.ldp + r] = mx;
    a.part_s[tile * a.ldp + r] = s;
    const int64_t t = a.target[r];
    if (t != a.ignore_index && t >= n0 && t < n0 + ncols) a.zt[r] = Cs[tid][t - n0];
  }
}

}  // namespace flce
