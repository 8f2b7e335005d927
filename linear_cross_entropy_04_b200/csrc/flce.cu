// Host side of the fused linear cross-entropy library: argument checks, the
// bounded-workspace chunk plan, TMA descriptors, and the launch sequence.
//
// Per chunk of rows (the "chunking" of "Liger Kernel: Efficient Triton Kernels
// for LLM Training", paper review, 提案手法; and of "Liger-Kernel 項目詳細介紹",
// 技術原理 > 分塊計算):
//   A1+A2  logits GEMM z = X_c W^T with the online-softmax epilogue
//   A3     row combine: lse, per-row loss, per-tile factors
//   A4     in-place dlogits over the chunk store (技術原理 > 原地操作)
//   A5+A6  grad_X_c = dz W and grad_W (+)= dz^T X_c, in one persistent launch
//          or two (grad_combined)
// then one fixed-order loss reduction. The full BT x V logits never exist:
// the store holds one chunk of rows at a time (except on request: the
// two-phase flags keep the whole batch as one chunk between two calls).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/flce.h"
#include "aux_kernels.cuh"
#include "tc_gemm.cuh"
#include "tc_gemm2.cuh"

namespace flce {

__device__ uint32_t g_err_word;  // device error word (FLCE_DEVERR_* bits), one per device
// checkpoint counters of the wide grad_X tiles' soft K-synchronisation (zeroed
// before each launch that uses them; launches that overlap on the GPU only
// disturb each other's pacing, not their results)
__device__ uint32_t g_ksync_ctr[KSYNC_MAX_CKPT];

namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kDefaultLimit = 512ll << 20;
constexpr int64_t kMaxChunk = 32768;
constexpr int64_t kMinDefaultChunk = 2048;
constexpr int64_t kRecomputeRowBlock = 4096;
constexpr int kCeSliceMax = 32768;  // largest slice of the shared-memory one-pass CE kernel (64 KB staged)  // rows per logits launch in the recompute schedule's first pass

struct DeviceCtx {
  bool init = false;
  bool supported = false;
  int sms = 0;
  int pairs = 0;  // CTA pairs of the cluster engine that fit on the device at once
  int ce_max_cluster = 0;  // largest cluster the one-pass cross-entropy kernel can launch with
  uint32_t* err = nullptr;
  uint32_t* ksync = nullptr;     // device address of g_ksync_ctr
  cudaMemPool_t pool = nullptr;  // library-owned stream-ordered pool for workspaces
};

std::mutex g_mu;
DeviceCtx g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

struct PhaseRec {
  int phase;
  cudaEvent_t a, b;
};
std::vector<PhaseRec> g_phase_recs;
std::vector<cudaEvent_t> g_event_pool;

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

flce_status device_ctx(DeviceCtx** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLCE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FLCE_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceCtx& c = g_dev[dev];
  if (!c.init) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return FLCE_ERR_CUDA;
    c.supported = prop.major == 10 && prop.minor == 0;
    c.sms = prop.multiProcessorCount;
    if (c.supported) {
      if (cudaGetSymbolAddress(reinterpret_cast<void**>(&c.err), g_err_word) != cudaSuccess ||
          cudaGetSymbolAddress(reinterpret_cast<void**>(&c.ksync), g_ksync_ctr) != cudaSuccess)
        return FLCE_ERR_CUDA;
      if (cudaFuncSetAttribute(tc_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               TC_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(tc_gemm_pair_kernel<NoShards>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               T2_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(tc_gemm_pair_kernel<ShardMaps>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               T2_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(tc_gemm_pair_kernel<NoShards, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               T2W_SMEM_BYTES) != cudaSuccess)
        return FLCE_ERR_CUDA;
      {
        cudaLaunchConfig_t cfg;
        std::memset(&cfg, 0, sizeof(cfg));
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (c.sms / 2));
        cfg.blockDim = dim3(TC_THREADS);
        cfg.dynamicSmemBytes = T2_SMEM_BYTES;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int nc = 0;
        if (cudaOccupancyMaxActiveClusters(&nc, tc_gemm_pair_kernel<NoShards>, &cfg) != cudaSuccess || nc <= 0) {
          cudaGetLastError();
          nc = c.sms / 2;
        }
        c.pairs = std::min(nc, c.sms / 2);
      }
      // The one-pass cross-entropy kernel runs clusters of up to 16 CTAs (a
      // non-portable size) when the device can hold one, else up to 8.
      c.ce_max_cluster = 8;
      if (cudaFuncSetAttribute(ce_row_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kCeSliceMax * 2) !=
          cudaSuccess)
        return FLCE_ERR_CUDA;
      if (cudaFuncSetAttribute(ce_row_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
              cudaSuccess &&
          cudaFuncSetAttribute(ce_row_smem_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
              cudaSuccess) {
        cudaLaunchConfig_t cfg;
        std::memset(&cfg, 0, sizeof(cfg));
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = CER_MAX_CLUSTER;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.gridDim = dim3(CER_MAX_CLUSTER, 1, 1);
        cfg.blockDim = dim3(CER_THREADS);
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int nc = 0, nc2 = 0;
        if (cudaOccupancyMaxActiveClusters(&nc, ce_row_cluster_kernel, &cfg) == cudaSuccess && nc > 0) {
          cfg.dynamicSmemBytes = kCeSliceMax * 2;  // the largest slice the shared-memory kernel stages
          if (cudaOccupancyMaxActiveClusters(&nc2, ce_row_smem_kernel, &cfg) == cudaSuccess && nc2 > 0)
            c.ce_max_cluster = CER_MAX_CLUSTER;
        }
      }
      cudaGetLastError();
      // Load the upstream-gradient kernels now: under lazy module loading a
      // kernel's first launch can block the host, and these run inside autograd's
      // backward, which must not wait for the GPU.
      {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, scale_grad_kernel<__nv_bfloat16, 8>) != cudaSuccess ||
            cudaFuncGetAttributes(&fa, scale_grad_kernel<__nv_bfloat16, 1>) != cudaSuccess ||
            cudaFuncGetAttributes(&fa, scale_grad_kernel<float, 4>) != cudaSuccess ||
            cudaFuncGetAttributes(&fa, scale_grad_kernel<float, 1>) != cudaSuccess)
          return FLCE_ERR_CUDA;
      }
      // A private pool that keeps freed workspace mapped, so repeated calls
      // reuse it stream-ordered instead of mapping and unmapping memory.
      cudaMemPoolProps pp;
      std::memset(&pp, 0, sizeof(pp));
      pp.allocType = cudaMemAllocationTypePinned;
      pp.handleTypes = cudaMemHandleTypeNone;
      pp.location.type = cudaMemLocationTypeDevice;
      pp.location.id = dev;
      if (cudaMemPoolCreate(&c.pool, &pp) != cudaSuccess) return FLCE_ERR_CUDA;
      uint64_t keep = ~0ull;
      if (cudaMemPoolSetAttribute(c.pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess)
        return FLCE_ERR_CUDA;
      if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
          return FLCE_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
      }
    }
    c.init = true;
  }
  if (!c.supported) return FLCE_ERR_UNSUPPORTED_DEVICE;
  *out = &c;
  return FLCE_OK;
}

// bf16 2-D tensor map: dims {inner, outer}, row pitch in bytes, box {bi, bo}, 128B swizzle.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
               uint64_t pitch_bytes, uint32_t bi, uint32_t bo,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {bi, bo};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int dtype_size(int32_t dt) { return dt == FLCE_F32 ? 4 : dt == FLCE_BF16 ? 2 : dt == FLCE_I64 ? 8 : 0; }

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// A row-major matrix of the given shape and dtype.
bool check_matrix(const flce_tensor* t, int32_t dtype, int64_t rows, int64_t cols) {
  if (!t || !t->data || t->dtype != dtype || t->ndim != 2) return false;
  if (t->shape[0] != rows || t->shape[1] != cols) return false;
  if (t->stride[1] != 1 || t->stride[0] < cols) return false;
  return true;
}

// Split-K factor for a problem of `tiles` output tiles and `kblocks` K-blocks
// on `units` concurrent workers (CTA pairs): the smallest S that minimises the
// number of tile-waves per unit of work, ceil(tiles * S / units) / S, keeping
// at least 32 K-blocks per split. S = 1 when splitting does not help.
int choose_ksplit(int64_t tiles, int64_t kblocks, int64_t units) {
  int best_s = 1;
  double best = (double)ceil_div(tiles, units);
  for (int S = 2; S <= 8 && kblocks / S >= 32; ++S) {
    const double w = (double)ceil_div(tiles * S, units) / S;
    if (w < best - 1e-9) {
      best = w;
      best_s = S;
    }
  }
  // every split must own at least one K-block
  const int64_t kps = ceil_div(kblocks, best_s);
  return (int)ceil_div(kblocks, kps);
}

// grad_X split-K partial buffer (fp32 elements) the plan reserves: the largest
// S * rows * H over the full and the last chunk, for the CTA-pair engine on a
// B200 (74 pairs). A device with fewer pairs gets S clamped to fit.
// Split-K for grad_X is opt-in (FLCE_GRADX_SPLITK=1): under the B200's power
// cap the step is power-bound, so filling idle SMs did not shorten it, and
// the partial buffer costs S * chunk_rows * H * 4 bytes of workspace.
bool gradx_splitk_enabled() {
  const char* s = std::getenv("FLCE_GRADX_SPLITK");
  return s && s[0] == '1';
}

int64_t gradx_partial_elems(int64_t BT, int64_t H, int64_t V, int64_t chunk) {
  if (BT <= 0 || !gradx_splitk_enabled()) return 0;
  const int64_t last = BT - (ceil_div(BT, chunk) - 1) * chunk;
  int64_t best = 0;
  for (int64_t rows : {std::min(chunk, BT), last}) {
    const int64_t tiles = ceil_div(rows, 256) * ceil_div(H, 256);
    const int S = choose_ksplit(tiles, ceil_div(V, 64), 74);
    if (S > 1) best = std::max(best, S * rows * H);
  }
  return best;
}

// FLCE_CHUNK_ROWS=<n> sets the chunk rows of calls whose options leave
// chunk_rows at 0 (rounded up to a multiple of 128, like the option).
// Unset, empty, non-numeric or non-positive values leave the default plan.
int64_t env_chunk_rows() {
  const char* s = std::getenv("FLCE_CHUNK_ROWS");
  if (!s || !*s) return 0;
  char* end = nullptr;
  const long long v = std::strtoll(s, &end, 10);
  if (end == s || *end != '\0' || v <= 0) return 0;
  return round_up(std::min<int64_t>(v, kMaxChunk), 128);
}

struct Plan {
  int64_t BT, H, V;
  int32_t dtype;
  int64_t chunk, n_chunks;
  int64_t tile_w;  // partial tile width (columns)
  int64_t ntile, lde, ldp;
  size_t off_nvalid, off_rowloss, off_zt, off_pm, off_ps, off_e, off_facc, off_xpart, off_lse, off_gwl, total;
  bool keep;  // FLCE_FLAG_KEEP_LOGITS / FLCE_FLAG_FROM_KEPT: one chunk, lse kept in the workspace
  bool facc;
  bool gw_local;  // grad_W shards: chunks before the last accumulate into a local bf16 [V, H]
  // recompute schedule (FLCE_FLAG_RECOMPUTE): chunk = vocabulary columns per chunk, n_chunks =
  // vocabulary chunks, the store is [BT, chunk]; the first pass takes rows in blocks of r1
  bool recompute;
  int64_t r1;
  int64_t xpart_elems;  // grad_X split-K partials (fp32 elements)
};

flce_status make_plan(int64_t BT, int64_t H, int64_t V, int32_t dtype, bool want_gw,
                      const flce_options* opt, bool need_rowloss, Plan* p) {
  if (BT < 0 || H <= 0 || V <= 0) return FLCE_ERR_INVALID_ARG;
  if (dtype != FLCE_BF16 && dtype != FLCE_F32) return FLCE_ERR_UNSUPPORTED_DTYPE;
  p->BT = BT;
  p->H = H;
  p->V = V;
  p->dtype = dtype;
  const int64_t esz = dtype == FLCE_BF16 ? 2 : 4;
  p->tile_w = dtype == FLCE_BF16 ? TC_BN : SG_BN;
  p->ntile = ceil_div(V, p->tile_w);
  p->lde = round_up(V, 64);
  const int64_t per_row = p->lde * esz + p->ntile * 8 + 4;
  int64_t chunk = opt && opt->chunk_rows > 0 ? round_up(opt->chunk_rows, 128) : env_chunk_rows();
  const int64_t bt_r = std::max<int64_t>(round_up(std::max<int64_t>(BT, 1), 128), 128);
  p->keep = opt && (opt->flags & (FLCE_FLAG_KEEP_LOGITS | FLCE_FLAG_FROM_KEPT));
  p->recompute = opt && (opt->flags & FLCE_FLAG_RECOMPUTE);
  p->gw_local = false;
  p->r1 = 0;
  if (p->recompute) {
    if (dtype != FLCE_BF16) return FLCE_ERR_UNSUPPORTED_DTYPE;
    if (p->keep || (opt->n_shards > 0)) return FLCE_ERR_INVALID_ARG;
    // vocabulary columns per chunk: the option, else the store budget over all rows
    int64_t vc = opt->chunk_rows > 0 ? round_up(opt->chunk_rows, 256) : 0;
    if (vc == 0) {
      const int64_t limit = opt->workspace_limit_bytes > 0 ? opt->workspace_limit_bytes : kDefaultLimit;
      vc = (limit / (bt_r * 2)) / 256 * 256;
    }
    vc = std::max<int64_t>(256, std::min<int64_t>(vc, round_up(V, 256)));
    p->chunk = vc;
    p->n_chunks = BT > 0 ? ceil_div(V, vc) : 0;
    p->lde = vc;
    p->r1 = std::min<int64_t>(bt_r, kRecomputeRowBlock);
    p->ldp = round_up(p->r1, 32);
    p->facc = false;
    p->xpart_elems = 0;
    size_t o = 0;
    p->off_nvalid = o; o = align256(o + 8);
    p->off_rowloss = o; o = align256(o + (need_rowloss ? (size_t)std::max<int64_t>(BT, 1) * 4 : 0));
    p->off_zt = o; o = align256(o + (size_t)p->r1 * 4);
    p->off_pm = o; o = align256(o + (size_t)p->ntile * p->ldp * 4);
    p->off_ps = o; o = align256(o + (size_t)p->ntile * p->ldp * 4);
    p->off_e = o; o = align256(o + (size_t)std::max<int64_t>(BT, 1) * vc * 2);
    p->off_lse = o; o = align256(o + (size_t)std::max<int64_t>(BT, 1) * 4);
    p->off_facc = p->off_xpart = p->off_gwl = o;
    p->total = o;
    return FLCE_OK;
  }
  if (p->keep) {
    // the whole batch is one chunk whose store outlives the call
    if (bt_r > kMaxChunk) return FLCE_ERR_INVALID_ARG;
    chunk = bt_r;
  }
  if (chunk == 0) {
    if (opt && opt->workspace_limit_bytes > 0) {
      chunk = (opt->workspace_limit_bytes / per_row) / 128 * 128;
    } else {
      // default: at most 512 MiB of chunk store, but at least 2048 rows (grad_W's
      // K: shorter chunks leave its tiles epilogue-bound and repeat the per-chunk
      // passes), and at most half of the rows, so the logits of the whole batch
      // are never held at once
      const int64_t half = round_up(ceil_div(std::max<int64_t>(BT, 1), 2), 128);
      chunk = std::min<int64_t>(std::max<int64_t>((kDefaultLimit / per_row) / 128 * 128, kMinDefaultChunk), half);
    }
    if (chunk < 128) chunk = 128;
    if (chunk > kMaxChunk) chunk = kMaxChunk;
    // even out the chunks: same count, rows spread as evenly as 128-row tiles allow
    if (BT > 0) chunk = round_up(ceil_div(BT, ceil_div(BT, chunk)), 128);
  }
  if (chunk > bt_r) chunk = bt_r;
  if (chunk > kMaxChunk) chunk = kMaxChunk;  // grid.y of the row kernels stays below 65536
  p->chunk = chunk;
  p->n_chunks = BT > 0 ? ceil_div(BT, chunk) : 0;
  p->ldp = round_up(chunk, 32);
  p->facc = want_gw && dtype == FLCE_BF16 && opt && opt->grad_w_accum == FLCE_GRADW_ACCUM_FP32 &&
            p->n_chunks > 1;
  size_t o = 0;
  p->off_nvalid = o; o = align256(o + 8);
  p->off_rowloss = o; o = align256(o + (need_rowloss ? (size_t)std::max<int64_t>(BT, 1) * 4 : 0));
  p->off_zt = o; o = align256(o + (size_t)chunk * 4);
  p->off_pm = o; o = align256(o + (size_t)p->ntile * p->ldp * 4);
  p->off_ps = o; o = align256(o + (size_t)p->ntile * p->ldp * 4);
  p->off_e = o; o = align256(o + (size_t)chunk * p->lde * esz);
  p->off_facc = o; o = align256(o + (p->facc ? (size_t)V * H * 4 : 0));
  p->xpart_elems = dtype == FLCE_BF16 ? gradx_partial_elems(BT, H, V, chunk) : 0;
  p->off_xpart = o; o = align256(o + (size_t)p->xpart_elems * 4);
  p->off_lse = o; o = align256(o + (p->keep ? (size_t)chunk * 4 : 0));
  p->gw_local = dtype == FLCE_BF16 && opt && opt->n_shards > 0 && !(opt->flags & FLCE_FLAG_ROUTE_EVERY_CHUNK) &&
                p->n_chunks > 1;
  p->off_gwl = o; o = align256(o + (p->gw_local ? (size_t)V * H * 2 : 0));
  p->total = o;
  return FLCE_OK;
}

cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Names of the phases of flce_phase_times, also used for the NVTX ranges.
const char* const kPhaseNames[FLCE_NUM_PHASES] = {"count_valid", "logits_gemm_softmax", "row_combine",
                                                  "dlogits_inplace", "grad_gemms", "loss_reduce"};

// NVTX range for the host-side span of a call or a phase launch (seen by
// profilers that attach an NVTX tool; otherwise each push/pop is a no-op call).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Launch bookkeeping: optional phase events, NVTX ranges, launch-error checks,
// counts. `chunk` (or -1) names the row chunk in the phase's NVTX range.
struct Launcher {
  cudaStream_t stream;
  bool timing, sync_check;
  int launches = 0;
  int64_t chunk = -1;
  template <typename F>
  flce_status run(int phase, F&& f) {
    char name[64];
    if (chunk >= 0)
      std::snprintf(name, sizeof(name), "flce %s chunk %lld", kPhaseNames[phase], (long long)chunk);
    else
      std::snprintf(name, sizeof(name), "flce %s", kPhaseNames[phase]);
    const NvtxRange range(name);
    cudaEvent_t a = nullptr, b = nullptr;
    if (timing) {
      std::lock_guard<std::mutex> lk(g_mu);
      a = pool_event();
      b = pool_event();
    }
    if (a) cudaEventRecord(a, stream);
    f();
    ++launches;
    if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;
    if (b) {
      cudaEventRecord(b, stream);
      std::lock_guard<std::mutex> lk(g_mu);
      g_phase_recs.push_back({phase, a, b});
    }
    if (sync_check) {
      if (cudaStreamSynchronize(stream) != cudaSuccess) return FLCE_ERR_CUDA;
      if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;
    }
    return FLCE_OK;
  }
};

bool env_debug() {
  const char* s = std::getenv("FLCE_DEBUG");
  return s && s[0] && s[0] != '0';
}

// Workspace holder: caller's buffer or a stream-ordered allocation.
struct Workspace {
  void* ptr = nullptr;
  bool owned = false;
  cudaStream_t stream = nullptr;
  ~Workspace() {
    if (owned && ptr) cudaFreeAsync(ptr, stream);
  }
};

flce_status get_workspace(const flce_options* opt, size_t bytes, cudaStream_t stream,
                          cudaMemPool_t pool, Workspace* ws) {
  ws->stream = stream;
  if (opt && opt->workspace) {
    if ((size_t)opt->workspace_bytes < bytes) return FLCE_ERR_WORKSPACE_TOO_SMALL;
    if (!is_aligned(opt->workspace, 256)) return FLCE_ERR_INVALID_ARG;
    ws->ptr = opt->workspace;
    return FLCE_OK;
  }
  if (cudaMallocFromPoolAsync(&ws->ptr, bytes, pool, stream) != cudaSuccess) {
    cudaGetLastError();
    ws->ptr = nullptr;
    return FLCE_ERR_ALLOC;
  }
  ws->owned = true;
  return FLCE_OK;
}

// Tensor-core engine: the CTA-pair kernel (256 x 256 tiles, default) or the
// single-CTA kernel (128 x 256 tiles), chosen with FLCE_ENGINE=2sm|1sm.
struct Engine {
  bool pair;
  int bm;         // tile rows
  int b_box_rows; // rows of B in one K-major TMA box (per CTA)
};

Engine engine() {
  const char* s = std::getenv("FLCE_ENGINE");
  if (s && std::strcmp(s, "1sm") == 0) return Engine{false, TC_BM, TC_BN};
  return Engine{true, T2_BM, T2_HALF};
}

// grad_X and grad_W of a chunk in one persistent launch ("combined") or in two
// back-to-back launches ("split"). Split avoids the two problems contending for
// L2; combined lets grad_W tiles fill the SMs that grad_X's few output tiles
// leave idle. The default picks combined when grad_X alone would keep less
// than 80% of the workers busy over its waves (measured crossover on B200);
// FLCE_GRAD_LAUNCH=split|combined forces one.
// FLCE_CE=multipass selects the partials + combine + grad kernels for bf16
// logits that the one-pass cluster kernel would otherwise take.
bool ce_one_pass_enabled() {
  const char* s = std::getenv("FLCE_CE");
  return !(s && std::strcmp(s, "multipass") == 0);
}

// FLCE_CE=regs keeps the one-pass CE slice in registers (ce_row_cluster_kernel)
// instead of staging it in shared memory (ce_row_smem_kernel, the default).
bool ce_slice_in_registers() {
  const char* s = std::getenv("FLCE_CE");
  return s && std::strcmp(s, "regs") == 0;
}

// CTAs per row (the cluster size) of the shared-memory one-pass CE kernel; each
// stages ceil(V / C) columns, rounded up to 8, in shared memory (2 bytes each, at
// most kCeSliceMax columns). What decides the speed is how many CTAs share an SM,
// which the slice's shared memory sets (5 up to about 22500 columns, 4 up to about
// 28000, 3 beyond), against how many CTAs meet at each row's exchange. Measured on
// B200 (4096 rows, one exponential per element): V = 32000: 0.107 ms with 2 CTAs;
// 50000: 0.154 with 2 (0.158 with 3); 128256: 0.374 with 6 (0.377 with 7, 0.382
// with 5); 152064: 0.447 with 7, 0.453 with 6; 256000: 0.776 with 10 of 25600
// columns, against 0.815 with 8 and 0.805 with 12. So C = ceil(V / 25600), or,
// when that is above the largest cluster the device runs (max_cluster: 16 on
// B200, else 8), ceil(V / 32768); above that the multi-pass kernels take the row.
// FLCE_CE_SLICE=<columns> (a multiple of 8 in [2048, 32768]) sets the slice
// instead: C = ceil(V / slice).
int64_t ce_smem_ctas(int64_t V, int max_cluster) {
  const char* s = std::getenv("FLCE_CE_SLICE");
  if (s && *s) {
    char* end = nullptr;
    const long v = std::strtol(s, &end, 10);
    if (end != s && *end == '\0' && v >= 2048 && v <= kCeSliceMax && v % 8 == 0) return ceil_div(V, v);
  }
  const int64_t c = ceil_div(V, 25600);
  return c <= max_cluster ? c : ceil_div(V, kCeSliceMax);
}

// Share of `units` workers kept busy over the waves of `tiles` equal tiles.
double wave_efficiency(int64_t tiles, int64_t units) {
  return (double)tiles / (double)(ceil_div(tiles, units) * units);
}

// grad_X on the pair engine's wide 256 x 512 tiles whenever that keeps at least
// as many pairs busy over its waves as 256 x 256 tiles would. It then runs as a
// launch of its own: on B200 the wide tiles on their own beat the narrow ones
// run together with grad_W (Qwen2-7B head: 43.2 against 46.1 ms per call).
// FLCE_GRADX_TILE=wide|narrow forces the choice.
bool gradx_wide(int64_t tiles_m, int64_t N, int64_t units) {
  const char* s = std::getenv("FLCE_GRADX_TILE");
  if (s && std::strcmp(s, "wide") == 0) return true;
  if (s && std::strcmp(s, "narrow") == 0) return false;
  const double en = wave_efficiency(tiles_m * ceil_div(N, 256), units);
  const double ew = wave_efficiency(tiles_m * ceil_div(N, 512), units);
  return ew >= en - 1e-9;
}

// FLCE_KSYNC=0 turns off the soft K-synchronisation of one-wave wide grad_X tiles.
bool ksync_enabled() {
  const char* s = std::getenv("FLCE_KSYNC");
  return !(s && s[0] == '0');
}

bool grad_combined(int64_t gradx_tiles, int64_t units) {
  const char* s = std::getenv("FLCE_GRAD_LAUNCH");
  if (s && std::strcmp(s, "combined") == 0) return true;
  if (s && std::strcmp(s, "split") == 0) return false;
  const double eff = (double)gradx_tiles / (double)(ceil_div(gradx_tiles, units) * units);
  return eff < 0.8;
}

TcProblem make_problem(const Engine& eg, int M, int N, int K, int a_mn, int b_mn, int epi, int m_fastest) {
  TcProblem P;
  std::memset(&P, 0, sizeof(P));
  P.M = M;
  P.N = N;
  P.K = K;
  P.tiles_m = (int)ceil_div(M, eg.bm);
  P.tiles_n = (int)ceil_div(N, TC_BN);
  P.kblocks = (int)ceil_div(K, TC_BK);
  P.a_mn = a_mn;
  P.b_mn = b_mn;
  P.epi = epi;
  P.m_fastest = m_fastest;
  P.ksplit = 1;
  P.kb_per_split = P.kblocks;
  return P;
}



// Output map for the pair engine's TMA epilogue: bf16 [rows, cols] with row
// pitch `ld` elements, written in unswizzled 32 x 32 boxes.
bool make_out_tmap(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld) {
  return make_tmap(m, base, cols, rows, ld * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// wide: the pair engine's 256 x 512 tiles (one problem, bf16 TMA-store epilogue,
// tiles_n counted in 512-column tiles).
void launch_tc(const Engine& eg, const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& a1,
               const CUtensorMap& b1, const TcParams& prm, const DeviceCtx* dev, cudaStream_t stream,
               const CUtensorMap* c0 = nullptr, const CUtensorMap* c1 = nullptr, const ShardMaps* shards = nullptr,
               bool wide = false) {
  CUtensorMap zc;
  std::memset(&zc, 0, sizeof(zc));
  NoShards ns;
  ns.unused = 0;
  const int sms = dev->sms;
  int64_t tiles = (int64_t)prm.prob[0].tiles_m * prm.prob[0].tiles_n;
  if (prm.nprob > 1) tiles += (int64_t)prm.prob[1].tiles_m * prm.prob[1].tiles_n;
  if (eg.pair) {
    const int pairs = (int)std::min<int64_t>(dev->pairs, tiles);
    if (wide)
      tc_gemm_pair_kernel<NoShards, true><<<2 * pairs, TC_THREADS, T2W_SMEM_BYTES, stream>>>(
          a0, b0, a1, b1, c0 ? *c0 : zc, c1 ? *c1 : zc, ns, prm);
    else if (shards)
      tc_gemm_pair_kernel<ShardMaps><<<2 * pairs, TC_THREADS, T2_SMEM_BYTES, stream>>>(
          a0, b0, a1, b1, c0 ? *c0 : zc, c1 ? *c1 : zc, *shards, prm);
    else
      tc_gemm_pair_kernel<NoShards><<<2 * pairs, TC_THREADS, T2_SMEM_BYTES, stream>>>(
          a0, b0, a1, b1, c0 ? *c0 : zc, c1 ? *c1 : zc, ns, prm);
  } else {
    const int grid = (int)std::min<int64_t>(sms, tiles);
    tc_gemm_kernel<<<grid, TC_THREADS, TC_SMEM_BYTES, stream>>>(a0, b0, a1, b1, prm);
  }
}

// ------------------------------------------------------------------ recompute schedule
// FLCE_FLAG_RECOMPUTE: the vocabulary-outer schedule. The first pass runs the
// logits GEMM over row blocks with the online-softmax epilogue but stores
// nothing, and the row combine keeps lse. The second pass takes the vocabulary
// in chunks of Vc columns: the logits of all rows over the chunk are rebuilt
// by GEMM and the epilogue writes dz = (softmax - onehot) * scale straight into
// a [BT, Vc] store; then grad_X (+)= dz W_c (K = Vc; added into grad_X in L2
// after the first chunk) and grad_W[chunk] = dz^T X (K = BT, complete in one
// GEMM). 8 * BT * H * V tensor FLOPs instead of 6, for a store whose size the
// caller picks down to BT * 256 * 2 bytes.
flce_status run_recompute_passes(const flce_tensor* X, const flce_tensor* W, const int64_t* tgt,
                                 int64_t ignore_index, int32_t reduction, flce_tensor* grad_X, flce_tensor* grad_W,
                                 bool want_gx, bool want_gw, const Plan& pl, uint8_t* base, const int64_t* nvalid,
                                 float* row_loss, const float* row_grad, float* lse_out, const Engine& eg,
                                 const DeviceCtx* dev, cudaStream_t stream, Launcher& L) {
  const int64_t BT = pl.BT, H = pl.H, V = pl.V;
  const int64_t ldx = X->stride[0], ldw = W->stride[0];
  const __nv_bfloat16* Xp = static_cast<const __nv_bfloat16*>(X->data);
  const __nv_bfloat16* Wp = static_cast<const __nv_bfloat16*>(W->data);
  float* zt = reinterpret_cast<float*>(base + pl.off_zt);
  float* pm = reinterpret_cast<float*>(base + pl.off_pm);
  float* ps = reinterpret_cast<float*>(base + pl.off_ps);
  __nv_bfloat16* E = reinterpret_cast<__nv_bfloat16*>(base + pl.off_e);
  float* lse = lse_out ? lse_out : reinterpret_cast<float*>(base + pl.off_lse);
  CUtensorMap z;
  std::memset(&z, 0, sizeof(z));
  flce_status st = FLCE_OK;
  // pass 1: row logsumexp and per-row losses, nothing stored
  for (int64_t r0 = 0, blk = 0; r0 < BT; r0 += pl.r1, ++blk) {
    L.chunk = blk;
    const int rows = (int)std::min<int64_t>(pl.r1, BT - r0);
    CUtensorMap ta, tb;
    if (!make_tmap(&ta, Xp + r0 * ldx, H, rows, ldx * 2, 64, 128) || !make_tmap(&tb, Wp, H, V, ldw * 2, 64, eg.b_box_rows))
      return FLCE_ERR_CUDA;
    TcParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.nprob = 1;
    prm.prob[0] = make_problem(eg, rows, (int)V, (int)H, 0, 0, EPI_LOGITS, 1);
    prm.lg.target = tgt + r0;
    prm.lg.ignore_index = ignore_index;
    prm.lg.V = V;
    prm.lg.part_m = pm;
    prm.lg.part_s = ps;
    prm.lg.ldp = pl.ldp;
    prm.lg.zt = zt;
    prm.lg.store = 0;
    prm.err = dev->err;
    st = L.run(1, [&] { launch_tc(eg, ta, tb, z, z, prm, dev, stream, &z); });
    if (st != FLCE_OK) return st;
    CombineArgs a{tgt + r0, ignore_index, V, rows, (int)pl.ntile, pl.ldp, pm, ps, zt, row_loss + r0, lse + r0, nvalid,
                  reduction, nullptr, 1};
    st = L.run(2, [&] { combine_kernel<<<(unsigned)ceil_div(rows, 32), CB_THREADS, 0, stream>>>(a); });
    if (st != FLCE_OK) return st;
  }
  if (!want_gx && !want_gw) return FLCE_OK;
  // pass 2: per vocabulary chunk, dz by GEMM, then the two gradient contractions
  const int64_t vc = pl.chunk;
  for (int64_t c = 0; c < pl.n_chunks; ++c) {
    L.chunk = c;
    const int64_t v0 = c * vc;
    const int cols = (int)std::min<int64_t>(vc, V - v0);
    const __nv_bfloat16* Wc = Wp + v0 * ldw;
    {
      CUtensorMap ta, tb, te;
      if (!make_tmap(&ta, Xp, H, BT, ldx * 2, 64, 128) || !make_tmap(&tb, Wc, H, cols, ldw * 2, 64, eg.b_box_rows) ||
          !make_out_tmap(&te, E, BT, cols, vc))
        return FLCE_ERR_CUDA;
      TcParams prm;
      std::memset(&prm, 0, sizeof(prm));
      prm.nprob = 1;
      TcProblem P = make_problem(eg, (int)BT, cols, (int)H, 0, 0, EPI_DLOGITS, 1);
      P.group_m = 16;  // a group's X rows (16 x 256 rows) stay in L2 while it sweeps the chunk's columns
      prm.prob[0] = P;
      prm.lg.target = tgt;
      prm.lg.ignore_index = ignore_index;
      prm.lg.V = V;
      prm.lg.lse = lse;
      prm.lg.n_valid = nvalid;
      prm.lg.reduction = reduction;
      prm.lg.row_grad = row_grad;
      prm.lg.v0 = v0;
      prm.err = dev->err;
      st = L.run(1, [&] { launch_tc(eg, ta, tb, z, z, prm, dev, stream, &te); });
      if (st != FLCE_OK) return st;
    }
    CUtensorMap tm[4], tc[2];
    std::memset(tm, 0, sizeof(tm));
    std::memset(tc, 0, sizeof(tc));
    TcParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.err = dev->err;
    int np = 0;
    if (want_gx) {
      // grad_X (+)= dz_c W_c: dz K-major [BT, cols], W_c MN-major [cols, H]
      if (!make_tmap(&tm[2 * np], E, cols, BT, vc * 2, 64, TC_BM) || !make_tmap(&tm[2 * np + 1], Wc, H, cols, ldw * 2, 64, 64))
        return FLCE_ERR_CUDA;
      TcProblem P = make_problem(eg, (int)BT, (int)H, cols, 0, 1, EPI_GRADW, 1);
      P.group_m = 16;
      P.out = grad_X->data;
      P.ldo = grad_X->stride[0];
      P.gw_mode = c == 0 ? GW_STORE_BF16 : GW_ADD_BF16;
      if (!make_out_tmap(&tc[np], P.out, BT, H, grad_X->stride[0])) return FLCE_ERR_CUDA;
      prm.prob[np++] = P;
    }
    if (want_gw) {
      // grad_W[v0 : v0 + cols] = dz_c^T X: dz MN-major (K = BT), X MN-major
      if (!make_tmap(&tm[2 * np], E, cols, BT, vc * 2, 64, 64) || !make_tmap(&tm[2 * np + 1], Xp, H, BT, ldx * 2, 64, 64))
        return FLCE_ERR_CUDA;
      TcProblem P = make_problem(eg, cols, (int)H, (int)BT, 1, 1, EPI_GRADW, 0);
      P.out = static_cast<__nv_bfloat16*>(grad_W->data) + v0 * grad_W->stride[0];
      P.ldo = grad_W->stride[0];
      P.gw_mode = GW_STORE_BF16;
      if (!make_out_tmap(&tc[np], P.out, cols, H, grad_W->stride[0])) return FLCE_ERR_CUDA;
      prm.prob[np++] = P;
    }
    const int64_t units = dev->pairs;
    if (np == 2 && !grad_combined((int64_t)prm.prob[0].tiles_m * prm.prob[0].tiles_n, units)) {
      TcParams p1 = prm, p2 = prm;
      p1.nprob = 1;
      p1.prob[1] = TcProblem{};
      p2.nprob = 1;
      p2.prob[0] = prm.prob[1];
      p2.prob[1] = TcProblem{};
      st = L.run(4, [&] { launch_tc(eg, tm[0], tm[1], z, z, p1, dev, stream, &tc[0]); });
      if (st != FLCE_OK) return st;
      st = L.run(4, [&] { launch_tc(eg, tm[2], tm[3], z, z, p2, dev, stream, &tc[1]); });
    } else {
      prm.nprob = np;
      st = L.run(4, [&] { launch_tc(eg, tm[0], tm[1], tm[2], tm[3], prm, dev, stream, &tc[0], &tc[1]); });
    }
    if (st != FLCE_OK) return st;
  }
  return FLCE_OK;
}

// ------------------------------------------------------------------ FLCE
flce_status run_flce(const flce_tensor* X, const flce_tensor* W, const flce_tensor* target,
                     int64_t ignore_index, int32_t reduction, flce_tensor* loss,
                     flce_tensor* grad_X, flce_tensor* grad_W, cudaStream_t stream,
                     const flce_options* opt, flce_stats* stats) {
  // ---- host-side argument checks (nothing is enqueued before they pass)
  if (!X || !W || !target || !loss) return FLCE_ERR_INVALID_ARG;
  if (reduction != FLCE_MEAN && reduction != FLCE_SUM && reduction != FLCE_NONE) return FLCE_ERR_INVALID_ARG;
  const int32_t dt = X->dtype;
  if (dt != FLCE_BF16 && dt != FLCE_F32) return FLCE_ERR_UNSUPPORTED_DTYPE;
  if (W->dtype != dt) return FLCE_ERR_UNSUPPORTED_DTYPE;
  if (X->ndim != 2 || W->ndim != 2) return FLCE_ERR_INVALID_ARG;
  const int64_t BT = X->shape[0], H = X->shape[1], V = W->shape[0];
  if (BT < 0 || H <= 0 || V <= 0 || W->shape[1] != H) return FLCE_ERR_INVALID_ARG;
  if (BT >= (1ll << 31) || V >= (1ll << 31) || H >= (1ll << 31)) return FLCE_ERR_INVALID_ARG;
  if ((BT > 0 && !check_matrix(X, dt, BT, H)) || !check_matrix(W, dt, V, H)) return FLCE_ERR_INVALID_ARG;
  if (target->dtype != FLCE_I64 || target->ndim != 1 || target->shape[0] != BT ||
      (BT > 0 && (!target->data || target->stride[0] != 1)))
    return FLCE_ERR_INVALID_ARG;
  if (reduction == FLCE_NONE) {
    // per-row losses: f32 [BT], contiguous
    if (loss->dtype != FLCE_F32 || loss->ndim != 1 || loss->shape[0] != BT ||
        (BT > 0 && (!loss->data || loss->stride[0] != 1)))
      return FLCE_ERR_INVALID_ARG;
  } else if (!loss->data || loss->dtype != FLCE_F32 || loss->ndim > 1 ||
             (loss->ndim == 1 && loss->shape[0] != 1)) {
    return FLCE_ERR_INVALID_ARG;
  }
  if (grad_X && (BT > 0 && !check_matrix(grad_X, dt, BT, H))) return FLCE_ERR_INVALID_ARG;
  if (grad_W && !check_matrix(grad_W, dt, V, H)) return FLCE_ERR_INVALID_ARG;
  // grad_W scattered to (possibly peer) shards
  const bool sharded = opt && opt->n_shards > 0;
  if (sharded) {
    if (dt != FLCE_BF16 || grad_W || !opt->grad_w_shards || opt->n_shards > MAX_SHARDS) return FLCE_ERR_INVALID_ARG;
    if (opt->shard_rows <= 0 || opt->shard_rows % 32 || opt->shard_rows * opt->n_shards < V) return FLCE_ERR_INVALID_ARG;
    if (opt->grad_w_shard_ld < H || opt->grad_w_shard_ld % 8 || opt->grad_w_accum != FLCE_GRADW_ACCUM_OUTPUT)
      return FLCE_ERR_INVALID_ARG;
    for (int k = 0; k < opt->n_shards; ++k)
      if (k * opt->shard_rows < V && (!opt->grad_w_shards[k] || !is_aligned(opt->grad_w_shards[k], 16)))
        return FLCE_ERR_INVALID_ARG;
    if (!engine().pair) return FLCE_ERR_INVALID_ARG;  // shard routing lives in the pair engine's epilogue
  }
  if (dt == FLCE_BF16) {
    // TMA and 16-byte vector stores: 16-byte aligned bases and rows
    if (H % 8 || !is_aligned(W->data, 16) || W->stride[0] % 8) return FLCE_ERR_INVALID_ARG;
    if (BT > 0 && (!is_aligned(X->data, 16) || X->stride[0] % 8)) return FLCE_ERR_INVALID_ARG;
    if (grad_X && BT > 0 && (!is_aligned(grad_X->data, 16) || grad_X->stride[0] % 8)) return FLCE_ERR_INVALID_ARG;
    if (grad_W && (!is_aligned(grad_W->data, 16) || grad_W->stride[0] % 8)) return FLCE_ERR_INVALID_ARG;
  }
  // two-phase use: a forward pass that keeps its chunk store, then gradients from it
  const bool keep = opt && (opt->flags & FLCE_FLAG_KEEP_LOGITS);
  const bool from_kept = opt && (opt->flags & FLCE_FLAG_FROM_KEPT);
  if (keep && from_kept) return FLCE_ERR_INVALID_ARG;
  if ((keep || from_kept) && !opt->workspace) return FLCE_ERR_INVALID_ARG;  // must outlive the call
  if (keep && (grad_X || grad_W || sharded)) return FLCE_ERR_INVALID_ARG;
  if (opt && (opt->flags & FLCE_FLAG_RECOMPUTE) && !engine().pair) return FLCE_ERR_INVALID_ARG;
  const bool want_gx = grad_X != nullptr && BT > 0;
  const bool want_gw = grad_W != nullptr || sharded;
  const bool need_rowloss = reduction != FLCE_NONE && !(opt && opt->row_loss);
  Plan pl;
  flce_status st = make_plan(BT, H, V, dt, want_gw, opt, need_rowloss, &pl);
  if (st != FLCE_OK) return st;

  DeviceCtx* dev = nullptr;
  st = device_ctx(&dev);
  if (st != FLCE_OK) return st;

  Launcher L{stream, opt && (opt->flags & FLCE_FLAG_TIME_PHASES), env_debug() || (opt && (opt->flags & FLCE_FLAG_SYNC_CHECK))};
  if (stats) {
    std::memset(stats, 0, sizeof(*stats));
    stats->chunk_rows = pl.chunk;
    stats->n_chunks = pl.n_chunks;
    stats->workspace_bytes = (int64_t)pl.total;
    stats->materialized_logits_bytes = BT * V * 2;
    stats->path = dt == FLCE_BF16 ? 1 : 0;
  }
  if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;

  // the caller's grad_W-ready event: recorded once, mid-step when the last chunk can order
  // grad_W before grad_X, else at the end
  const cudaEvent_t gw_event = opt ? static_cast<cudaEvent_t>(opt->grad_w_ready_event) : nullptr;
  bool gw_event_done = false;
  auto record_gw_event = [&]() -> flce_status {
    if (!gw_event || gw_event_done) return FLCE_OK;
    gw_event_done = true;
    return cudaEventRecord(gw_event, stream) == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
  };

  if (BT == 0) {
    if (reduction != FLCE_NONE && cudaMemsetAsync(loss->data, 0, 4, stream) != cudaSuccess) return FLCE_ERR_CUDA;
    // shards receive additions only: nothing to add for an empty batch
    if (grad_W && cudaMemset2DAsync(grad_W->data, grad_W->stride[0] * dtype_size(dt), 0,
                                    H * dtype_size(dt), V, stream) != cudaSuccess)
      return FLCE_ERR_CUDA;
    if (stats) stats->workspace_bytes = 0;
    return record_gw_event();
  }

  Workspace ws;
  st = get_workspace(opt, pl.total, stream, dev->pool, &ws);
  if (st != FLCE_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(ws.ptr);
  int64_t* nvalid_local = reinterpret_cast<int64_t*>(base + pl.off_nvalid);
  const int64_t* nvalid = (opt && opt->n_valid) ? opt->n_valid : nvalid_local;
  float* row_loss = reduction == FLCE_NONE ? static_cast<float*>(loss->data)
                    : need_rowloss ? reinterpret_cast<float*>(base + pl.off_rowloss) : opt->row_loss;
  const float* row_grad = opt ? opt->row_grad : nullptr;
  float* zt = reinterpret_cast<float*>(base + pl.off_zt);
  float* pm = reinterpret_cast<float*>(base + pl.off_pm);
  float* ps = reinterpret_cast<float*>(base + pl.off_ps);
  void* estore = base + pl.off_e;
  float* facc = pl.facc ? reinterpret_cast<float*>(base + pl.off_facc) : nullptr;
  float* xpart = pl.xpart_elems ? reinterpret_cast<float*>(base + pl.off_xpart) : nullptr;
  float* lse_out = opt ? opt->lse : nullptr;
  float* lse_kept = pl.keep ? reinterpret_cast<float*>(base + pl.off_lse) : nullptr;
  __nv_bfloat16* gw_local = pl.gw_local ? reinterpret_cast<__nv_bfloat16*>(base + pl.off_gwl) : nullptr;
  const int64_t* tgt = static_cast<const int64_t*>(target->data);

  // A0: N (always run: it also flags targets outside [0, V))
  st = L.run(0, [&] {
    count_valid_kernel<<<1, 1024, 0, stream>>>(tgt, BT, V, ignore_index, nvalid_local, dev->err);
  });
  if (st != FLCE_OK) return st;

  const int64_t ldx = X->stride[0], ldw = W->stride[0];
  const Engine eg = engine();
  if (pl.recompute) {
    st = run_recompute_passes(X, W, tgt, ignore_index, reduction, grad_X, grad_W, want_gx, want_gw, pl, base,
                              nvalid, row_loss, row_grad, lse_out, eg, dev, stream, L);
    if (st != FLCE_OK) return st;
  }
  // the stored-chunk schedule (the recompute schedule ran above instead)
  const int64_t stored_chunks = pl.recompute ? 0 : pl.n_chunks;
  for (int64_t c = 0; c < stored_chunks; ++c) {
    L.chunk = c;
    const int64_t r0 = c * pl.chunk;
    const int rows = (int)std::min<int64_t>(pl.chunk, BT - r0);
    const int64_t* tgt_c = tgt + r0;
    if (from_kept) {
      // the store and tile maxima are those the KEEP_LOGITS call left; turn the
      // maxima into factors with this call's row_grad and scale
      FactorArgs a{tgt_c, ignore_index, V, rows, (int)pl.ntile, pl.ldp, pm, lse_kept, nvalid, reduction,
                   row_grad ? row_grad + r0 : nullptr};
      st = L.run(2, [&] { factor_kernel<<<(unsigned)ceil_div(rows, 32), CB_THREADS, 0, stream>>>(a); });
      if (st != FLCE_OK) return st;
    } else if (dt == FLCE_BF16) {
      const __nv_bfloat16* Xc = static_cast<const __nv_bfloat16*>(X->data) + r0 * ldx;
      const __nv_bfloat16* Wp = static_cast<const __nv_bfloat16*>(W->data);
      __nv_bfloat16* E = static_cast<__nv_bfloat16*>(estore);
      // A1 + A2
      {
        CUtensorMap ta, tb, z;
        std::memset(&z, 0, sizeof(z));
        if (!make_tmap(&ta, Xc, H, rows, ldx * 2, 64, 128) || !make_tmap(&tb, Wp, H, V, ldw * 2, 64, eg.b_box_rows))
          return FLCE_ERR_CUDA;
        TcParams prm;
        std::memset(&prm, 0, sizeof(prm));
        prm.nprob = 1;
        prm.prob[0] = make_problem(eg, rows, (int)V, (int)H, 0, 0, EPI_LOGITS, 1);
        prm.lg = LogitsArgs{tgt_c, ignore_index, V, E, pl.lde, pm, ps, pl.ldp, zt};
        prm.lg.store = 1;
        prm.err = dev->err;
        // the pair engine writes the chunk store through TMA boxes
        CUtensorMap te;
        if (!make_out_tmap(&te, E, rows, V, pl.lde)) return FLCE_ERR_CUDA;
        st = L.run(1, [&] { launch_tc(eg, ta, tb, z, z, prm, dev, stream, &te); });
        if (st != FLCE_OK) return st;
      }
    } else {
      SimtArgs s;
      std::memset(&s, 0, sizeof(s));
      s.A = static_cast<const float*>(X->data) + r0 * ldx; s.sam = ldx; s.sak = 1;
      s.B = static_cast<const float*>(W->data); s.sbn = ldw; s.sbk = 1;
      s.M = rows; s.N = (int)V; s.K = (int)H;
      s.epi = SEPI_LOGITS;
      s.out = static_cast<float*>(estore); s.ldo = pl.lde;
      s.target = tgt_c; s.ignore_index = ignore_index;
      s.part_m = pm; s.part_s = ps; s.ldp = pl.ldp; s.zt = zt;
      st = L.run(1, [&] {
        simt_gemm_kernel<<<dim3((unsigned)ceil_div(V, SG_BN), (unsigned)ceil_div(rows, SG_BM)), 256, 0, stream>>>(s);
      });
      if (st != FLCE_OK) return st;
    }
    // A3
    if (!from_kept) {
      CombineArgs a{tgt_c, ignore_index, V, rows, (int)pl.ntile, pl.ldp, pm, ps, zt,
                    row_loss + r0, keep ? lse_kept : (lse_out ? lse_out + r0 : nullptr), nvalid, reduction,
                    row_grad ? row_grad + r0 : nullptr, keep ? 1 : 0};
      st = L.run(2, [&] { combine_kernel<<<(unsigned)ceil_div(rows, 32), CB_THREADS, 0, stream>>>(a); });
      if (st != FLCE_OK) return st;
      if (keep && lse_out &&
          cudaMemcpyAsync(lse_out, lse_kept, (size_t)rows * 4, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
        return FLCE_ERR_CUDA;
    }
    if (!want_gx && !want_gw) continue;
    // A4
    {
      const int shift = dt == FLCE_BF16 ? 8 : 6;
      const dim3 grid((unsigned)ceil_div(V, (int64_t)DL_COLS), (unsigned)rows);
      if (dt == FLCE_BF16) {
        __nv_bfloat16* E = static_cast<__nv_bfloat16*>(estore);
        DlogitsArgs<__nv_bfloat16> a{E, pl.lde, E, pl.lde, tgt_c, ignore_index, V, pm, pl.ldp, shift, nvalid, reduction,
                                     row_grad ? row_grad + r0 : nullptr};
        st = L.run(3, [&] { dlogits_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(a); });
      } else {
        float* E = static_cast<float*>(estore);
        DlogitsArgs<float> a{E, pl.lde, E, pl.lde, tgt_c, ignore_index, V, pm, pl.ldp, shift, nvalid, reduction,
                             row_grad ? row_grad + r0 : nullptr};
        st = L.run(3, [&] { dlogits_kernel<float><<<grid, 256, 0, stream>>>(a); });
      }
      if (st != FLCE_OK) return st;
    }
    // A5 + A6
    if (dt == FLCE_BF16) {
      const __nv_bfloat16* Xc = static_cast<const __nv_bfloat16*>(X->data) + r0 * ldx;
      const __nv_bfloat16* Wp = static_cast<const __nv_bfloat16*>(W->data);
      __nv_bfloat16* E = static_cast<__nv_bfloat16*>(estore);
      CUtensorMap tm[4], tc[2];
      std::memset(tm, 0, sizeof(tm));
      std::memset(tc, 0, sizeof(tc));
      ShardMaps shard_maps;
      std::memset(&shard_maps, 0, sizeof(shard_maps));
      TcParams prm;
      std::memset(&prm, 0, sizeof(prm));
      prm.err = dev->err;
      int np = 0;
      int gx_split = 1;
      bool gx_wide = false;  // grad_X on 256 x 512 tiles (then launched on its own)
      if (want_gx) {
        if (!make_tmap(&tm[2 * np], E, V, rows, pl.lde * 2, 64, TC_BM) ||
            !make_tmap(&tm[2 * np + 1], Wp, H, V, ldw * 2, 64, 64))
          return FLCE_ERR_CUDA;
        TcProblem P = make_problem(eg, rows, (int)H, (int)V, 0, 1, EPI_STORE_BF16, 1);
        P.out = static_cast<__nv_bfloat16*>(grad_X->data) + r0 * grad_X->stride[0];
        P.ldo = grad_X->stride[0];
        if (!make_out_tmap(&tc[np], P.out, rows, H, grad_X->stride[0])) return FLCE_ERR_CUDA;
        // few output tiles and a long K: split K so every SM (pair) has work
        int S = choose_ksplit((int64_t)P.tiles_m * P.tiles_n, P.kblocks, eg.pair ? dev->pairs : dev->sms);
        while (S > 1 && (int64_t)S * rows * H > pl.xpart_elems) --S;
        if (S > 1) {
          P.kb_per_split = (int)ceil_div(P.kblocks, S);
          P.ksplit = (int)ceil_div(P.kblocks, P.kb_per_split);
          P.epi = EPI_STORE_F32;
          P.out = xpart;
          P.ldo = H;
          P.split_stride = (int64_t)rows * H;
          gx_split = P.ksplit;
        }
        if (eg.pair && gx_split == 1 && gradx_wide(P.tiles_m, H, dev->pairs)) {
          gx_wide = true;
          P.tiles_n = (int)ceil_div(H, T2W_BN);
          // one wave of wide tiles: keep the pairs in step along K (counters zeroed first)
          const int64_t wide_tiles = (int64_t)P.tiles_m * P.tiles_n;
          const int64_t ckpts = P.kblocks / KSYNC_EVERY + 1;
          if (wide_tiles <= dev->pairs && ckpts <= KSYNC_MAX_CKPT && ksync_enabled()) {
            if (cudaMemsetAsync(dev->ksync, 0, (size_t)ckpts * 4, stream) != cudaSuccess) return FLCE_ERR_CUDA;
            prm.kprog = dev->ksync;
            prm.ksync_pairs = (int)wide_tiles;
          }
        }
        prm.prob[np++] = P;
      }
      if (want_gw) {
        if (!make_tmap(&tm[2 * np], E, V, rows, pl.lde * 2, 64, 64) ||
            !make_tmap(&tm[2 * np + 1], Xc, H, rows, ldx * 2, 64, 64))
          return FLCE_ERR_CUDA;
        TcProblem P = make_problem(eg, (int)V, (int)H, rows, 1, 1, EPI_GRADW, 0);
        const bool last = c == pl.n_chunks - 1;
        if (gw_local && !last) {
          // shards, chunk before the last: accumulate locally (store, then L2 adds)
          P.out = gw_local;
          P.ldo = H;
          if (!make_out_tmap(&tc[np], gw_local, V, H, H)) return FLCE_ERR_CUDA;
          P.gw_mode = c == 0 ? GW_STORE_BF16 : GW_ADD_BF16;
        } else if (sharded) {
          P.n_shards = opt->n_shards;
          P.shard_rows = opt->shard_rows;
          P.gw_mode = GW_ADD_BF16;
          for (int k = 0; k < opt->n_shards; ++k) {
            const int64_t r0k = k * opt->shard_rows;
            if (r0k >= V) break;
            if (!make_out_tmap(&shard_maps.m[k], opt->grad_w_shards[k], std::min(opt->shard_rows, V - r0k), H,
                               opt->grad_w_shard_ld))
              return FLCE_ERR_CUDA;
          }
          // the last chunk adds the earlier chunks' local sum to each box on its way to the owner
          if (gw_local) {
            P.gw_local = gw_local;
            P.ld_local = H;
          }
          P.gw_mode = GW_ADD_BF16;
        } else {
          P.out = grad_W->data;
          P.ldo = grad_W->stride[0];
          if (!make_out_tmap(&tc[np], P.out, V, H, grad_W->stride[0])) return FLCE_ERR_CUDA;
          if (!pl.facc) P.gw_mode = c == 0 ? GW_STORE_BF16 : GW_ADD_BF16;
          else P.gw_mode = c == 0 ? GW_STORE_F32 : (last ? GW_FINAL_F32 : GW_ADD_F32);
        }
        P.facc = facc;
        P.ld_facc = H;
        prm.prob[np++] = P;
      }
      // this chunk's grad_W boxes go to the owner shards (the last chunk, or every
      // chunk when there is no local accumulation)
      const bool route = sharded && want_gw && (!gw_local || c == pl.n_chunks - 1);
      const int64_t units = eg.pair ? dev->pairs : dev->sms;
      if (np == 2 && (gx_wide || !grad_combined((int64_t)prm.prob[0].tiles_m * prm.prob[0].tiles_n * prm.prob[0].ksplit,
                                                 units))) {
        // grad_X and grad_W as two launches: they contend for L2 when interleaved
        TcParams p1 = prm;
        p1.nprob = 1;
        p1.prob[1] = TcProblem{};
        TcParams p2 = prm;
        p2.nprob = 1;
        p2.prob[0] = prm.prob[1];
        p2.prob[1] = TcProblem{};
        p2.kprog = nullptr;  // the K-synchronisation is grad_X's
        p2.ksync_pairs = 0;
        CUtensorMap z;
        std::memset(&z, 0, sizeof(z));
        auto run_gx = [&] {
          return L.run(4, [&] { launch_tc(eg, tm[0], tm[1], z, z, p1, dev, stream, &tc[0], nullptr, nullptr,
                                          gx_wide); });
        };
        auto run_gw = [&] {
          return L.run(4, [&] { launch_tc(eg, tm[2], tm[3], z, z, p2, dev, stream, &tc[1], nullptr,
                                          route ? &shard_maps : nullptr); });
        };
        if (gw_event && c == pl.n_chunks - 1) {
          // the last chunk: grad_W first, then the event, so that the caller's work behind it
          // overlaps the grad_X GEMM
          st = run_gw();
          if (st != FLCE_OK) return st;
          st = record_gw_event();
          if (st != FLCE_OK) return st;
          st = run_gx();
        } else {
          st = run_gx();
          if (st != FLCE_OK) return st;
          st = run_gw();
        }
      } else if (np == 1 && gx_wide) {
        prm.nprob = 1;
        st = L.run(4, [&] { launch_tc(eg, tm[0], tm[1], tm[2], tm[3], prm, dev, stream, &tc[0], nullptr, nullptr,
                                      true); });
      } else {
        prm.nprob = np;
        st = L.run(4, [&] { launch_tc(eg, tm[0], tm[1], tm[2], tm[3], prm, dev, stream, &tc[0], &tc[1],
                                      route ? &shard_maps : nullptr); });
      }
      if (st != FLCE_OK) return st;
      if (gx_split > 1) {
        __nv_bfloat16* gx = static_cast<__nv_bfloat16*>(grad_X->data) + r0 * grad_X->stride[0];
        const int64_t n4 = (int64_t)rows * H / 4;
        const int blocks = (int)std::min<int64_t>(ceil_div(n4, 256), 8 * dev->sms);
        st = L.run(4, [&] {
          splitk_reduce_kernel<<<blocks, 256, 0, stream>>>(xpart, gx_split, (int64_t)rows * H, rows, (int)H, gx,
                                                           grad_X->stride[0]);
        });
        if (st != FLCE_OK) return st;
      }
    } else {
      float* E = static_cast<float*>(estore);
      if (want_gx) {
        SimtArgs s;
        std::memset(&s, 0, sizeof(s));
        s.A = E; s.sam = pl.lde; s.sak = 1;
        s.B = static_cast<const float*>(W->data); s.sbn = 1; s.sbk = ldw;
        s.M = rows; s.N = (int)H; s.K = (int)V;
        s.epi = SEPI_STORE;
        s.out = static_cast<float*>(grad_X->data) + r0 * grad_X->stride[0];
        s.ldo = grad_X->stride[0];
        st = L.run(4, [&] {
          simt_gemm_kernel<<<dim3((unsigned)ceil_div(H, SG_BN), (unsigned)ceil_div(rows, SG_BM)), 256, 0, stream>>>(s);
        });
        if (st != FLCE_OK) return st;
      }
      if (want_gw) {
        SimtArgs s;
        std::memset(&s, 0, sizeof(s));
        s.A = E; s.sam = 1; s.sak = pl.lde;
        s.B = static_cast<const float*>(X->data) + r0 * ldx; s.sbn = 1; s.sbk = ldx;
        s.M = (int)V; s.N = (int)H; s.K = rows;
        s.epi = c == 0 ? SEPI_GRADW_STORE : SEPI_GRADW_ADD;
        s.out = static_cast<float*>(grad_W->data);
        s.ldo = grad_W->stride[0];
        st = L.run(4, [&] {
          simt_gemm_kernel<<<dim3((unsigned)ceil_div(H, SG_BN), (unsigned)ceil_div(V, SG_BM)), 256, 0, stream>>>(s);
        });
        if (st != FLCE_OK) return st;
      }
    }
  }
  L.chunk = -1;
  if (reduction != FLCE_NONE && !from_kept) {
    st = L.run(5, [&] {
      finalize_loss_kernel<<<1, 1024, 0, stream>>>(row_loss, BT, nvalid, reduction,
                                                   static_cast<float*>(loss->data));
    });
    if (st != FLCE_OK) return st;
  }
  if (stats) stats->kernel_launches = L.launches;
  return record_gw_event();
}

// ------------------------------------------------------------------ CE (logits given)
flce_status run_ce(const flce_tensor* Z, const flce_tensor* target, int64_t ignore_index,
                   int32_t reduction, flce_tensor* loss, flce_tensor* grad, cudaStream_t stream,
                   const flce_options* opt) {
  if (!Z || !target || !loss) return FLCE_ERR_INVALID_ARG;
  if (reduction != FLCE_MEAN && reduction != FLCE_SUM && reduction != FLCE_NONE) return FLCE_ERR_INVALID_ARG;
  const int32_t dt = Z->dtype;
  if (dt != FLCE_BF16 && dt != FLCE_F32) return FLCE_ERR_UNSUPPORTED_DTYPE;
  if (Z->ndim != 2) return FLCE_ERR_INVALID_ARG;
  const int64_t BT = Z->shape[0], V = Z->shape[1];
  if (BT < 0 || V <= 0 || BT >= (1ll << 31) || V >= (1ll << 31)) return FLCE_ERR_INVALID_ARG;
  if (BT > 0 && !check_matrix(Z, dt, BT, V)) return FLCE_ERR_INVALID_ARG;
  if (target->dtype != FLCE_I64 || target->ndim != 1 || target->shape[0] != BT ||
      (BT > 0 && (!target->data || target->stride[0] != 1)))
    return FLCE_ERR_INVALID_ARG;
  if (reduction == FLCE_NONE) {
    if (loss->dtype != FLCE_F32 || loss->ndim != 1 || loss->shape[0] != BT ||
        (BT > 0 && (!loss->data || loss->stride[0] != 1)))
      return FLCE_ERR_INVALID_ARG;
  } else if (!loss->data || loss->dtype != FLCE_F32 || loss->ndim > 1 ||
             (loss->ndim == 1 && loss->shape[0] != 1)) {
    return FLCE_ERR_INVALID_ARG;
  }
  const int esz = dtype_size(dt);
  if (BT > 0 && (!is_aligned(Z->data, 16) || (Z->stride[0] * esz) % 16)) return FLCE_ERR_INVALID_ARG;
  if (grad && BT > 0) {
    if (!check_matrix(grad, dt, BT, V)) return FLCE_ERR_INVALID_ARG;
    if (!is_aligned(grad->data, 16) || (grad->stride[0] * esz) % 16) return FLCE_ERR_INVALID_ARG;
  }
  DeviceCtx* dev = nullptr;
  flce_status st = device_ctx(&dev);
  if (st != FLCE_OK) return st;
  if (BT == 0) {
    if (reduction == FLCE_NONE) return FLCE_OK;
    return cudaMemsetAsync(loss->data, 0, 4, stream) == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
  }
  const int shift = 10;
  // bf16 rows up to (slice columns) * (largest cluster) take a one-pass cluster
  // kernel, which needs no partials; the rest take partials + combine + grad
  const bool regs = ce_slice_in_registers();
  const int64_t cer_c64 = regs ? ceil_div(V, CER_SLICE) : ce_smem_ctas(V, dev->ce_max_cluster);
  const int cer_c = (int)std::min<int64_t>(cer_c64, 1 << 20);
  const bool one_pass = dt == FLCE_BF16 && cer_c <= dev->ce_max_cluster && ce_one_pass_enabled();
  const int64_t ntile = one_pass ? 0 : ceil_div(V, 1 << shift), ldp = round_up(BT, 32);
  size_t o = 0;
  const size_t off_nv = o; o = align256(o + 8);
  const size_t off_rl = o; o = align256(o + (size_t)BT * 4);
  const size_t off_lse = o; o = align256(o + (one_pass ? 0 : (size_t)BT * 4));
  const size_t off_zt = o; o = align256(o + (one_pass ? 0 : (size_t)BT * 4));
  const size_t off_pm = o; o = align256(o + (size_t)ntile * ldp * 4);
  const size_t off_ps = o; o = align256(o + (size_t)ntile * ldp * 4);
  Workspace ws;
  st = get_workspace(nullptr, o, stream, dev->pool, &ws);
  if (st != FLCE_OK) return st;
  uint8_t* b = static_cast<uint8_t*>(ws.ptr);
  int64_t* nv_local = reinterpret_cast<int64_t*>(b + off_nv);
  const int64_t* nv = (opt && opt->n_valid) ? opt->n_valid : nv_local;
  float* rl = reduction == FLCE_NONE ? static_cast<float*>(loss->data)
              : (opt && opt->row_loss) ? opt->row_loss : reinterpret_cast<float*>(b + off_rl);
  const float* row_grad = opt ? opt->row_grad : nullptr;
  float* lse = (opt && opt->lse) ? opt->lse : reinterpret_cast<float*>(b + off_lse);
  float* zt = reinterpret_cast<float*>(b + off_zt);
  float* pm = reinterpret_cast<float*>(b + off_pm);
  float* ps = reinterpret_cast<float*>(b + off_ps);
  const int64_t* tgt = static_cast<const int64_t*>(target->data);
  Launcher L{stream, opt && (opt->flags & FLCE_FLAG_TIME_PHASES), env_debug() || (opt && (opt->flags & FLCE_FLAG_SYNC_CHECK))};
  st = L.run(0, [&] { count_valid_kernel<<<1, 1024, 0, stream>>>(tgt, BT, V, ignore_index, nv_local, dev->err); });
  if (st != FLCE_OK) return st;
  if (one_pass) {
    const int slice = (int)round_up(ceil_div(V, cer_c), 8);
    for (int64_t r0 = 0; r0 < BT; r0 += 65535) {
      const int rows = (int)std::min<int64_t>(65535, BT - r0);
      CeRowArgs a{static_cast<const __nv_bfloat16*>(Z->data) + r0 * Z->stride[0], Z->stride[0],
                  grad ? static_cast<__nv_bfloat16*>(grad->data) + r0 * grad->stride[0] : nullptr,
                  grad ? grad->stride[0] : 0, tgt + r0, ignore_index, V, rl + r0,
                  (opt && opt->lse) ? opt->lse + r0 : nullptr, nv, reduction, row_grad ? row_grad + r0 : nullptr,
                  slice};
      st = L.run(1, [&] {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)cer_c, (unsigned)rows, 1);
        cfg.blockDim = dim3(CER_THREADS, 1, 1);
        cfg.dynamicSmemBytes = regs ? 0 : (size_t)slice * 2;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)cer_c;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (regs)
          cudaLaunchKernelEx(&cfg, ce_row_cluster_kernel, a);
        else
          cudaLaunchKernelEx(&cfg, ce_row_smem_kernel, a, dev->err);
      });
      if (st != FLCE_OK) return st;
    }
    if (reduction == FLCE_NONE) return FLCE_OK;
    return L.run(5, [&] {
      finalize_loss_kernel<<<1, 1024, 0, stream>>>(rl, BT, nv, reduction, static_cast<float*>(loss->data));
    });
  }
  const int64_t warps = BT * ntile;
  if (dt == FLCE_BF16) {
    CePartialArgs<__nv_bfloat16> a{static_cast<const __nv_bfloat16*>(Z->data), Z->stride[0], tgt, ignore_index, V,
                                   pm, ps, ldp, zt, (int)BT, (int)ntile, shift};
    st = L.run(1, [&] { ce_partials_kernel<__nv_bfloat16><<<(unsigned)ceil_div(warps, 8), 256, 0, stream>>>(a); });
  } else {
    CePartialArgs<float> a{static_cast<const float*>(Z->data), Z->stride[0], tgt, ignore_index, V,
                           pm, ps, ldp, zt, (int)BT, (int)ntile, shift};
    st = L.run(1, [&] { ce_partials_kernel<float><<<(unsigned)ceil_div(warps, 8), 256, 0, stream>>>(a); });
  }
  if (st != FLCE_OK) return st;
  for (int64_t r0 = 0; r0 < BT; r0 += 65535 * 32) {
    const int rows = (int)std::min<int64_t>(65535 * 32, BT - r0);
    CombineArgs a{tgt + r0, ignore_index, V, rows, (int)ntile, ldp, pm + r0, ps + r0, zt + r0, rl + r0, lse + r0, nv, reduction,
                  row_grad ? row_grad + r0 : nullptr};
    st = L.run(2, [&] { combine_kernel<<<(unsigned)ceil_div(rows, 32), CB_THREADS, 0, stream>>>(a); });
    if (st != FLCE_OK) return st;
  }
  if (grad) {
    for (int64_t r0 = 0; r0 < BT; r0 += 65535) {
      const int rows = (int)std::min<int64_t>(65535, BT - r0);
      const dim3 grid((unsigned)ceil_div(V, CEG_BLOCK_COLS), (unsigned)rows);
      if (dt == FLCE_BF16) {
        CeGradArgs<__nv_bfloat16> a{static_cast<const __nv_bfloat16*>(Z->data) + r0 * Z->stride[0], Z->stride[0],
                                    static_cast<__nv_bfloat16*>(grad->data) + r0 * grad->stride[0], grad->stride[0],
                                    tgt + r0, ignore_index, V, lse + r0, nv, reduction,
                                    row_grad ? row_grad + r0 : nullptr};
        st = L.run(3, [&] { ce_grad_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(a); });
      } else {
        CeGradArgs<float> a{static_cast<const float*>(Z->data) + r0 * Z->stride[0], Z->stride[0],
                            static_cast<float*>(grad->data) + r0 * grad->stride[0], grad->stride[0],
                            tgt + r0, ignore_index, V, lse + r0, nv, reduction,
                            row_grad ? row_grad + r0 : nullptr};
        st = L.run(3, [&] { ce_grad_kernel<float><<<grid, 256, 0, stream>>>(a); });
      }
      if (st != FLCE_OK) return st;
    }
  }
  if (reduction == FLCE_NONE) return FLCE_OK;
  return L.run(5, [&] {
    finalize_loss_kernel<<<1, 1024, 0, stream>>>(rl, BT, nv, reduction, static_cast<float*>(loss->data));
  });
}

// ------------------------------------------------------------------ CE without allocation
// Some callers cannot allocate device memory at the point where they need the
// loss: code running while a CUDA graph is being captured around it, hosts
// that hand all device memory to their own allocator and forbid outside
// allocations, or real-time loops where an allocation (and the implicit
// synchronisation it may bring) is not allowed. For them,
// flce_cross_entropy_noalloc keeps its scratch in the fixed device array
// below instead of asking for a workspace. The array is part of the library
// image, so every GPU that loads the library holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocDevice {
  bool init = false;
  bool supported = false;
  uint8_t* scratch = nullptr;  // device address of g_noalloc_scratch on this device
  uint32_t* err = nullptr;     // device address of the error word on this device
};
std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[kMaxDevices];

// Once per device, with that device current: look up the device addresses of
// the scratch array and the error word, and load the kernels the entry point
// launches. (In host code the array's name is only a host-side stand-in; the
// kernels must be given the address found here.)
flce_status noalloc_device(NoAllocDevice** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLCE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FLCE_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoAllocDevice& d = g_noalloc_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return FLCE_ERR_CUDA;
    d.supported = major == 10 && minor == 0;
    if (d.supported) {
      if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d.scratch), g_noalloc_scratch) != cudaSuccess)
        return FLCE_ERR_CUDA;
      if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d.err), g_err_word) != cudaSuccess)
        return FLCE_ERR_CUDA;
      // load every kernel this entry point launches, so that no later call is the
      // first launch of one of them (under lazy module loading that may block the host)
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, count_valid_kernel) != cudaSuccess ||
          cudaFuncGetAttributes(&fa, ce_partials_kernel<__nv_bfloat16>) != cudaSuccess ||
          cudaFuncGetAttributes(&fa, ce_partials_kernel<float>) != cudaSuccess ||
          cudaFuncGetAttributes(&fa, combine_kernel) != cudaSuccess ||
          cudaFuncGetAttributes(&fa, ce_grad_kernel<__nv_bfloat16>) != cudaSuccess ||
          cudaFuncGetAttributes(&fa, ce_grad_kernel<float>) != cudaSuccess ||
          cudaFuncGetAttributes(&fa, finalize_loss_kernel) != cudaSuccess)
        return FLCE_ERR_CUDA;
    }
    d.init = true;
  }
  if (!d.supported) return FLCE_ERR_UNSUPPORTED_DEVICE;
  *out = &d;
  return FLCE_OK;
}

flce_status run_ce_noalloc(const flce_tensor* Z, const flce_tensor* target, int64_t ignore_index,
                           int32_t reduction, flce_tensor* loss, flce_tensor* grad, cudaStream_t stream) {
  if (!Z || !target || !loss) return FLCE_ERR_INVALID_ARG;
  if (reduction != FLCE_MEAN && reduction != FLCE_SUM) return FLCE_ERR_INVALID_ARG;
  const int32_t dt = Z->dtype;
  if (dt != FLCE_BF16 && dt != FLCE_F32) return FLCE_ERR_UNSUPPORTED_DTYPE;
  if (Z->ndim != 2) return FLCE_ERR_INVALID_ARG;
  const int64_t BT = Z->shape[0], V = Z->shape[1];
  if (BT < 0 || V <= 0 || BT >= (1ll << 31) || V >= (1ll << 31)) return FLCE_ERR_INVALID_ARG;
  if (BT > 0 && !check_matrix(Z, dt, BT, V)) return FLCE_ERR_INVALID_ARG;
  if (target->dtype != FLCE_I64 || target->ndim != 1 || target->shape[0] != BT ||
      (BT > 0 && (!target->data || target->stride[0] != 1)))
    return FLCE_ERR_INVALID_ARG;
  if (!loss->data || loss->dtype != FLCE_F32 || loss->ndim > 1 ||
      (loss->ndim == 1 && loss->shape[0] != 1))
    return FLCE_ERR_INVALID_ARG;
  const int esz = dtype_size(dt);
  if (BT > 0 && (!is_aligned(Z->data, 16) || (Z->stride[0] * esz) % 16)) return FLCE_ERR_INVALID_ARG;
  if (grad && BT > 0) {
    if (!check_matrix(grad, dt, BT, V)) return FLCE_ERR_INVALID_ARG;
    if (!is_aligned(grad->data, 16) || (grad->stride[0] * esz) % 16) return FLCE_ERR_INVALID_ARG;
  }
  // scratch plan; sizes beyond the fixed array are refused before any GPU work
  const int shift = 10;
  const int64_t ntile = ceil_div(V, 1 << shift), ldp = round_up(std::max<int64_t>(BT, 1), 32);
  size_t o = 0;
  const size_t off_nv = o; o = align256(o + 8);
  const size_t off_rl = o; o = align256(o + (size_t)BT * 4);
  const size_t off_lse = o; o = align256(o + (size_t)BT * 4);
  const size_t off_zt = o; o = align256(o + (size_t)BT * 4);
  const size_t off_pm = o; o = align256(o + (size_t)ntile * ldp * 4);
  const size_t off_ps = o; o = align256(o + (size_t)ntile * ldp * 4);
  if (o > kNoAllocScratchBytes) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  NoAllocDevice* d = nullptr;
  flce_status st = noalloc_device(&d);
  if (st != FLCE_OK) return st;
  if (BT == 0) return cudaMemsetAsync(loss->data, 0, 4, stream) == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
  // Every value read from the scratch below is written earlier in the same
  // call (count, partials, per-row values), so what a previous call left in
  // the array never leaks into this one and nothing needs clearing first.
  uint8_t* b = d->scratch;
  int64_t* nv = reinterpret_cast<int64_t*>(b + off_nv);
  float* rl = reinterpret_cast<float*>(b + off_rl);
  float* lse = reinterpret_cast<float*>(b + off_lse);
  float* zt = reinterpret_cast<float*>(b + off_zt);
  float* pm = reinterpret_cast<float*>(b + off_pm);
  float* ps = reinterpret_cast<float*>(b + off_ps);
  const int64_t* tgt = static_cast<const int64_t*>(target->data);
  count_valid_kernel<<<1, 1024, 0, stream>>>(tgt, BT, V, ignore_index, nv, d->err);
  const int64_t warps = BT * ntile;
  if (dt == FLCE_BF16) {
    CePartialArgs<__nv_bfloat16> a{static_cast<const __nv_bfloat16*>(Z->data), Z->stride[0], tgt, ignore_index, V,
                                   pm, ps, ldp, zt, (int)BT, (int)ntile, shift};
    ce_partials_kernel<__nv_bfloat16><<<(unsigned)ceil_div(warps, 8), 256, 0, stream>>>(a);
  } else {
    CePartialArgs<float> a{static_cast<const float*>(Z->data), Z->stride[0], tgt, ignore_index, V,
                           pm, ps, ldp, zt, (int)BT, (int)ntile, shift};
    ce_partials_kernel<float><<<(unsigned)ceil_div(warps, 8), 256, 0, stream>>>(a);
  }
  for (int64_t r0 = 0; r0 < BT; r0 += 65535 * 32) {
    const int rows = (int)std::min<int64_t>(65535 * 32, BT - r0);
    CombineArgs a{tgt + r0, ignore_index, V, rows, (int)ntile, ldp, pm + r0, ps + r0, zt + r0, rl + r0, lse + r0, nv, reduction};
    combine_kernel<<<(unsigned)ceil_div(rows, 32), CB_THREADS, 0, stream>>>(a);
  }
  if (grad) {
    for (int64_t r0 = 0; r0 < BT; r0 += 65535) {
      const int rows = (int)std::min<int64_t>(65535, BT - r0);
      const dim3 grid((unsigned)ceil_div(V, CEG_BLOCK_COLS), (unsigned)rows);
      if (dt == FLCE_BF16) {
        CeGradArgs<__nv_bfloat16> a{static_cast<const __nv_bfloat16*>(Z->data) + r0 * Z->stride[0], Z->stride[0],
                                    static_cast<__nv_bfloat16*>(grad->data) + r0 * grad->stride[0], grad->stride[0],
                                    tgt + r0, ignore_index, V, lse + r0, nv, reduction};
        ce_grad_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(a);
      } else {
        CeGradArgs<float> a{static_cast<const float*>(Z->data) + r0 * Z->stride[0], Z->stride[0],
                            static_cast<float*>(grad->data) + r0 * grad->stride[0], grad->stride[0],
                            tgt + r0, ignore_index, V, lse + r0, nv, reduction};
        ce_grad_kernel<float><<<grid, 256, 0, stream>>>(a);
      }
    }
  }
  finalize_loss_kernel<<<1, 1024, 0, stream>>>(rl, BT, nv, reduction, static_cast<float*>(loss->data));
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

// The engine on a plain GEMM (flce_gemm_bf16), optionally with the failure-path
// test hook (test_stall = output tile number + 1, 0 = off).
flce_status run_gemm_bf16(const void* A, const void* B, float* C, int64_t M, int64_t N, int64_t K, int64_t lda,
                          int64_t ldb, int64_t ldc, int32_t a_mn_major, int32_t b_mn_major, int test_stall,
                          cudaStream_t stream) {
  if (!A || !B || !C || M <= 0 || N <= 0 || K <= 0) return FLCE_ERR_INVALID_ARG;
  if (M >= (1ll << 31) || N >= (1ll << 31) || K >= (1ll << 31)) return FLCE_ERR_INVALID_ARG;
  if (lda % 8 || ldb % 8 || ldc % 4) return FLCE_ERR_INVALID_ARG;
  if (!is_aligned(A, 16) || !is_aligned(B, 16) || !is_aligned(C, 16)) return FLCE_ERR_INVALID_ARG;
  if (lda < (a_mn_major ? M : K) || ldb < (b_mn_major ? N : K) || ldc < N) return FLCE_ERR_INVALID_ARG;
  DeviceCtx* dev = nullptr;
  const flce_status st = device_ctx(&dev);
  if (st != FLCE_OK) return st;
  CUtensorMap ta, tb, z;
  std::memset(&z, 0, sizeof(z));
  const Engine eg = engine();
  const bool ok = (a_mn_major ? make_tmap(&ta, A, M, K, lda * 2, 64, 64) : make_tmap(&ta, A, K, M, lda * 2, 64, 128)) &&
                  (b_mn_major ? make_tmap(&tb, B, N, K, ldb * 2, 64, 64) : make_tmap(&tb, B, K, N, ldb * 2, 64, eg.b_box_rows));
  if (!ok) return FLCE_ERR_CUDA;
  TcParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.nprob = 1;
  prm.prob[0] = make_problem(eg, (int)M, (int)N, (int)K, a_mn_major ? 1 : 0, b_mn_major ? 1 : 0, EPI_STORE_F32, 1);
  prm.prob[0].out = C;
  prm.prob[0].ldo = ldc;
  prm.err = dev->err;
  prm.test_stall = test_stall;
  launch_tc(eg, ta, tb, z, z, prm, dev, stream);
  if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;
  if (env_debug() && cudaStreamSynchronize(stream) != cudaSuccess) return FLCE_ERR_CUDA;
  return FLCE_OK;
}

}  // namespace
}  // namespace flce

using namespace flce;

extern "C" {

void flce_options_init(flce_options* opt) {
  if (opt) std::memset(opt, 0, sizeof(*opt));
}

flce_status flce_fwd_bwd_ex(const flce_tensor* X, const flce_tensor* W, const flce_tensor* target,
                            int64_t ignore_index, int32_t reduction, flce_tensor* loss,
                            flce_tensor* grad_X, flce_tensor* grad_W, flce_stream_t stream,
                            const flce_options* opt, flce_stats* stats) {
  try {
    const NvtxRange range("flce_fwd_bwd");
    return run_flce(X, W, target, ignore_index, reduction, loss, grad_X, grad_W,
                    reinterpret_cast<cudaStream_t>(stream), opt, stats);
  } catch (...) {
    return FLCE_ERR_CUDA;
  }
}

flce_status flce_fwd_bwd(const flce_tensor* X, const flce_tensor* W, const flce_tensor* target,
                         int64_t ignore_index, int32_t reduction, flce_tensor* loss,
                         flce_tensor* grad_X, flce_tensor* grad_W, flce_stream_t stream) {
  return flce_fwd_bwd_ex(X, W, target, ignore_index, reduction, loss, grad_X, grad_W, stream,
                         nullptr, nullptr);
}

flce_status flce_plan(int64_t BT, int64_t H, int64_t V, int32_t dtype, int32_t want_grad_W,
                      const flce_options* opt, flce_stats* out) {
  if (!out) return FLCE_ERR_INVALID_ARG;
  Plan pl;
  const flce_status st = make_plan(BT, H, V, dtype, want_grad_W != 0, opt, !(opt && opt->row_loss), &pl);
  if (st != FLCE_OK) return st;
  std::memset(out, 0, sizeof(*out));
  out->chunk_rows = pl.chunk;
  out->n_chunks = pl.n_chunks;
  out->workspace_bytes = BT > 0 ? (int64_t)pl.total : 0;
  out->materialized_logits_bytes = BT * V * 2;
  out->path = dtype == FLCE_BF16 ? 1 : 0;
  return FLCE_OK;
}

size_t flce_workspace_bytes(int64_t BT, int64_t H, int64_t V, int32_t dtype, const flce_options* opt) {
  flce_stats st;
  if (flce_plan(BT, H, V, dtype, 1, opt, &st) != FLCE_OK) return (size_t)-1;
  return (size_t)st.workspace_bytes;
}

flce_status flce_count_valid(const flce_tensor* target, int64_t V, int64_t ignore_index,
                             int64_t* n_valid_out, flce_stream_t stream) {
  if (!target || !n_valid_out || V <= 0) return FLCE_ERR_INVALID_ARG;
  if (target->dtype != FLCE_I64 || target->ndim != 1 || target->shape[0] < 0) return FLCE_ERR_INVALID_ARG;
  const int64_t BT = target->shape[0];
  if (BT > 0 && (!target->data || target->stride[0] != 1)) return FLCE_ERR_INVALID_ARG;
  DeviceCtx* dev = nullptr;
  const flce_status st = device_ctx(&dev);
  if (st != FLCE_OK) return st;
  count_valid_kernel<<<1, 1024, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const int64_t*>(target->data), BT, V, ignore_index, n_valid_out, dev->err);
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

flce_status flce_cross_entropy(const flce_tensor* logits, const flce_tensor* target,
                               int64_t ignore_index, int32_t reduction, flce_tensor* loss,
                               flce_tensor* grad_logits, flce_stream_t stream,
                               const flce_options* opt) {
  try {
    const NvtxRange range("flce_cross_entropy");
    return run_ce(logits, target, ignore_index, reduction, loss, grad_logits,
                  reinterpret_cast<cudaStream_t>(stream), opt);
  } catch (...) {
    return FLCE_ERR_CUDA;
  }
}

flce_status flce_cross_entropy_noalloc(const flce_tensor* logits, const flce_tensor* target,
                                       int64_t ignore_index, int32_t reduction, flce_tensor* loss,
                                       flce_tensor* grad_logits, flce_stream_t stream) {
  try {
    return run_ce_noalloc(logits, target, ignore_index, reduction, loss, grad_logits,
                          reinterpret_cast<cudaStream_t>(stream));
  } catch (...) {
    return FLCE_ERR_CUDA;
  }
}

flce_status flce_gemm_bf16(const void* A, const void* B, float* C, int64_t M, int64_t N,
                           int64_t K, int64_t lda, int64_t ldb, int64_t ldc, int32_t a_mn_major,
                           int32_t b_mn_major, flce_stream_t stream) {
  return run_gemm_bf16(A, B, C, M, N, K, lda, ldb, ldc, a_mn_major, b_mn_major, 0,
                       reinterpret_cast<cudaStream_t>(stream));
}

flce_status flce_gemm_bf16_wait_test(const void* A, const void* B, float* C, int64_t M, int64_t N, int64_t K,
                                     int64_t lda, int64_t ldb, int64_t ldc, int32_t stall_tile,
                                     flce_stream_t stream) {
  if (stall_tile < 0) return FLCE_ERR_INVALID_ARG;
  if (!engine().pair) return FLCE_ERR_INVALID_ARG;  // the hook lives in the pair engine
  return run_gemm_bf16(A, B, C, M, N, K, lda, ldb, ldc, 0, 0, stall_tile + 1, reinterpret_cast<cudaStream_t>(stream));
}

flce_status flce_scale_grad(flce_tensor* t, const float* scale, flce_stream_t stream) {
  if (!t || !scale) return FLCE_ERR_INVALID_ARG;
  if (t->dtype != FLCE_BF16 && t->dtype != FLCE_F32) return FLCE_ERR_UNSUPPORTED_DTYPE;
  if (t->ndim < 0 || t->ndim > 2) return FLCE_ERR_INVALID_ARG;
  int64_t rows = 1, cols = 1, ld = 1;
  if (t->ndim == 1) {
    cols = t->shape[0];
    if (cols < 0 || (cols > 1 && t->stride[0] != 1)) return FLCE_ERR_INVALID_ARG;
    ld = cols;
  } else if (t->ndim == 2) {
    rows = t->shape[0];
    cols = t->shape[1];
    if (rows < 0 || cols < 0 || (cols > 1 && t->stride[1] != 1) || (rows > 1 && t->stride[0] < cols))
      return FLCE_ERR_INVALID_ARG;
    ld = rows > 1 ? t->stride[0] : cols;
  }
  if (rows == 0 || cols == 0) return FLCE_OK;
  if (!t->data) return FLCE_ERR_INVALID_ARG;
  DeviceCtx* dev = nullptr;
  const flce_status st = device_ctx(&dev);
  if (st != FLCE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int esz = dtype_size(t->dtype);
  const int vec = 16 / esz;
  const bool vector = cols % vec == 0 && ld % vec == 0 && is_aligned(t->data, 16);
  const int64_t units = rows * (vector ? cols / vec : cols);
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(units, 256), 8ll * dev->sms));
  if (t->dtype == FLCE_BF16) {
    __nv_bfloat16* p = static_cast<__nv_bfloat16*>(t->data);
    if (vector) scale_grad_kernel<__nv_bfloat16, 8><<<blocks, 256, 0, s>>>(p, rows, cols, ld, scale);
    else scale_grad_kernel<__nv_bfloat16, 1><<<blocks, 256, 0, s>>>(p, rows, cols, ld, scale);
  } else {
    float* p = static_cast<float*>(t->data);
    if (vector) scale_grad_kernel<float, 4><<<blocks, 256, 0, s>>>(p, rows, cols, ld, scale);
    else scale_grad_kernel<float, 1><<<blocks, 256, 0, s>>>(p, rows, cols, ld, scale);
  }
  if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;
  if (env_debug() && cudaStreamSynchronize(s) != cudaSuccess) return FLCE_ERR_CUDA;
  return FLCE_OK;
}

flce_status flce_get_device_error(flce_stream_t stream, uint32_t* err) {
  if (!err) return FLCE_ERR_INVALID_ARG;
  DeviceCtx* dev = nullptr;
  const flce_status st = device_ctx(&dev);
  if (st != FLCE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FLCE_ERR_CUDA;
  if (cudaMemcpy(err, dev->err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return FLCE_ERR_CUDA;
  if (cudaMemset(dev->err, 0, 4) != cudaSuccess) return FLCE_ERR_CUDA;
  return FLCE_OK;
}

flce_status flce_phase_times(double* ms, int32_t* count, int32_t n_phases, int32_t reset) {
  if (n_phases < 0) return FLCE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  for (int p = 0; p < n_phases; ++p) {
    if (ms) ms[p] = 0.0;
    if (count) count[p] = 0;
  }
  for (const PhaseRec& r : g_phase_recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) return FLCE_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) return FLCE_ERR_CUDA;
    if (r.phase < n_phases) {
      if (ms) ms[r.phase] += t;
      if (count) count[r.phase] += 1;
    }
  }
  if (reset) {
    for (const PhaseRec& r : g_phase_recs) {
      g_event_pool.push_back(r.a);
      g_event_pool.push_back(r.b);
    }
    g_phase_recs.clear();
  }
  return FLCE_OK;
}

const char* flce_status_string(int32_t s) {
  switch (s) {
    case FLCE_OK: return "ok";
    case FLCE_ERR_INVALID_ARG: return "invalid argument";
    case FLCE_ERR_UNSUPPORTED_DTYPE: return "unsupported dtype";
    case FLCE_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs sm_100)";
    case FLCE_ERR_ALLOC: return "workspace allocation failed";
    case FLCE_ERR_CUDA: return "CUDA error";
    case FLCE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    default: return "unknown status";
  }
}

int32_t flce_version(void) { return FLCE_VERSION; }

}  // extern "C"
