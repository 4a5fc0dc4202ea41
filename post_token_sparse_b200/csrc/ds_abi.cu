// C ABI of libds.so: argument checks, launch configuration and launches.
//
// All kernels live in this one translation unit (no relocatable device code).
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "ds.h"

#include "attend.cuh"
#include "attend_group.cuh"
#include "calib.cuh"
#include "common.cuh"
#include "label.cuh"
#include "score.cuh"
#include "step.cuh"
#include "select.cuh"
#include "topk.cuh"

namespace {

using namespace ds;

std::atomic<uint64_t> g_launches{0};

// One NVTX range per C-ABI call (visible in Nsight timelines; a no-op when no
// tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
#define DS_TRACE(name) NvtxRange ds_nvtx_range_(name)
thread_local char g_cuda_err[256] = "no error";

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// K and V may be device memory or page-locked host memory mapped into the
// device's address space (the KV cache offloaded to the host; kernels then
// read the rows they need over the host link).  Any other host memory is
// refused before a launch could touch it.  When the runtime cannot be asked
// (no device), the launch itself reports the error.  *device (optional): p is
// plain device memory.
ds_status check_kv_ptr(const void* p, bool* device = nullptr) {
  if (device) *device = false;
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return DS_OK;
  }
  if (device) *device = a.type == cudaMemoryTypeDevice;
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return DS_OK;
  if (a.type == cudaMemoryTypeHost && a.devicePointer == p) return DS_OK;
  return DS_ERR_INVALID_ARG;
}

// *device (optional): K and V are both plain device memory.
ds_status check_kv(const void* K, const void* V, bool* device = nullptr) {
  bool dk = false, dv = true;
  ds_status s = check_kv_ptr(K, &dk);
  if (s == DS_OK && V != nullptr) s = check_kv_ptr(V, &dv);
  if (device) *device = dk && dv;
  return s;
}

// ds_decode_step also takes its query and its outputs in mapped host memory:
// the step's input and result then cross the host link inside the kernel.
ds_status check_io(const void* Q, const void* O, const void* lse) {
  ds_status s = check_kv(Q, O);
  return s != DS_OK || lse == nullptr ? s : check_kv_ptr(lse);
}

ds_status cuda_fail(cudaError_t e) {
  std::snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return DS_ERR_CUDA;
}

// Call after each launch.
ds_status launched() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DS_OK : cuda_fail(e);
}

ds_status check_dims(const ds_dims& d) {
  if (d.B < 1 || d.Hq < 1 || d.Hkv < 1 || d.T_cap < 1 || d.r < 1 || d.d < 1)
    return DS_ERR_INVALID_ARG;
  if (d.Hq % d.Hkv != 0) return DS_ERR_INVALID_ARG;
  if (d.r > d.d) return DS_ERR_INVALID_ARG;
  if (d.d != kHeadDim) return DS_ERR_UNSUPPORTED;
  // grid-dimension limits of the launches below
  if ((int64_t)d.B * d.Hq > 65535 || (int64_t)d.B * d.Hkv > 65535) return DS_ERR_UNSUPPORTED;
  return DS_OK;
}

// ---- attention work plan (device independent) -------------------------------
// attn_plan (attend.cuh): every warp of one wave takes an equal, contiguous
// range of the heads' rows; the workspace holds the arrival counters at a
// fixed place, then the partials of the heads that several warps share.
size_t attend_ws_bytes(int heads, int rows) { return attn_workspace_bytes(attn_plan(heads, rows)); }

// Attention over rows shared by a whole group of query heads (all T tokens, or
// a group-shared token set) runs group by group (k_attend_group) when a KV head
// has 2..8 query heads, else head by head.
bool group_kernel_applies(const ds_dims& d) {
  const int G = d.Hq / d.Hkv;
  return G >= 2 && G <= kGrpMaxG;
}
// workspace of an attention call whose rows are shared by each group
size_t shared_rows_ws_bytes(const ds_dims& d, int rows) {
  if (group_kernel_applies(d)) return grp_workspace_bytes(grp_plan(d.B * d.Hkv, rows));
  return attend_ws_bytes(d.B * d.Hq, rows);
}

// ---- per-device one-time kernel attributes ----------------------------------
constexpr int kMaxDevices = 64;
std::once_flag g_attr_once[kMaxDevices];
cudaError_t g_attr_err[kMaxDevices];


template <class Kern>
cudaError_t allow_smem(Kern k, size_t bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <class Src>
cudaError_t topk_attrs() {
  cudaError_t e = allow_smem(k_topk<Src>, TopkLayout(kMaxKeysPerCta, kMaxCluster).bytes());
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_topk<Src>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
}

ds_status ensure_attrs() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return DS_ERR_UNSUPPORTED;
  std::call_once(g_attr_once[dev], [dev] {
    cudaError_t r = cudaSuccess;
    auto acc = [&r](cudaError_t x) {
      if (r == cudaSuccess) r = x;
    };
    acc(allow_smem(k_attend<true>, kAttnSmemBytes));
    acc(allow_smem(k_attend<false>, kAttnSmemBytes));
    acc(allow_smem(k_attend_group<true>, kGrpSmemBytes));
    acc(allow_smem(k_attend_group<false>, kGrpSmemBytes));
    acc(topk_attrs<ScoresSource>());
    acc(topk_attrs<LabelSource<8>>());
    acc(topk_attrs<LabelSource<16>>());
    acc(topk_attrs<LabelSource<32>>());
    acc(topk_attrs<LabelSource<64>>());
    acc(topk_attrs<LabelSource<128>>());
    const size_t hier_max = HierLayout(TopkLayout(2 * kHierMaxK, 1)).bytes();
    acc(allow_smem(k_hier_topk<LabelSource<8>>, hier_max));
    acc(allow_smem(k_hier_topk<LabelSource<16>>, hier_max));
    acc(allow_smem(k_hier_topk<LabelSource<32>>, hier_max));
    acc(allow_smem(k_hier_topk<LabelSource<64>>, hier_max));
    acc(allow_smem(k_hier_topk<LabelSource<128>>, hier_max));
    const size_t step_max = 227 * 1024;
    acc(allow_smem(k_step<8>, step_max));
    acc(allow_smem(k_step<16>, step_max));
    acc(allow_smem(k_step<32>, step_max));
    acc(allow_smem(k_step<64>, step_max));
    acc(allow_smem(k_step<128>, step_max));
    g_attr_err[dev] = r;
  });
  return g_attr_err[dev] == cudaSuccess ? DS_OK : cuda_fail(g_attr_err[dev]);
}

// ---- top-k launch -----------------------------------------------------------
struct TopkPlan {
  int cs;
  int chunk;
};

// A head of at most kSample tokens is one CTA (it computes every key of the
// head anyway).  Longer heads are cut so that one CTA's expected number of
// candidates -- the tokens inside the sample bracket -- stays near half its
// list, and, with few heads, further (down to kTopkMinKeys tokens per CTA):
// into the largest cluster size of which every head's cluster runs at once.
constexpr int kTopkMinKeys = 2048;
// Clusters of each size that run at once on B200 at three selection CTAs per
// SM (cudaOccupancyMaxActiveClusters: clusters are placed whole inside a GPC,
// so large clusters pack worse).  Spreading uses these sizes only.
constexpr int kSpreadSizes[] = {16, 14, 12, 10, 8, 6, 4, 2};
constexpr int kActiveClusters[] = {21, 24, 31, 41, 48, 71, 104, 222};

bool plan_topk(int BH, int T, int k, TopkPlan* out) {
  int cs = (T + kMaxKeysPerCta - 1) / kMaxKeysPerCta;
  if (cs > kMaxCluster) return false;
  if (T > kSample) {
    const double p = (double)k / T, e = p * kSample;
    const double frac = 2.0 * (kBracketSigmas * std::sqrt(e * (1.0 - p)) + 3.0) / kSample;
    const double max_chunk = 0.5 * kCandCap / std::max(frac, 1e-9);
    cs = std::max(cs, (int)std::min<double>(kMaxCluster, std::ceil(T / max_chunk)));
    for (int i = 0; i < 8; ++i) {
      const int c = kSpreadSizes[i];
      if (c > cs && c <= T / kTopkMinKeys && BH <= kActiveClusters[i]) {
        cs = c;
        break;
      }
    }
  }
  int chunk = (T + cs - 1) / cs;
  chunk = (chunk + 31) & ~31;
  cs = (T + chunk - 1) / chunk;
  out->cs = cs;
  out->chunk = chunk;
  return true;
}

template <class Src>
ds_status launch_topk(const Src& src, int32_t* idx, int BH, int T, int k, cudaStream_t st) {
  TopkPlan tp;
  if (!plan_topk(BH, T, k, &tp)) return DS_ERR_UNSUPPORTED;
  const size_t smem = TopkLayout(tp.chunk, tp.cs).bytes();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tp.cs, BH, 1);
  cfg.blockDim = dim3(kTopkThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = tp.cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = tp.cs > 1 ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_topk<Src>, src, idx, T, k, tp.chunk);
  if (e != cudaSuccess) return cuda_fail(e);
  return launched();
}

ds_status launch_score(const uint16_t* Q, const int32_t* C, const uint16_t* label, float* scores,
                       const ds_dims& d, int T, cudaStream_t st) {
  const int BH = d.B * d.Hq;
  auto vec = [&](auto kern, int tokens_per_cta) {
    dim3 grid((T + tokens_per_cta - 1) / tokens_per_cta, BH);
    kern<<<grid, kScoreThreads, 0, st>>>(Q, C, label, scores, d.Hq, d.T_cap, T);
    return launched();
  };
  switch (d.r) {
    case 8: return vec(k_score_vec<8>, ScoreShape<8>::kTokensPerCta);
    case 16: return vec(k_score_vec<16>, ScoreShape<16>::kTokensPerCta);
    case 32: return vec(k_score_vec<32>, ScoreShape<32>::kTokensPerCta);
    case 64: return vec(k_score_vec<64>, ScoreShape<64>::kTokensPerCta);
    case 128: return vec(k_score_vec<128>, ScoreShape<128>::kTokensPerCta);
    default: {
      dim3 grid((T + kScoreThreads - 1) / kScoreThreads, BH);
      k_score_any<<<grid, kScoreThreads, 0, st>>>(Q, C, label, scores, d.Hq, d.T_cap, T, d.r);
      return launched();
    }
  }
}

template <int R>
ds_status fused_topk(const uint16_t* Q, const int32_t* C, const uint16_t* label, float* scores,
                     int32_t* idx, const ds_dims& d, int T, int k, cudaStream_t st) {
  LabelSource<R> src{Q, C, label, scores, d.Hq, d.T_cap};
  return launch_topk(src, idx, d.B * d.Hq, T, k, st);
}

// One-launch selection with a prefix workspace (select.cuh): r with a vector
// path and 4096 < T <= 32768 (shorter heads are one k_topk CTA each).
bool sel_applies(int r, int T) {
  return (r == 8 || r == 16 || r == 32 || r == 64 || r == 128) && T > kSample && T <= kSelMaxT;
}

template <int R>
ds_status launch_sel(const uint16_t* Q, const int32_t* C, const uint16_t* label, float* scores,
                     int32_t* idx, const ds_dims& d, int T, int k, void* ws, cudaStream_t st) {
  SelParams sp;
  sp.Q = Q;
  sp.C = C;
  sp.label = label;
  sp.scores = scores;
  sp.idx = idx;
  sp.arrivals = static_cast<uint32_t*>(ws);
  sp.prefixes = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + kCounterBytes);
  sp.BH = d.B * d.Hq;
  sp.Hq = d.Hq;
  sp.T_cap = d.T_cap;
  sp.T = T;
  sp.k = k;
  dim3 grid((T + kSelTile - 1) / kSelTile, sp.BH);
  k_score_select<R><<<grid, kSelThreads, 0, st>>>(sp);
  return launched();
}

// One-launch top-k over written scores (k_scores_select) for heads of
// 4096 < T <= 16384 given a workspace of sel_ws_bytes(BH, T).  Measured against
// the plain selection: 39.0 -> 33.9 us (128 rows of 16384), 41.1 -> 28.7 us
// (256 of 8192); at 32768 tokens a row no faster (1024 rows) or slower (64).
bool scores_sel_applies(int T) { return T > kSample && T <= 16384; }

ds_status launch_scores_sel(const float* scores, int32_t* idx, int BH, int T, int k, void* ws,
                            cudaStream_t st) {
  SelParams sp = {};
  sp.scores = const_cast<float*>(scores);
  sp.idx = idx;
  sp.arrivals = static_cast<uint32_t*>(ws);
  sp.prefixes = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + kCounterBytes);
  sp.BH = BH;
  sp.T = T;
  sp.k = k;
  dim3 grid((T + kScoresTile - 1) / kScoresTile, BH);
  k_scores_select<<<grid, kSelThreads, 0, st>>>(sp);
  return launched();
}

// Top-k over written scores: one launch when a large enough workspace is given.
ds_status topk_scores(const float* scores, int32_t* idx, int BH, int T, int k, void* ws,
                      size_t ws_bytes, cudaStream_t st) {
  if (scores_sel_applies(T) && ws && aligned16(ws) && ws_bytes >= sel_ws_bytes(BH, T))
    return launch_scores_sel(scores, idx, BH, T, k, ws, st);
  return launch_topk(ScoresSource{scores}, idx, BH, T, k, st);
}

// Workspace of ds_group_decode_step: the attention's, then (when the one-launch
// selection applies) the selection's, 256-byte aligned.  *sel_off: its offset
// (0: none).
size_t group_step_ws(const ds_dims& d, int T, int k, size_t* sel_off) {
  size_t n = shared_rows_ws_bytes(d, k);
  size_t off = 0;
  if (scores_sel_applies(T)) {
    off = (n + 255) & ~(size_t)255;
    n = off + sel_ws_bytes(d.B * d.Hkv, T);
  }
  if (sel_off) *sel_off = off;
  return n;
}

ds_status score_select(const uint16_t* Q, const int32_t* C, const uint16_t* label, float* scores,
                       int32_t* idx, const ds_dims& d, int T, int k, void* ws, cudaStream_t st) {
  switch (d.r) {
    case 8: return launch_sel<8>(Q, C, label, scores, idx, d, T, k, ws, st);
    case 16: return launch_sel<16>(Q, C, label, scores, idx, d, T, k, ws, st);
    case 32: return launch_sel<32>(Q, C, label, scores, idx, d, T, k, ws, st);
    case 64: return launch_sel<64>(Q, C, label, scores, idx, d, T, k, ws, st);
    default: return launch_sel<128>(Q, C, label, scores, idx, d, T, k, ws, st);
  }
}

// Host-side check of the workspace (no CUDA calls).
ds_status check_attend_ws(const ds_dims& d, int rows, const void* ws, size_t ws_bytes) {
  const size_t need = attend_ws_bytes(d.B * d.Hq, rows);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws))) return DS_ERR_WORKSPACE;
  return DS_OK;
}

// Host-side check of the workspace of a call whose rows each group shares.
ds_status check_shared_rows_ws(const ds_dims& d, int rows, const void* ws, size_t ws_bytes) {
  const size_t need = shared_rows_ws_bytes(d, rows);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws))) return DS_ERR_WORKSPACE;
  return DS_OK;
}

// Group-by-group attention (group_kernel_applies): idx [B*Hkv, rows] shared
// token ids, or null for all T tokens.
ds_status launch_attend_group(const ds_dims& d, const void* Q, const void* K, const void* V,
                              const int32_t* idx, float* O, float* lse, int T, int rows,
                              float scale, void* ws, cudaStream_t st) {
  const int groups = d.B * d.Hkv;
  const AttnPlan pl = grp_plan(groups, rows);
  GrpParams p;
  p.Q = static_cast<const uint16_t*>(Q);
  p.K = static_cast<const uint16_t*>(K);
  p.V = static_cast<const uint16_t*>(V);
  p.idx = idx;
  p.O = O;
  p.lse = lse;
  p.arrivals = pl.slots ? static_cast<uint32_t*>(ws) : nullptr;
  p.partial = pl.slots ? reinterpret_cast<float*>(static_cast<char*>(ws) + kCounterBytes)
                       : nullptr;
  p.groups = groups;
  p.G = d.Hq / d.Hkv;
  p.Hq = d.Hq;
  p.Hkv = d.Hkv;
  p.T_cap = d.T_cap;
  p.T = T;
  p.rows = rows;
  p.per = pl.per;
  p.units = pl.units;
  p.scale_log2 = scale * 1.4426950408889634f;
  const int grid = (pl.units + kGrpWarps - 1) / kGrpWarps;
  if (idx)
    k_attend_group<true><<<grid, kGrpThreads, kGrpSmemBytes, st>>>(p);
  else
    k_attend_group<false><<<grid, kGrpThreads, kGrpSmemBytes, st>>>(p);
  return launched();
}

ds_status launch_attend(const ds_dims& d, const void* Q, const void* K, const void* V,
                        const int32_t* idx, float* O, float* lse, int T, int rows, float scale,
                        void* ws, cudaStream_t st, bool idx_per_group = false,
                        int block = 0) {
  const bool sparse = idx != nullptr;
  const int heads = d.B * d.Hq;
  const AttnPlan pl = attn_plan(heads, rows);

  AttnParams p;
  p.Q = static_cast<const uint16_t*>(Q);
  p.K = static_cast<const uint16_t*>(K);
  p.V = static_cast<const uint16_t*>(V);
  p.idx = idx;
  p.idx_per_group = idx_per_group ? 1 : 0;
  p.block = block;
  p.O = O;
  p.lse = lse;
  p.arrivals = pl.slots ? static_cast<uint32_t*>(ws) : nullptr;
  p.partial = pl.slots ? reinterpret_cast<float*>(static_cast<char*>(ws) + kCounterBytes)
                       : nullptr;
  p.heads = heads;
  p.Hq = d.Hq;
  p.Hkv = d.Hkv;
  p.T_cap = d.T_cap;
  p.T = T;
  p.rows = rows;
  p.per = pl.per;
  p.units = pl.units;
  p.scale_log2 = scale * 1.4426950408889634f;

  const int grid = (pl.units + kAttnWarps - 1) / kAttnWarps;
  if (sparse)
    k_attend<true><<<grid, kAttnThreads, kAttnSmemBytes, st>>>(p);
  else
    k_attend<false><<<grid, kAttnThreads, kAttnSmemBytes, st>>>(p);
  return launched();
}

// The fused step applies when r has a vector path, the head's selection fits
// one CTA, k is small enough for its index list to stay in shared memory, and
// the whole layout fits a CTA's shared memory.  Depends only on the sizes.
// Selection from the label cache: one fused launch (scores computed while
// selecting), or, for r >= 16 on heads longer than one sample, the scores
// written first and the selection run over them.  The second needs a score
// buffer but measured faster there: the score kernel streams the labels once
// at full rate, and the selection's passes then read 4 bytes a token.
bool prefer_score_then_select(int r, int T) { return r >= 16 && T > kSample; }

// The one-launch step runs every head's whole chain in one CTA at two CTAs per
// SM.  That pays while all heads fit one wave; with more heads the separate
// kernels (three top-k CTAs and six attention CTAs per SM) hide each other's
// latency better, so the step falls back to them.
constexpr int kStepMaxHeads = 2 * 148;

bool step_fused(const ds_dims& d, int T, int k, int* chunk_out, size_t* smem_out) {
  const int r = d.r;
  if (!(r == 8 || r == 16 || r == 32 || r == 64 || r == 128)) return false;
  if (k > kStepMaxK) return false;
  if (d.B * d.Hq > kStepMaxHeads) return false;
  TopkPlan tp;
  if (!plan_topk(d.B * d.Hq, T, k, &tp) || tp.cs != 1) return false;
  const size_t smem = StepLayout(tp.chunk, k).bytes();
  if (smem > 227 * 1024) return false;
  *chunk_out = tp.chunk;
  *smem_out = smem;
  return true;
}

// Workspace of the separate-kernels step: the attention's counters and
// partials, then the selection's workspace (one-launch selection) or, when the
// selection runs over written scores, [BH, T] fp32 scores.  Returns the total;
// *sel_off gets the offset of the second part (0: none).
size_t step_fallback_ws(const ds_dims& d, int T, int k, size_t* sel_off) {
  const int BH = d.B * d.Hq;
  size_t n = attend_ws_bytes(BH, k);
  size_t off = 0;
  if (sel_applies(d.r, T)) {
    off = (n + 255) & ~(size_t)255;
    n = off + sel_ws_bytes(BH, T);
  } else if (prefer_score_then_select(d.r, T)) {
    off = (n + 255) & ~(size_t)255;
    n = off + (((size_t)BH * T * sizeof(float) + 255) & ~(size_t)255);
  }
  if (sel_off) *sel_off = off;
  return n;
}

template <int R>
ds_status launch_step(const StepParams& sp, int BH, int chunk, size_t smem, cudaStream_t st) {
  k_step<R><<<BH, kTopkThreads, smem, st>>>(sp, chunk);
  return launched();
}

}  // namespace

extern "C" {

const char* ds_status_string(ds_status s) {
  switch (s) {
    case DS_OK: return "DS_OK";
    case DS_ERR_INVALID_ARG: return "DS_ERR_INVALID_ARG";
    case DS_ERR_UNSUPPORTED: return "DS_ERR_UNSUPPORTED";
    case DS_ERR_WORKSPACE: return "DS_ERR_WORKSPACE";
    case DS_ERR_CUDA: return "DS_ERR_CUDA";
  }
  return "DS_ERR_UNKNOWN";
}

const char* ds_last_cuda_error(void) { return g_cuda_err; }

uint64_t ds_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

size_t ds_workspace_size(int32_t op, ds_dims dims, int32_t T, int32_t k) {
  if (check_dims(dims) != DS_OK || T < 1 || T > dims.T_cap) return 0;
  const int BH = dims.B * dims.Hq;
  switch (op) {
    case DS_OP_SPARSE_DECODE:
      if (k < 1 || k > T) return 0;
      return attend_ws_bytes(BH, k);
    case DS_OP_DECODE:
      return shared_rows_ws_bytes(dims, T);
    case DS_OP_SCORE_TOPK:
      if (k < 1 || k > T) return 0;
      return sel_applies(dims.r, T) ? sel_ws_bytes(BH, T) : 0;
    case DS_OP_DECODE_STEP: {
      if (k < 1 || k > T) return 0;
      int chunk;
      size_t smem;
      if (step_fused(dims, T, k, &chunk, &smem)) return 0;
      return step_fallback_ws(dims, T, k, nullptr);
    }
    case DS_OP_BLOCK_SPARSE_DECODE:  // k: kept rows, blocks x block size
      if (k < 1) return 0;
      return attend_ws_bytes(BH, k);
    case DS_OP_GROUP_SPARSE_DECODE:
      if (k < 1 || k > T) return 0;
      return shared_rows_ws_bytes(dims, k);
    case DS_OP_TOPK:
      if (k < 1 || k > T) return 0;
      return scores_sel_applies(T) ? sel_ws_bytes(BH, T) : 0;
    case DS_OP_GROUP_DECODE_STEP:
      if (k < 1 || k > T) return 0;
      return group_step_ws(dims, T, k, nullptr);
    case DS_OP_CALIBRATE: {
      if (k < 1) return 0;  // k: calibration queries per head
      const size_t nck = (T + kAbsumRows - 1) / kAbsumRows, ncq = (k + kAbsumRows - 1) / kAbsumRows;
      const size_t bytes = ((size_t)dims.B * dims.Hkv * nck + (size_t)BH * ncq) * kHeadDim * 4;
      return (bytes + 255) & ~(size_t)255;
    }
    default:
      return 0;
  }
}

ds_status ds_device_status(uint32_t* bits, int32_t clear, ds_stream_t stream) {
  DS_TRACE("ds_device_status");
  if (!bits) return DS_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e);
  if (clear) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_status, &z, sizeof(z));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  *bits = v;
  return DS_OK;
}

ds_status ds_label_append(const void* K, const int32_t* C, void* label, ds_dims dims, int32_t t0,
                          int32_t n, ds_stream_t stream) {
  DS_TRACE("ds_label_append");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!K || !C || !label || !aligned16(K) || !aligned16(C) || !aligned16(label))
    return DS_ERR_INVALID_ARG;
  if (t0 < 0 || n < 1 || (int64_t)t0 + n > dims.T_cap) return DS_ERR_INVALID_ARG;
  const int G = dims.Hq / dims.Hkv;
  const size_t cs_bytes = (size_t)G * dims.r * sizeof(int32_t);
  if (cs_bytes > 40 * 1024) return DS_ERR_UNSUPPORTED;
  s = check_kv(K, nullptr);
  if (s != DS_OK) return s;
  dim3 grid((n + kLabelTile - 1) / kLabelTile, dims.B * dims.Hkv);
  k_label_append<<<grid, kLabelThreads, cs_bytes, stream>>>(
      static_cast<const uint16_t*>(K), C, static_cast<uint16_t*>(label), dims.Hq, dims.Hkv,
      dims.T_cap, dims.r, t0, n);
  return launched();
}

ds_status ds_score(const void* Q, const int32_t* C, const void* label, float* scores,
                   ds_dims dims, int32_t T, ds_stream_t stream) {
  DS_TRACE("ds_score");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!Q || !C || !label || !scores || !aligned16(Q) || !aligned16(C) || !aligned16(label) ||
      !aligned16(scores))
    return DS_ERR_INVALID_ARG;
  if (T < 1 || T > dims.T_cap) return DS_ERR_INVALID_ARG;
  return launch_score(static_cast<const uint16_t*>(Q), C, static_cast<const uint16_t*>(label),
                      scores, dims, T, stream);
}

ds_status ds_topk(const float* scores, int32_t* idx, int32_t BH, int32_t T, int32_t k, void* ws,
                  size_t ws_bytes, ds_stream_t stream) {
  DS_TRACE("ds_topk");
  if (!scores || !idx || !aligned16(scores) || !aligned16(idx)) return DS_ERR_INVALID_ARG;
  if (BH < 1 || T < 1 || k < 1 || k > T) return DS_ERR_INVALID_ARG;
  if (BH > 65535 || T > kMaxCluster * kMaxKeysPerCta) return DS_ERR_UNSUPPORTED;
  ds_status s = ensure_attrs();
  if (s != DS_OK) return s;
  return topk_scores(scores, idx, BH, T, k, ws, ws_bytes, stream);
}

ds_status ds_score_topk(const void* Q, const int32_t* C, const void* label, float* scores,
                        int32_t* idx, ds_dims dims, int32_t T, int32_t k, void* ws,
                        size_t ws_bytes, ds_stream_t stream) {
  DS_TRACE("ds_score_topk");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!Q || !C || !label || !idx || !aligned16(Q) || !aligned16(C) || !aligned16(label) ||
      !aligned16(idx) || (scores && !aligned16(scores)))
    return DS_ERR_INVALID_ARG;
  if (T < 1 || T > dims.T_cap || k < 1 || k > T) return DS_ERR_INVALID_ARG;
  if (T > kMaxCluster * kMaxKeysPerCta) return DS_ERR_UNSUPPORTED;
  const bool fused = dims.r == 8 || dims.r == 16 || dims.r == 32 || dims.r == 64 || dims.r == 128;
  if (!fused && !scores) return DS_ERR_UNSUPPORTED;
  s = ensure_attrs();
  if (s != DS_OK) return s;
  auto Qb = static_cast<const uint16_t*>(Q);
  auto Lb = static_cast<const uint16_t*>(label);
  if (sel_applies(dims.r, T) && ws && aligned16(ws) &&
      ws_bytes >= sel_ws_bytes(dims.B * dims.Hq, T))
    return score_select(Qb, C, Lb, scores, idx, dims, T, k, ws, stream);
  if (scores && prefer_score_then_select(dims.r, T)) {
    s = launch_score(Qb, C, Lb, scores, dims, T, stream);
    if (s != DS_OK) return s;
    return launch_topk(ScoresSource{scores}, idx, dims.B * dims.Hq, T, k, stream);
  }
  switch (dims.r) {
    case 8: return fused_topk<8>(Qb, C, Lb, scores, idx, dims, T, k, stream);
    case 16: return fused_topk<16>(Qb, C, Lb, scores, idx, dims, T, k, stream);
    case 32: return fused_topk<32>(Qb, C, Lb, scores, idx, dims, T, k, stream);
    case 64: return fused_topk<64>(Qb, C, Lb, scores, idx, dims, T, k, stream);
    case 128: return fused_topk<128>(Qb, C, Lb, scores, idx, dims, T, k, stream);
    default:
      // other r: two launches through the caller's score buffer
      s = launch_score(Qb, C, Lb, scores, dims, T, stream);
      if (s != DS_OK) return s;
      return launch_topk(ScoresSource{scores}, idx, dims.B * dims.Hq, T, k, stream);
  }
}

ds_status ds_sparse_decode(const void* Q, const void* K, const void* V, const int32_t* idx,
                           float* O, float* lse, ds_dims dims, int32_t T, int32_t k, float scale,
                           void* ws, size_t ws_bytes, ds_stream_t stream) {
  DS_TRACE("ds_sparse_decode");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!Q || !K || !V || !idx || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) ||
      !aligned16(idx) || !aligned16(O) || (lse && !aligned16(lse)))
    return DS_ERR_INVALID_ARG;
  if (T < 1 || T > dims.T_cap || k < 1 || k > T) return DS_ERR_INVALID_ARG;
  s = check_attend_ws(dims, k, ws, ws_bytes);
  if (s != DS_OK) return s;
  s = check_kv(K, V);
  if (s != DS_OK) return s;
  s = ensure_attrs();
  if (s != DS_OK) return s;
  return launch_attend(dims, Q, K, V, idx, O, lse, T, k, scale, ws, stream);
}

ds_status ds_decode(const void* Q, const void* K, const void* V, float* O, float* lse,
                    ds_dims dims, int32_t T, float scale, void* ws, size_t ws_bytes,
                    ds_stream_t stream) {
  DS_TRACE("ds_decode");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!Q || !K || !V || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) ||
      !aligned16(O) || (lse && !aligned16(lse)))
    return DS_ERR_INVALID_ARG;
  if (T < 1 || T > dims.T_cap) return DS_ERR_INVALID_ARG;
  s = check_shared_rows_ws(dims, T, ws, ws_bytes);
  if (s != DS_OK) return s;
  s = check_kv(K, V);
  if (s != DS_OK) return s;
  s = ensure_attrs();
  if (s != DS_OK) return s;
  if (group_kernel_applies(dims))
    return launch_attend_group(dims, Q, K, V, nullptr, O, lse, T, T, scale, ws, stream);
  return launch_attend(dims, Q, K, V, nullptr, O, lse, T, T, scale, ws, stream);
}

}  // extern "C"

// ---- sparse decode with library-owned scratch ---------------------------------
// For callers that must not allocate device memory: the workspace of
// ds_sparse_decode -- arrival counters at its start, then the split partials --
// lives in this fixed file-scope array instead.  It is zero when the library is
// loaded and every call leaves its counters at zero, so no call has to clear
// anything first.  Every call on a device shares it, so calls that overlap on
// the GPU race on it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DS_NOALLOC_SCRATCH_BYTES];
static_assert(kCounterBytes < DS_NOALLOC_SCRATCH_BYTES, "the counters fit the scratch array");

namespace {
std::once_flag g_scratch_once[kMaxDevices];
std::atomic<void*> g_scratch_addr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a host-side handle, so the address is looked up once
// per device, with that device current.
ds_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return DS_ERR_UNSUPPORTED;
  void* a = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (a == nullptr) {
    std::call_once(g_scratch_once[dev], [dev] {
      void* p = nullptr;
      g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (g_scratch_err[dev] == cudaSuccess) g_scratch_addr[dev].store(p, std::memory_order_release);
    });
    if (g_scratch_err[dev] != cudaSuccess) return cuda_fail(g_scratch_err[dev]);
    a = g_scratch_addr[dev].load(std::memory_order_acquire);
  }
  *out = a;
  return DS_OK;
}
}  // namespace

extern "C" ds_status ds_sparse_decode_noalloc(const void* Q, const void* K, const void* V,
                                              const int32_t* idx, float* O, float* lse,
                                              ds_dims dims, int32_t T, int32_t k, float scale,
                                              ds_stream_t stream) {
  DS_TRACE("ds_sparse_decode_noalloc");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!Q || !K || !V || !idx || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) ||
      !aligned16(idx) || !aligned16(O) || (lse && !aligned16(lse)))
    return DS_ERR_INVALID_ARG;
  if (T < 1 || T > dims.T_cap || k < 1 || k > T) return DS_ERR_INVALID_ARG;
  const size_t need = attend_ws_bytes(dims.B * dims.Hq, k);
  if (need > DS_NOALLOC_SCRATCH_BYTES) return DS_ERR_WORKSPACE;
  s = check_kv(K, V);
  if (s != DS_OK) return s;
  s = ensure_attrs();
  if (s != DS_OK) return s;
  void* scratch = nullptr;
  if (need > 0) {
    s = noalloc_scratch(&scratch);
    if (s != DS_OK) return s;
  }
  return launch_attend(dims, Q, K, V, idx, O, lse, T, k, scale, scratch, stream);
}

namespace {

// ds_decode_step, and ds_decode_step_kv when K_new is given (then append is 1).
ds_status decode_step(const void* Q, const void* K_new, const void* V_new, const void* K,
                      const void* V, const int32_t* C, void* label, int32_t* idx, float* O,
                      float* lse, ds_dims dims, int32_t T, int32_t k, float scale,
                      int32_t append, void* ws, size_t ws_bytes, ds_stream_t stream) {
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!Q || !K || !V || !C || !label || !idx || !O || !aligned16(Q) || !aligned16(K) ||
      !aligned16(V) || !aligned16(C) || !aligned16(label) || !aligned16(idx) || !aligned16(O) ||
      (lse && !aligned16(lse)))
    return DS_ERR_INVALID_ARG;
  if (T < 1 || T > dims.T_cap || k < 1 || k > T) return DS_ERR_INVALID_ARG;
  if (K_new) {
    if (!V_new || !aligned16(K_new) || !aligned16(V_new)) return DS_ERR_INVALID_ARG;
    s = check_kv(K_new, V_new);
    if (s != DS_OK) return s;
  }
  if (T > kMaxCluster * kMaxKeysPerCta) return DS_ERR_UNSUPPORTED;
  int chunk = 0;
  size_t smem = 0;
  const bool fused = step_fused(dims, T, k, &chunk, &smem);
  size_t scores_off = 0;
  if (!fused) {
    s = check_attend_ws(dims, k, ws, ws_bytes);
    if (s != DS_OK) return s;
    if (ws_bytes < step_fallback_ws(dims, T, k, &scores_off)) return DS_ERR_WORKSPACE;
    const bool vec = dims.r == 8 || dims.r == 16 || dims.r == 32 || dims.r == 64 ||
                     dims.r == 128;
    if (!vec) return DS_ERR_UNSUPPORTED;  // the fused score+select needs a vector path
  }
  bool kv_device = false;
  s = check_kv(K, V, &kv_device);
  if (s != DS_OK) return s;
  s = check_io(Q, O, lse);
  if (s != DS_OK) return s;
  s = ensure_attrs();
  if (s != DS_OK) return s;
  if (fused) {
    StepParams sp;
    sp.Q = static_cast<const uint16_t*>(Q);
    sp.K = static_cast<const uint16_t*>(K);
    sp.V = static_cast<const uint16_t*>(V);
    sp.K_new = static_cast<const uint16_t*>(K_new);
    sp.V_new = static_cast<const uint16_t*>(V_new);
    sp.C = C;
    sp.label = static_cast<uint16_t*>(label);
    sp.idx = idx;
    sp.O = O;
    sp.lse = lse;
    sp.Hq = dims.Hq;
    sp.Hkv = dims.Hkv;
    sp.T_cap = dims.T_cap;
    sp.T = T;
    sp.k = k;
    sp.append = append ? 1 : 0;
    sp.prefetch = kv_device ? 1 : 0;
    sp.scale_log2 = scale * 1.4426950408889634f;
    const int BH = dims.B * dims.Hq;
    switch (dims.r) {
      case 8: return launch_step<8>(sp, BH, chunk, smem, stream);
      case 16: return launch_step<16>(sp, BH, chunk, smem, stream);
      case 32: return launch_step<32>(sp, BH, chunk, smem, stream);
      case 64: return launch_step<64>(sp, BH, chunk, smem, stream);
      default: return launch_step<128>(sp, BH, chunk, smem, stream);
    }
  }
  // the same step as separate calls
  if (K_new) {
    s = ds_kv_append(K_new, V_new, const_cast<void*>(K), const_cast<void*>(V), dims, T - 1,
                     stream);
    if (s != DS_OK) return s;
  }
  if (append) {
    s = ds_label_append(K, C, label, dims, T - 1, 1, stream);
    if (s != DS_OK) return s;
  }
  if (sel_applies(dims.r, T)) {
    s = ds_score_topk(Q, C, label, nullptr, idx, dims, T, k, static_cast<char*>(ws) + scores_off,
                      ws_bytes - scores_off, stream);
  } else {
    float* scores = prefer_score_then_select(dims.r, T)
                        ? reinterpret_cast<float*>(static_cast<char*>(ws) + scores_off)
                        : nullptr;
    s = ds_score_topk(Q, C, label, scores, idx, dims, T, k, nullptr, 0, stream);
  }
  if (s != DS_OK) return s;
  return launch_attend(dims, Q, K, V, idx, O, lse, T, k, scale, ws, stream);
}

}  // namespace

extern "C" ds_status ds_decode_step(const void* Q, const void* K, const void* V, const int32_t* C,
                                    void* label, int32_t* idx, float* O, float* lse,
                                    ds_dims dims, int32_t T, int32_t k, float scale,
                                    int32_t append, void* ws, size_t ws_bytes,
                                    ds_stream_t stream) {
  DS_TRACE("ds_decode_step");
  return decode_step(Q, nullptr, nullptr, K, V, C, label, idx, O, lse, dims, T, k, scale, append,
                     ws, ws_bytes, stream);
}

extern "C" ds_status ds_decode_step_kv(const void* Q, const void* K_new, const void* V_new,
                                       void* K, void* V, const int32_t* C, void* label,
                                       int32_t* idx, float* O, float* lse, ds_dims dims,
                                       int32_t T, int32_t k, float scale, void* ws,
                                       size_t ws_bytes, ds_stream_t stream) {
  DS_TRACE("ds_decode_step_kv");
  if (!K_new || !V_new) return DS_ERR_INVALID_ARG;
  return decode_step(Q, K_new, V_new, K, V, C, label, idx, O, lse, dims, T, k, scale, 1, ws,
                     ws_bytes, stream);
}

extern "C" ds_status ds_calibrate(const void* Qc, int32_t Nq, const void* K, ds_dims dims,
                                  int32_t T, int32_t* C, float* importance, void* ws,
                                  size_t ws_bytes, ds_stream_t stream) {
  DS_TRACE("ds_calibrate");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!Qc || !K || !C || !aligned16(Qc) || !aligned16(K) || !aligned16(C))
    return DS_ERR_INVALID_ARG;
  if (importance && !aligned16(importance)) return DS_ERR_INVALID_ARG;
  if (Nq < 1 || T < 1 || T > dims.T_cap) return DS_ERR_INVALID_ARG;
  const int nck = (T + kAbsumRows - 1) / kAbsumRows, ncq = (Nq + kAbsumRows - 1) / kAbsumRows;
  if (nck > 65535 || ncq > 65535) return DS_ERR_UNSUPPORTED;
  const size_t need = ds_workspace_size(DS_OP_CALIBRATE, dims, T, Nq);
  if (!ws || ws_bytes < need || !aligned16(ws)) return DS_ERR_WORKSPACE;
  s = check_kv(K, nullptr);
  if (s != DS_OK) return s;
  float* pk = static_cast<float*>(ws);
  float* pq = pk + (size_t)dims.B * dims.Hkv * nck * kHeadDim;
  if ((int64_t)dims.B * (dims.Hkv + dims.Hq) > 65535) return DS_ERR_UNSUPPORTED;
  k_absum<<<dim3(std::max(nck, ncq), dims.B * (dims.Hkv + dims.Hq)), kAbsumThreads, 0, stream>>>(
      static_cast<const uint16_t*>(K), (size_t)dims.T_cap * kHeadDim, T, dims.B * dims.Hkv, pk,
      static_cast<const uint16_t*>(Qc), (size_t)Nq * kHeadDim, Nq, pq);
  s = launched();
  if (s != DS_OK) return s;
  const float inv_pairs = (float)(1.0 / ((double)dims.B * (double)Nq * (double)T));
  k_calib_select<<<dims.Hq, kHeadDim, 0, stream>>>(pk, nck, pq, ncq, dims.B, dims.Hq, dims.Hkv,
                                                   dims.r, inv_pairs, C, importance);
  return launched();
}

namespace {

// Kc: the K cache when the newest token's label rows are appended first, else null.
template <int R>
ds_status launch_group_score(const uint16_t* Q, const int32_t* C, const uint16_t* label,
                             float* sg, const ds_dims& d, int T, cudaStream_t st,
                             const uint16_t* Kc = nullptr) {
  using S = ScoreShape<R>;
  const int G = d.Hq / d.Hkv;
  dim3 grid((T + S::kTokensPerCta - 1) / S::kTokensPerCta, d.B * d.Hkv);
  const size_t smem = (size_t)G * R * (sizeof(float) + (Kc ? 2 : 0));
  k_group_score<R><<<grid, kScoreThreads, smem, st>>>(Q, C, const_cast<uint16_t*>(label), sg,
                                                      d.Hq, d.Hkv, d.T_cap, T, Kc);
  return launched();
}

}  // namespace

extern "C" ds_status ds_group_score_topk(const void* Q, const int32_t* C, const void* label,
                                         float* group_scores, int32_t* idx, ds_dims dims,
                                         int32_t T, int32_t k, ds_stream_t stream) {
  DS_TRACE("ds_group_score_topk");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!Q || !C || !label || !group_scores || !idx || !aligned16(Q) || !aligned16(C) ||
      !aligned16(label) || !aligned16(group_scores) || !aligned16(idx))
    return DS_ERR_INVALID_ARG;
  if (T < 1 || T > dims.T_cap || k < 1 || k > T) return DS_ERR_INVALID_ARG;
  if (T > kMaxCluster * kMaxKeysPerCta) return DS_ERR_UNSUPPORTED;
  const int G = dims.Hq / dims.Hkv;
  if ((size_t)G * dims.r * sizeof(float) > 48 * 1024) return DS_ERR_UNSUPPORTED;
  if (!(dims.r == 8 || dims.r == 16 || dims.r == 32 || dims.r == 64 || dims.r == 128))
    return DS_ERR_UNSUPPORTED;
  s = ensure_attrs();
  if (s != DS_OK) return s;
  auto Qb = static_cast<const uint16_t*>(Q);
  auto Lb = static_cast<const uint16_t*>(label);
  switch (dims.r) {
    case 8: s = launch_group_score<8>(Qb, C, Lb, group_scores, dims, T, stream); break;
    case 16: s = launch_group_score<16>(Qb, C, Lb, group_scores, dims, T, stream); break;
    case 32: s = launch_group_score<32>(Qb, C, Lb, group_scores, dims, T, stream); break;
    case 64: s = launch_group_score<64>(Qb, C, Lb, group_scores, dims, T, stream); break;
    case 128: s = launch_group_score<128>(Qb, C, Lb, group_scores, dims, T, stream); break;
    default: return DS_ERR_UNSUPPORTED;
  }
  if (s != DS_OK) return s;
  return launch_topk(ScoresSource{group_scores}, idx, dims.B * dims.Hkv, T, k, stream);
}

extern "C" ds_status ds_group_sparse_decode(const void* Q, const void* K, const void* V,
                                            const int32_t* idx, float* O, float* lse,
                                            ds_dims dims, int32_t T, int32_t k, float scale,
                                            void* ws, size_t ws_bytes, ds_stream_t stream) {
  DS_TRACE("ds_group_sparse_decode");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!Q || !K || !V || !idx || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) ||
      !aligned16(idx) || !aligned16(O) || (lse && !aligned16(lse)))
    return DS_ERR_INVALID_ARG;
  if (T < 1 || T > dims.T_cap || k < 1 || k > T) return DS_ERR_INVALID_ARG;
  s = check_shared_rows_ws(dims, k, ws, ws_bytes);
  if (s != DS_OK) return s;
  s = check_kv(K, V);
  if (s != DS_OK) return s;
  s = ensure_attrs();
  if (s != DS_OK) return s;
  if (group_kernel_applies(dims))
    return launch_attend_group(dims, Q, K, V, idx, O, lse, T, k, scale, ws, stream);
  return launch_attend(dims, Q, K, V, idx, O, lse, T, k, scale, ws, stream, true);
}

extern "C" ds_status ds_group_decode_step(const void* Q, const void* K, const void* V,
                                          const int32_t* C, void* label, float* group_scores,
                                          int32_t* idx, float* O, float* lse, ds_dims dims,
                                          int32_t T, int32_t k, float scale, int32_t append,
                                          void* ws, size_t ws_bytes, ds_stream_t stream) {
  DS_TRACE("ds_group_decode_step");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!Q || !K || !V || !C || !label || !group_scores || !idx || !O || !aligned16(Q) ||
      !aligned16(K) || !aligned16(V) || !aligned16(C) || !aligned16(label) ||
      !aligned16(group_scores) || !aligned16(idx) || !aligned16(O) || (lse && !aligned16(lse)))
    return DS_ERR_INVALID_ARG;
  if (T < 1 || T > dims.T_cap || k < 1 || k > T) return DS_ERR_INVALID_ARG;
  if (T > kMaxCluster * kMaxKeysPerCta) return DS_ERR_UNSUPPORTED;
  const int G = dims.Hq / dims.Hkv;
  if ((size_t)G * dims.r * (sizeof(float) + 2) > 48 * 1024) return DS_ERR_UNSUPPORTED;
  if (!(dims.r == 8 || dims.r == 16 || dims.r == 32 || dims.r == 64 || dims.r == 128))
    return DS_ERR_UNSUPPORTED;
  size_t sel_off = 0;
  const size_t need = group_step_ws(dims, T, k, &sel_off);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws))) return DS_ERR_WORKSPACE;
  s = check_kv(K, V);
  if (s != DS_OK) return s;
  s = ensure_attrs();
  if (s != DS_OK) return s;
  auto Qb = static_cast<const uint16_t*>(Q);
  auto Lb = static_cast<const uint16_t*>(label);
  const uint16_t* Kc = append ? static_cast<const uint16_t*>(K) : nullptr;
  switch (dims.r) {
    case 8: s = launch_group_score<8>(Qb, C, Lb, group_scores, dims, T, stream, Kc); break;
    case 16: s = launch_group_score<16>(Qb, C, Lb, group_scores, dims, T, stream, Kc); break;
    case 32: s = launch_group_score<32>(Qb, C, Lb, group_scores, dims, T, stream, Kc); break;
    case 64: s = launch_group_score<64>(Qb, C, Lb, group_scores, dims, T, stream, Kc); break;
    default: s = launch_group_score<128>(Qb, C, Lb, group_scores, dims, T, stream, Kc); break;
  }
  if (s != DS_OK) return s;
  if (sel_off)
    s = launch_scores_sel(group_scores, idx, dims.B * dims.Hkv, T, k,
                          static_cast<char*>(ws) + sel_off, stream);
  else
    s = launch_topk(ScoresSource{group_scores}, idx, dims.B * dims.Hkv, T, k, stream);
  if (s != DS_OK) return s;
  if (group_kernel_applies(dims))
    return launch_attend_group(dims, Q, K, V, idx, O, lse, T, k, scale, ws, stream);
  return launch_attend(dims, Q, K, V, idx, O, lse, T, k, scale, ws, stream, true);
}


namespace {

bool block_size_ok(int bs) { return bs >= 1 && bs <= 64 && (bs & (bs - 1)) == 0; }

template <int R>
ds_status launch_block_score(const uint16_t* Q, const int32_t* C, const uint16_t* label,
                             float* sb, const ds_dims& d, int T, int bs, cudaStream_t st) {
  using S = ScoreShape<R>;
  dim3 grid((T + S::kTokensPerCta - 1) / S::kTokensPerCta, d.B * d.Hq);
  k_block_score<R><<<grid, kScoreThreads, 0, st>>>(Q, C, label, sb, d.Hq, d.T_cap, T, bs);
  return launched();
}

}  // namespace

extern "C" ds_status ds_block_score_topk(const void* Q, const int32_t* C, const void* label,
                                         float* block_scores, int32_t* bidx, ds_dims dims,
                                         int32_t T, int32_t bs, int32_t kb, ds_stream_t stream) {
  DS_TRACE("ds_block_score_topk");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!Q || !C || !label || !block_scores || !bidx || !aligned16(Q) || !aligned16(C) ||
      !aligned16(label) || !aligned16(block_scores) || !aligned16(bidx))
    return DS_ERR_INVALID_ARG;
  if (!block_size_ok(bs)) return DS_ERR_INVALID_ARG;
  if (T < 1 || T > dims.T_cap) return DS_ERR_INVALID_ARG;
  const int nblk = (T + bs - 1) / bs;
  if (kb < 1 || kb > nblk) return DS_ERR_INVALID_ARG;
  if (!(dims.r == 8 || dims.r == 16 || dims.r == 32 || dims.r == 64 || dims.r == 128))
    return DS_ERR_UNSUPPORTED;
  s = ensure_attrs();
  if (s != DS_OK) return s;
  auto Qb = static_cast<const uint16_t*>(Q);
  auto Lb = static_cast<const uint16_t*>(label);
  switch (dims.r) {
    case 8: s = launch_block_score<8>(Qb, C, Lb, block_scores, dims, T, bs, stream); break;
    case 16: s = launch_block_score<16>(Qb, C, Lb, block_scores, dims, T, bs, stream); break;
    case 32: s = launch_block_score<32>(Qb, C, Lb, block_scores, dims, T, bs, stream); break;
    case 64: s = launch_block_score<64>(Qb, C, Lb, block_scores, dims, T, bs, stream); break;
    default: s = launch_block_score<128>(Qb, C, Lb, block_scores, dims, T, bs, stream); break;
  }
  if (s != DS_OK) return s;
  return launch_topk(ScoresSource{block_scores}, bidx, dims.B * dims.Hq, nblk, kb, stream);
}

extern "C" ds_status ds_block_sparse_decode(const void* Q, const void* K, const void* V,
                                            const int32_t* bidx, float* O, float* lse,
                                            ds_dims dims, int32_t T, int32_t bs, int32_t kb,
                                            float scale, void* ws, size_t ws_bytes,
                                            ds_stream_t stream) {
  DS_TRACE("ds_block_sparse_decode");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!Q || !K || !V || !bidx || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) ||
      !aligned16(bidx) || !aligned16(O) || (lse && !aligned16(lse)))
    return DS_ERR_INVALID_ARG;
  if (!block_size_ok(bs)) return DS_ERR_INVALID_ARG;
  if (T < 1 || T > dims.T_cap) return DS_ERR_INVALID_ARG;
  if (kb < 1 || kb > (T + bs - 1) / bs) return DS_ERR_INVALID_ARG;
  const int rows = kb * bs;
  s = check_attend_ws(dims, rows, ws, ws_bytes);
  if (s != DS_OK) return s;
  s = check_kv(K, V);
  if (s != DS_OK) return s;
  s = ensure_attrs();
  if (s != DS_OK) return s;
  return launch_attend(dims, Q, K, V, bidx, O, lse, T, rows, scale, ws, stream, false, bs);
}

namespace {

template <int R>
ds_status launch_hier(const uint16_t* Q, const int32_t* C, const uint16_t* label, int32_t* idx,
                      const ds_dims& d, int T, int k, cudaStream_t st) {
  const size_t smem = HierLayout(TopkLayout((2 * k + 31) & ~31, 1)).bytes();
  LabelSource<R> src{Q, C, label, nullptr, d.Hq, d.T_cap};
  k_hier_topk<LabelSource<R>><<<d.B * d.Hq, kTopkThreads, smem, st>>>(src, idx, T, k);
  return launched();
}

}  // namespace

extern "C" ds_status ds_hier_score_topk(const void* Q, const int32_t* C, const void* label,
                                        int32_t* idx, ds_dims dims, int32_t T, int32_t k,
                                        ds_stream_t stream) {
  DS_TRACE("ds_hier_score_topk");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!Q || !C || !label || !idx || !aligned16(Q) || !aligned16(C) || !aligned16(label) ||
      !aligned16(idx))
    return DS_ERR_INVALID_ARG;
  if (T < 1 || T > dims.T_cap || k < 1 || k > T) return DS_ERR_INVALID_ARG;
  if (k > kHierMaxK) return DS_ERR_UNSUPPORTED;
  if (!(dims.r == 8 || dims.r == 16 || dims.r == 32 || dims.r == 64 || dims.r == 128))
    return DS_ERR_UNSUPPORTED;
  s = ensure_attrs();
  if (s != DS_OK) return s;
  auto Qb = static_cast<const uint16_t*>(Q);
  auto Lb = static_cast<const uint16_t*>(label);
  switch (dims.r) {
    case 8: return launch_hier<8>(Qb, C, Lb, idx, dims, T, k, stream);
    case 16: return launch_hier<16>(Qb, C, Lb, idx, dims, T, k, stream);
    case 32: return launch_hier<32>(Qb, C, Lb, idx, dims, T, k, stream);
    case 64: return launch_hier<64>(Qb, C, Lb, idx, dims, T, k, stream);
    default: return launch_hier<128>(Qb, C, Lb, idx, dims, T, k, stream);
  }
}

extern "C" ds_status ds_kv_append(const void* K_new, const void* V_new, void* K, void* V,
                                  ds_dims dims, int32_t t, ds_stream_t stream) {
  DS_TRACE("ds_kv_append");
  ds_status s = check_dims(dims);
  if (s != DS_OK) return s;
  if (!K_new || !V_new || !K || !V || !aligned16(K_new) || !aligned16(V_new) || !aligned16(K) ||
      !aligned16(V))
    return DS_ERR_INVALID_ARG;
  if (t < 0 || t >= dims.T_cap) return DS_ERR_INVALID_ARG;
  s = check_kv(K, V);
  if (s != DS_OK) return s;
  s = check_kv(K_new, V_new);
  if (s != DS_OK) return s;
  k_kv_append<<<dims.B * dims.Hkv, 32, 0, stream>>>(
      static_cast<const uint16_t*>(K_new), static_cast<const uint16_t*>(V_new),
      static_cast<uint16_t*>(K), static_cast<uint16_t*>(V), dims.T_cap, t);
  return launched();
}
