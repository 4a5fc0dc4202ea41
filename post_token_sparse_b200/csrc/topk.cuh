// Per-head top-k by radix select over shared-memory-resident keys.
//
// Token selection keeps the tokens with the highest approximate activation
// (Double Sparsity, Method details: Key design).  Contract: the k largest
// scores, ties to the lower token index, -0 == +0, output ascending.
//
// One thread-block cluster per head (cluster size CS = 1..16).  CTA c of the
// cluster owns the contiguous token range [c*chunk, min((c+1)*chunk, T)) and
// keeps its order-preserving uint32 keys in shared memory for the whole
// selection, so scores are read (or computed from the label cache) once.
//
//   1. fill    keys + local histogram of digit 0 (key bits 31..21)
//   2. digit   local histograms are added into CTA 0's shared memory through
//              distributed shared memory; after a cluster barrier every CTA
//              reads the merged histogram and finds the bin holding the k-th
//              largest key.  Digits: bits 31..21, 20..10, 9..0.  If the bin's
//              whole population is needed, selection is "key >= bin start"
//              and the remaining digits are skipped.
//   3. output  two passes over the keys: per-warp counts of (key > thr) and
//              (key == thr), a cluster-wide exclusive scan of the per-CTA
//              counts (read through distributed shared memory), then warp
//              ballots place each selected index at its rank: ascending
//              order and the lower-index tie rule fall out of the scan order.
//
// Synchronisation is by hardware cluster / CTA barriers only; no spin waits.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "score.cuh"

namespace ds {

namespace cg = cooperative_groups;

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kMaxCluster = 16;
constexpr int kMaxKeysPerCta = 40960;
// digits of the 32-bit key: bits 31..21, 20..10, 9..0
__host__ __device__ constexpr int digit_shift(int d) { return d == 0 ? 21 : (d == 1 ? 10 : 0); }
__host__ __device__ constexpr int digit_bits(int d) { return d == 2 ? 10 : 11; }
__host__ __device__ constexpr int digit_bins(int d) { return 1 << digit_bits(d); }
constexpr int kBinsPerThread = 2048 / kTopkThreads;  // 4

// Shared-memory layout (32-bit words); keys follow.
struct TopkSmem {
  static constexpr int kHist = 0;                   // local histogram [2048]
  static constexpr int kMerged0 = kHist + 2048;     // merged digit 0 (used in CTA 0)
  static constexpr int kMerged1 = kMerged0 + 2048;  // merged digit 1
  static constexpr int kMerged2 = kMerged1 + 2048;  // merged digit 2 [1024]; kMerged0 + 2048*d
  static constexpr int kWarpGt = kMerged2 + 1024;   // per-warp counts
  static constexpr int kWarpEq = kWarpGt + kTopkWarps;
  static constexpr int kScan = kWarpEq + kTopkWarps;  // block-scan scratch [kTopkWarps]
  static constexpr int kMisc = kScan + kTopkWarps;    // 16 words of broadcast values
  static constexpr int kKeys = kMisc + 16;
  static constexpr size_t bytes(int keys) { return (size_t)(kKeys + keys) * 4; }
};
enum { M_BIN = 0, M_ABOVE = 1, M_CNT = 2, M_CTA_GT = 3, M_CTA_EQ = 4 };

__device__ __forceinline__ void cluster_or_cta_sync(int cs) {
  if (cs > 1)
    cg::this_cluster().sync();
  else
    __syncthreads();
}

// Exclusive block-wide prefix sum over threads in thread order.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  uint32_t wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += scratch[w];
  __syncthreads();
  return wbase + incl - v;
}

// Finds the bin b (counting bins from the top) such that
// count(bins > b) < krem <= count(bins >= b) and writes b, count(bins > b)
// and count(b) to misc.  `hist` may point into another CTA's shared memory.
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nbins, uint32_t krem,
                                         uint32_t* scratch, uint32_t* misc) {
  uint32_t c[kBinsPerThread];
  uint32_t sum = 0;
#pragma unroll
  for (int j = 0; j < kBinsPerThread; ++j) {
    const int b = nbins - 1 - (threadIdx.x * kBinsPerThread + j);
    c[j] = b >= 0 ? hist[b] : 0u;
    sum += c[j];
  }
  const uint32_t above = block_exclusive_scan(sum, scratch);
  if (sum > 0 && above < krem && krem <= above + sum) {
    uint32_t acc = above;
#pragma unroll
    for (int j = 0; j < kBinsPerThread; ++j) {
      if (acc + c[j] >= krem) {
        misc[M_BIN] = (uint32_t)(nbins - 1 - (threadIdx.x * kBinsPerThread + j));
        misc[M_ABOVE] = acc;
        misc[M_CNT] = c[j];
        break;
      }
      acc += c[j];
    }
  }
  __syncthreads();
}

// Key sources -----------------------------------------------------------------

// Keys from precomputed fp32 scores [BH, T].
struct ScoresSource {
  const float* scores;
  __device__ __forceinline__ void fill(int bh, int T, int c0, int len, uint32_t* keys,
                                       uint32_t* hist) const {
    const float* src = scores + (size_t)bh * T + c0;
    int i = threadIdx.x;
    for (; i + 3 * kTopkThreads < len; i += 4 * kTopkThreads) {
      float f[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) f[u] = __ldcs(src + i + u * kTopkThreads);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t key = order_key(f[u]);
        keys[i + u * kTopkThreads] = key;
        atomicAdd(&hist[key >> digit_shift(0)], 1u);
      }
    }
    for (; i < len; i += kTopkThreads) {
      const uint32_t key = order_key(__ldcs(src + i));
      keys[i] = key;
      atomicAdd(&hist[key >> digit_shift(0)], 1u);
    }
  }
};

// Keys computed from the label cache: the fused score + select path.  Scores
// are computed exactly as k_score_vec computes them.
template <int R>
struct LabelSource {
  const uint16_t* Q;
  const int32_t* C;
  const uint16_t* label;
  float* scores_out;  // optional
  int Hq, T_cap;
  static constexpr int kChunks = R / 8;
  static constexpr int kRows = kChunks >= 4 ? 1 : 4 / kChunks;

  __device__ __forceinline__ void fill(int bh, int T, int c0, int len, uint32_t* keys,
                                       uint32_t* hist) const {
    __shared__ __align__(16) float qs[R];
    load_qc(Q, C, bh, bh % Hq, R, qs);
    __syncthreads();
    const uint4* lab = reinterpret_cast<const uint4*>(label + ((size_t)bh * T_cap + c0) * R);
    float* out = scores_out ? scores_out + (size_t)bh * T + c0 : nullptr;
    for (int base = 0; base < len; base += kTopkThreads * kRows) {
      uint4 v[kRows][kChunks];
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const int t = base + threadIdx.x + i * kTopkThreads;
        if (t < len) {
#pragma unroll
          for (int c = 0; c < kChunks; ++c) v[i][c] = ldg_stream(lab + (size_t)t * kChunks + c);
        }
      }
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const int t = base + threadIdx.x + i * kTopkThreads;
        if (t < len) {
          const float s = row_score<R>(v[i], qs);
          if (out) out[t] = s;
          const uint32_t key = order_key(s);
          keys[t] = key;
          atomicAdd(&hist[key >> digit_shift(0)], 1u);
        }
      }
    }
  }
};

// grid (CS, BH), cluster (CS, 1, 1).  chunk: tokens per CTA.
template <class Source>
__global__ void __launch_bounds__(kTopkThreads)
k_topk(Source src, int32_t* __restrict__ idx, int T, int k, int chunk) {
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t* hist = sm + TopkSmem::kHist;
  uint32_t* scratch = sm + TopkSmem::kScan;
  uint32_t* misc = sm + TopkSmem::kMisc;
  uint32_t* keys = sm + TopkSmem::kKeys;

  const int cs = gridDim.x;
  const int rank = blockIdx.x;  // == cluster rank: the cluster spans grid dimension x
  const int bh = blockIdx.y;
  const int c0 = min(rank * chunk, T);
  const int len = min(chunk, T - c0);

  for (int i = threadIdx.x; i < TopkSmem::kKeys; i += kTopkThreads) sm[i] = 0u;
  // every CTA of the cluster is running and its merged buffers are zero
  // before any remote access
  cluster_or_cta_sync(cs);

  src.fill(bh, T, c0, len, keys, hist);
  __syncthreads();

  uint32_t krem = (uint32_t)k, prefix = 0u, thr = 0u, need = 0u;
  bool ge_mode = false;

  for (int d = 0; d < 3; ++d) {
    const int nbins = digit_bins(d), shift = digit_shift(d);
    if (d > 0) {
      // local histogram of digit d over the keys that carry the chosen prefix
      for (int i = threadIdx.x; i < nbins; i += kTopkThreads) hist[i] = 0u;
      __syncthreads();
      const int hi_shift = digit_shift(d - 1);
      for (int i = threadIdx.x; i < len; i += kTopkThreads) {
        const uint32_t key = keys[i];
        if ((key >> hi_shift) == prefix) atomicAdd(&hist[(key >> shift) & (nbins - 1)], 1u);
      }
      __syncthreads();
    }
    const uint32_t* merged = hist;
    if (cs > 1) {
      cg::cluster_group cl = cg::this_cluster();
      uint32_t* m0 = cl.map_shared_rank(sm + TopkSmem::kMerged0 + d * 2048, 0);
      for (int i = threadIdx.x; i < nbins; i += kTopkThreads) {
        const uint32_t v = hist[i];
        if (v) atomicAdd(m0 + i, v);
      }
      cl.sync();
      merged = m0;
    }
    find_bin(merged, nbins, krem, scratch, misc);
    const uint32_t bin = misc[M_BIN], above = misc[M_ABOVE], cnt = misc[M_CNT];
    krem -= above;
    prefix = (prefix << digit_bits(d)) | bin;
    if (cnt == krem) {  // the whole bin is selected
      ge_mode = true;
      thr = prefix << shift;
      break;
    }
    if (d == 2) {
      thr = prefix;
      need = krem;
    }
  }

  // ---- output: counts per warp --------------------------------------------
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = ((len + kTopkWarps - 1) / kTopkWarps + 31) & ~31;
  const int w0 = min(warp * seg, len), w1 = min(w0 + seg, len);
  uint32_t n_gt = 0, n_eq = 0;
  for (int i = w0 + lane; i - lane < w1; i += 32) {
    const bool in = i < w1;
    const uint32_t key = in ? keys[i] : 0u;
    const bool gt = in && (ge_mode ? key >= thr : key > thr);
    const bool eq = in && !ge_mode && key == thr;
    n_gt += __popc(__ballot_sync(0xffffffffu, gt));
    n_eq += __popc(__ballot_sync(0xffffffffu, eq));
  }
  if (lane == 0) {
    sm[TopkSmem::kWarpGt + warp] = n_gt;
    sm[TopkSmem::kWarpEq + warp] = n_eq;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t g = 0, e = 0;
    for (int w = 0; w < kTopkWarps; ++w) {
      g += sm[TopkSmem::kWarpGt + w];
      e += sm[TopkSmem::kWarpEq + w];
    }
    misc[M_CTA_GT] = g;
    misc[M_CTA_EQ] = e;
  }
  cluster_or_cta_sync(cs);

  // counts of the CTAs before this one in the cluster, then of earlier warps
  uint32_t gt_before = 0, eq_before = 0;
  if (cs > 1) {
    cg::cluster_group cl = cg::this_cluster();
    for (int c = 0; c < rank; ++c) {
      const uint32_t* m = cl.map_shared_rank(misc, c);
      gt_before += m[M_CTA_GT];
      eq_before += m[M_CTA_EQ];
    }
  }
  for (int w = 0; w < warp; ++w) {
    gt_before += sm[TopkSmem::kWarpGt + w];
    eq_before += sm[TopkSmem::kWarpEq + w];
  }

  // ---- output: place the selected indices ----------------------------------
  uint32_t tie = eq_before;
  uint32_t out = gt_before + min(eq_before, need);
  int32_t* dst = idx + (size_t)bh * k;
  const uint32_t lt = lanemask_lt();
  for (int i = w0 + lane; i - lane < w1; i += 32) {
    const bool in = i < w1;
    const uint32_t key = in ? keys[i] : 0u;
    const bool gt = in && (ge_mode ? key >= thr : key > thr);
    const bool eq = in && !ge_mode && key == thr;
    const uint32_t eq_mask = __ballot_sync(0xffffffffu, eq);
    const bool sel = gt || (eq && tie + __popc(eq_mask & lt) < need);
    const uint32_t sel_mask = __ballot_sync(0xffffffffu, sel);
    const uint32_t pos = out + __popc(sel_mask & lt);
    if (sel && pos < (uint32_t)k) dst[pos] = c0 + i;
    tie += __popc(eq_mask);
    out += __popc(sel_mask);
  }
  // no CTA leaves while another may still read its shared memory
  cluster_or_cta_sync(cs);
}

}  // namespace ds
