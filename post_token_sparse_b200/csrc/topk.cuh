// Per-head top-k: sample-bracketed selection in one streaming pass.
//
// Token selection keeps the tokens with the highest approximate activation
// (Double Sparsity, Method details: Key design).  Contract: the k largest
// scores, ties to the lower token index, -0 == +0, output ascending.
//
// One thread-block cluster per head (cluster size CS = 1..16); CTA c owns the
// tokens [c*chunk, min((c+1)*chunk, T)).  No CTA stores its keys: shared
// memory holds two bit masks and a short candidate list, so four CTAs share
// an SM and one CTA's selection work overlaps the others' streaming.
//
//   1. sample   exact keys of a stratified sample of the whole head: 128
//               blocks of 32 consecutive tokens spread over [0, T), or every
//               token when T <= 4096.  Every CTA of a cluster draws the same
//               sample, so all of them agree on what follows without talking.
//   2. bracket  list select on the sample (below): with the whole head sampled,
//               the exact k-th key (lo = hi = threshold), and the head's keys
//               are classified on the way; otherwise the sample's keys at
//               ranks k*m/T -/+ (5 standard deviations + 2) become hi / lo:
//               keys above hi are selected, keys below lo are not.
//   3. stream   one pass over this CTA's keys (computed from the label cache,
//               or read from the scores): key > hi sets a bit of the "above"
//               mask; lo <= key <= hi sets a bit of the "equal" mask when
//               lo == hi, else goes to the candidate list (exact key, token).
//   4. check    cluster totals must put the k-th key inside [lo, hi] with no
//               list overflow.  If not (a sample miss, or heavy ties), exact
//               refinement takes over: one histogram pass per key digit
//               narrows the bracket to the bin holding the k-th key and the
//               stream pass repeats; a one-value bracket always fits.
//   5. resolve  select of the remaining rank over the candidates (a list
//               select for one CTA; a radix select with histograms merged over
//               the cluster otherwise) gives the exact threshold key;
//               candidates above it join the "above" mask, candidates equal to
//               it the "equal" mask.
//
// List select: radix select over 11-bit digits in which, after each digit, the
// items of the chosen bin are compacted into a short list, so that the next
// digit and the end touch only those; once at most one item per thread is
// left, threads count the items above and equal to each.
//   6. write    per-warp counts, a cluster-wide exclusive scan (pushed into the
//               later CTAs before a barrier), then one 32-token group per lane:
//               indices in ascending order, ties taken in index order.
//
// Synchronisation is by hardware CTA / cluster barriers only; no spin waits.
// No CTA touches another's shared memory after the last cluster barrier.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "score.cuh"

namespace ds {

namespace cg = cooperative_groups;

constexpr int kTopkThreads = 256;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kMaxCluster = 16;
constexpr int kMaxKeysPerCta = 65536;
constexpr int kSample = 4096;                // sample size (the whole head when T <= kSample)
constexpr int kSampleBlocks = kSample / 32;  // 128 blocks of 32 consecutive tokens
constexpr int kCandCap = 4096;               // candidate list of one CTA
constexpr float kBracketSigmas = 5.f;
constexpr int kListCap = 1024;            // items of one list-select buffer
constexpr int kRankCount = kTopkThreads;  // items at which ranks are counted directly
constexpr int kSelectIters = 4;           // list select sources: 4 x (4 items per thread)
constexpr int kWideBits = 13;             // sample histogram of one CTA: top 13 key bits
constexpr int kWideBins = 1 << kWideBits;

// digits of the 32-bit key: bits 31..21, 20..10, 9..0
__host__ __device__ constexpr int digit_shift(int d) { return d == 0 ? 21 : (d == 1 ? 10 : 0); }
__host__ __device__ constexpr int digit_bits(int d) { return d == 2 ? 10 : 11; }
__host__ __device__ constexpr int digit_bins(int d) { return 1 << digit_bits(d); }
constexpr int kBinsPerThread = 2048 / kTopkThreads;  // 8

// Shared-memory layout in 32-bit words (depends on the chunk and cluster size).
struct TopkLayout {
  int merged0, merged1, small, masks, X, lists, words;
  __host__ __device__ TopkLayout(int chunk, int cs) {
    int o = 2048;  // histogram (2048 bins) at 0
    merged0 = o;   // cluster-merged histograms (CTA-local copies)
    if (cs > 1) o += 2048;
    merged1 = o;
    if (cs > 1) o += 2048;
    small = o;  // misc[32], warp_gt[8], warp_eq[8], scan[16], q[C] as fp32 [128]
    o += 192;
    masks = o;  // per 32-token group: "above" bits, then "equal" bits
    o += 2 * (chunk / 32);
    o = (o + 3) & ~3;
    X = o;  // candidates: keys [kCandCap], tokens [kCandCap]; while sampling, the
            // sample keys in the first half and two histograms in the second
    o += 2 * kCandCap;
    // list select: two buffers of kListCap (key, token) pairs; with a cluster
    // they overlay the merged histograms, which are not in use while a CTA
    // selects on its own
    if (cs > 1) {
      lists = merged0;
    } else {
      lists = o;
      o += 4 * kListCap;
    }
    words = o;
  }
  __host__ __device__ size_t bytes() const { return (size_t)words * 4; }
};
static_assert(kSample <= kCandCap, "sample keys live in the candidate-key half");
static_assert(4 * kListCap == 2 * 2048, "list buffers fit the two merged histograms");
static_assert(kCandCap + 4 * kListCap == kWideBins,
              "the wide sample histogram spans the candidate tokens and the lists");
static_assert(kRankCount == kTopkThreads, "one counted item per thread");
static_assert(kBinsPerThread == 8, "find_bins reads its bins as two 16-byte vectors");
static_assert(4 * kSelectIters * kTopkThreads >= kCandCap &&
                  4 * kSelectIters * kTopkThreads >= kSample,
              "every list select source fits the unrolled pass");

enum {
  M_BIN = 0, M_ABOVE = 1, M_CNT = 2,     // find_bins, target 1
  M_BIN2 = 3, M_ABOVE2 = 4, M_CNT2 = 5,  // find_bins, target 2
  M_NCAND = 6,                           // this CTA's candidate count
  M_LIST = 7,                            // list select: compaction counter (zero between uses)
  M_THR = 14, M_NEED = 15,               // list select: result key, its rank among equal keys
  M_HI = 16, M_LO = 17,                  // a cluster's bracket, written by CTAs 0 and 1
  M_TOT = 8,                             // cluster totals: above, equal, cand, overflow
  M_GT_BEFORE = 12, M_EQ_BEFORE = 13     // counts of the earlier CTAs of the cluster
};

__device__ __forceinline__ void cluster_or_cta_sync(int cs) {
  if (cs > 1)
    cg::this_cluster().sync();
  else
    __syncthreads();
}

// Exclusive block-wide prefix sum over threads in thread order.  One barrier;
// scratch[0..kTopkWarps) must not be written again before the caller's next
// barrier.
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
  return wbase + incl - v;
}

// For rank r (1 = largest) finds the bin b (bins counted from the top) with
// count(bins > b) < r <= count(bins >= b) and writes b, count(bins > b) and
// count(b) to out[0..2]; r == 0 finds nothing.  Two ranks share one scan.
__device__ __forceinline__ void find_bins(const uint32_t* hist, int nbins, uint32_t r1,
                                          uint32_t r2, uint32_t* scratch, uint32_t* out1,
                                          uint32_t* out2) {
  uint32_t c[kBinsPerThread];
  uint32_t sum = 0;
  const int top = nbins - 1 - threadIdx.x * kBinsPerThread;  // this thread's first bin
  if ((nbins & 7) == 0) {
    // bins top-7 .. top, 16-byte aligned: two vector loads
    if (top >= 7) {
      const uint4 lo = *reinterpret_cast<const uint4*>(hist + top - 7);
      const uint4 hi = *reinterpret_cast<const uint4*>(hist + top - 3);
      c[0] = hi.w; c[1] = hi.z; c[2] = hi.y; c[3] = hi.x;
      c[4] = lo.w; c[5] = lo.z; c[6] = lo.y; c[7] = lo.x;
    } else {
#pragma unroll
      for (int j = 0; j < kBinsPerThread; ++j) c[j] = 0u;
    }
#pragma unroll
    for (int j = 0; j < kBinsPerThread; ++j) sum += c[j];
  } else {
#pragma unroll
    for (int j = 0; j < kBinsPerThread; ++j) {
      const int b = top - j;
      c[j] = b >= 0 ? hist[b] : 0u;
      sum += c[j];
    }
  }
  const uint32_t above = block_exclusive_scan(sum, scratch);
  auto find = [&](uint32_t r, uint32_t* out) {
    if (r && sum > 0 && above < r && r <= above + sum) {
      uint32_t acc = above;
#pragma unroll
      for (int j = 0; j < kBinsPerThread; ++j) {
        if (acc + c[j] >= r) {
          out[0] = (uint32_t)(nbins - 1 - (threadIdx.x * kBinsPerThread + j));
          out[1] = acc;
          out[2] = c[j];
          break;
        }
        acc += c[j];
      }
    }
  };
  find(r1, out1);
  find(r2, out2);
  __syncthreads();
}

// find_bins over NB * kTopkThreads bins, NB per thread (read as vectors).
template <int NB>
__device__ __forceinline__ void find_bins_wide(const uint32_t* hist, uint32_t r1, uint32_t r2,
                                               uint32_t* scratch, uint32_t* out1,
                                               uint32_t* out2) {
  static_assert(NB % 16 == 0, "bins are read sixteen at a time");
  const int topb = NB * kTopkThreads - 1 - NB * (int)threadIdx.x;  // this thread's highest bin
  const uint4* v = reinterpret_cast<const uint4*>(hist + topb - (NB - 1));
  uint32_t sum = 0;
  // neighbouring threads' ranges are NB words apart: a rotated vector order
  // keeps the eight lanes of each shared-memory wavefront on distinct banks
#pragma unroll
  for (int q = 0; q < NB / 4; ++q) {
    const uint4 x = v[(q + threadIdx.x) % (NB / 4)];
    sum += x.x + x.y + x.z + x.w;
  }
  const uint32_t above = block_exclusive_scan(sum, scratch);
  auto find = [&](uint32_t r, uint32_t* out) {
    if (r && sum > 0 && above < r && r <= above + sum) {
      // this thread's bins, four vectors at a time from the top
      uint32_t acc = above;
      bool done = false;
#pragma unroll
      for (int q0 = NB / 4 - 4; q0 >= 0 && !done; q0 -= 4) {
        uint4 x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) x[u] = v[q0 + u];
#pragma unroll
        for (int u = 3; u >= 0; --u) {
          const uint32_t c4[4] = {x[u].w, x[u].z, x[u].y, x[u].x};  // descending bins
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (!done && acc + c4[e] >= r) {
              out[0] = (uint32_t)(topb - (NB - 1) + 4 * (q0 + u) + 3 - e);
              out[1] = acc;
              out[2] = c4[e];
              done = true;
            }
            if (!done) acc += c4[e];
          }
        }
      }
    }
  };
  find(r1, out1);
  find(r2, out2);
  __syncthreads();
}

__device__ __forceinline__ void find_bin(const uint32_t* hist, int nbins, uint32_t r,
                                         uint32_t* scratch, uint32_t* out) {
  find_bins(hist, nbins, r, 0u, scratch, out, out);
}

// hist (nbins bins) summed over the cluster into every CTA's merged copy;
// returns the histogram to read (the local one when cs == 1).
__device__ __forceinline__ const uint32_t* cluster_hist(uint32_t* hist, uint32_t* merged,
                                                        int nbins, int cs) {
  if (cs == 1) return hist;
  cg::cluster_group cl = cg::this_cluster();
  for (int i = threadIdx.x; i < nbins; i += kTopkThreads) {
    const uint32_t v = hist[i];
    if (v)
      for (int c = 0; c < cs; ++c) atomicAdd(cl.map_shared_rank(merged, c) + i, v);
  }
  cl.sync();
  return merged;
}

// Four counters summed over the cluster into misc[M_TOT..M_TOT+3] of every CTA
// (those words must be zero everywhere; the caller zeroes them after use,
// before its next cluster barrier).
__device__ __forceinline__ void cluster_totals(uint32_t* misc, const uint32_t (&v)[4], int cs) {
  if (threadIdx.x == 0) {
    if (cs == 1) {
      for (int i = 0; i < 4; ++i) misc[M_TOT + i] = v[i];
    } else {
      cg::cluster_group cl = cg::this_cluster();
      for (int c = 0; c < cs; ++c) {
        uint32_t* m = cl.map_shared_rank(misc, c);
        for (int i = 0; i < 4; ++i)
          if (v[i]) atomicAdd(m + M_TOT + i, v[i]);
      }
    }
  }
  cluster_or_cta_sync(cs);
}

// Key sources -----------------------------------------------------------------
// stream(): computes the keys of items j < n (token tok(j)) and calls
//   f(valid, j, key, score) on every thread for every item slot it owns; valid
//   is false for slots past n and, when several lanes share a label row, on all
//   but the row's first lane.  Every lane makes the same calls.

// Keys from precomputed fp32 scores [BH, T].
struct ScoresSource {
  const float* scores;
  __device__ __forceinline__ void prepare(int, float*) const {}
  __device__ __forceinline__ float* scores_out(int, int) const { return nullptr; }
  template <class Tok, class F>
  __device__ __forceinline__ void stream(int bh, int T, int n, Tok tok, F&& f,
                                         const float*) const {
    const float* src = scores + (size_t)bh * T;
    constexpr int kU = 8, kStep = kU * kTopkThreads;
    float v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int j = threadIdx.x + u * kTopkThreads;
      v[u] = j < n ? __ldcs(src + tok(j)) : 0.f;
    }
    for (int base = 0; base < n; base += kStep) {
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const float x = v[u];
        const int jn = base + kStep + threadIdx.x + u * kTopkThreads;
        if (jn < n) v[u] = __ldcs(src + tok(jn));
        const int j = base + threadIdx.x + u * kTopkThreads;
        f(j < n, j, order_key(x), x);
      }
    }
  }
};

// Keys computed from the label cache: the fused score + select path.  Scores
// are computed exactly as k_score_vec computes them (same order of fp32
// operations), r/8 lanes per row so that every warp load reads 512 contiguous
// bytes, with the next slice's loads in flight while a slice is consumed.
template <int R, int kSlotsT = 4>
struct LabelSource {
  const uint16_t* Q;
  const int32_t* C;
  const uint16_t* label;
  float* scores;  // optional output
  int Hq, T_cap;
  int over_t = -1;                  // this token's row is taken from over_row,
  const uint4* over_row = nullptr;  // not from the label cache (a row written
                                    // by the same kernel)
  static constexpr int kLanes = R / 8;
  static constexpr int kRowsPerInstr = 32 / kLanes;
  static constexpr int kSlots = kSlotsT;  // 16-byte loads in flight per thread
  static constexpr int kStep = kTopkWarps * kSlots * kRowsPerInstr;  // items per slice

  __device__ __forceinline__ void prepare(int bh, float* qs) const {
    load_qc(Q, C, bh, bh % Hq, R, qs);
  }
  __device__ __forceinline__ float* scores_out(int bh, int T) const {
    return scores ? scores + (size_t)bh * T : nullptr;
  }
  __device__ __forceinline__ int slot_item(int base, int i) const {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    return base + (warp * kSlots + i) * kRowsPerInstr + lane / kLanes;
  }
  // Rolling buffer: slot i of the next slice is loaded as soon as slot i of
  // this slice has been taken, so kSlots loads stay in flight per thread.
  template <class Tok, class F>
  __device__ __forceinline__ void stream(int bh, int, int n, Tok tok, F&& f,
                                         const float* qs) const {
    const uint4* lab = reinterpret_cast<const uint4*>(label + (size_t)bh * T_cap * R);
    const int chunk = (threadIdx.x & 31) % kLanes;
    uint4 v[kSlots];
#pragma unroll
    for (int i = 0; i < kSlots; ++i) {
      const int j = slot_item(0, i);
      if (j < n) v[i] = ldg_stream(lab + (size_t)tok(j) * kLanes + chunk);
    }
    for (int base = 0; base < n; base += kStep) {
#pragma unroll
      for (int i = 0; i < kSlots; ++i) {
        uint4 x = v[i];
        const int jn = slot_item(base + kStep, i);
        if (jn < n) v[i] = ldg_stream(lab + (size_t)tok(jn) * kLanes + chunk);
        const int j = slot_item(base, i);
        if (over_t >= 0 && j < n && tok(j) == over_t) x = over_row[chunk];
        const float s = lane_group_score<R>(x, qs, chunk);  // all lanes take part
        f(j < n && chunk == 0, j, order_key(s), s);
      }
    }
  }
};

// The key of rank r (1 = largest) among the ns <= kRankCount keys of a list
// (16-byte aligned, zero-padded to a multiple of 64; zero is below every key
// of a non-NaN score): each key's counts of larger and equal keys, split over
// P threads when the list is short.  Writes misc[M_THR] (the key) and
// misc[M_NEED] (its rank among the keys equal to it).  scratch: 2*kTopkThreads
// words.  Block-uniform; ends with a barrier.
__device__ __forceinline__ void rank_in_list(const uint32_t* sk, int ns, uint32_t r,
                                             uint32_t* scratch, uint32_t* misc) {
  const int P = ns <= 64 ? 4 : (ns <= 128 ? 2 : 1);
  const int per = kTopkThreads / P;
  const int i = threadIdx.x % per, part = threadIdx.x / per;
  const int span = ((ns + 63) & ~63) / P;
  uint32_t* pgt = scratch;
  uint32_t* peq = scratch + kTopkThreads;
  if (i < ns) {
    const uint32_t mine = sk[i];
    uint32_t gt = 0u, eq = 0u;
    const uint4* v = reinterpret_cast<const uint4*>(sk + part * span);
    for (int j = 0; j < span / 4; j += 4) {
      const uint4 x[4] = {v[j], v[j + 1], v[j + 2], v[j + 3]};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        gt += (x[q].x > mine ? 1u : 0u) + (x[q].y > mine ? 1u : 0u) +
              (x[q].z > mine ? 1u : 0u) + (x[q].w > mine ? 1u : 0u);
        eq += (x[q].x == mine ? 1u : 0u) + (x[q].y == mine ? 1u : 0u) +
              (x[q].z == mine ? 1u : 0u) + (x[q].w == mine ? 1u : 0u);
      }
    }
    pgt[threadIdx.x] = gt;
    peq[threadIdx.x] = eq;
  }
  __syncthreads();
  if (threadIdx.x < ns) {
    uint32_t gt = 0u, eq = 0u;
    for (int q = 0; q < P; ++q) {
      gt += pgt[q * per + threadIdx.x];
      eq += peq[q * per + threadIdx.x];
    }
    if (gt < r && r <= gt + eq) {  // every thread holding the result's value
      misc[M_THR] = sk[threadIdx.x];
      misc[M_NEED] = r - gt;
    }
  }
  __syncthreads();
}

// Called once for every token a whole-head list select settles on before the
// exact threshold is known: at some digit its key is in a higher bin than the
// k-th key's, all digits above being equal (token t: item t of the key array).
struct NoSureHook {
  __device__ __forceinline__ void operator()(int) const {}
};

// List select: the key of rank r (1 = largest) among the live items of a key
// array in shared memory.  Source item i < n has key key0[i] and token tok0(i);
// the live items are those that carry the prefix pf above bit `top` (top = 32:
// every item), and r is at most their number.  When the caller already has the
// first digit's bin, the count above it and its count (first_bin >= 0; the
// digit is first_bits wide), the first histogram is skipped.  With kCls, live items above the result set
// their token's bit in gtm and live items equal to it in eqm (tokens of
// [c0, c0 + len) only; bit t - c0); kSeqTok: tok0(i) == i, and c0 is a multiple
// of 32.  n <= 4 * kSelectIters * kTopkThreads, key0 16-byte aligned, and key0
// readable up to n rounded up to 4.  need: the result's rank among the keys
// equal to it.  misc[M_LIST] is zero on entry and on exit.  on_sure: see
// NoSureHook (kCls && kSeqTok).  Block-uniform.
template <bool kCls, bool kSeqTok, class TokFn, class SureHook = NoSureHook>
__device__ __forceinline__ uint32_t list_select(const uint32_t* key0, TokFn tok0, int n, int top,
                                                uint32_t pf, uint32_t r, int first_bits,
                                                int first_bin, uint32_t first_above,
                                                uint32_t first_cnt,
                                                uint32_t* hist, uint32_t* lists, uint32_t* misc,
                                                uint32_t* gtm, uint32_t* eqm, int c0, int len,
                                                uint32_t& need,
                                                const SureHook& on_sure = SureHook()) {
  const int lane = threadIdx.x & 31;
  const uint32_t* sk = key0;
  const uint32_t* st = nullptr;  // tokens of the current list (null: the source array)
  int ns = n, buf = 0;
  auto token = [&](int i) -> int { return st ? (int)st[i] : tok0(i); };
  auto mark = [&](uint32_t* m, int t) {
    const int j = t - c0;
    if (j >= 0 && j < len) atomicOr(&m[j >> 5], 1u << (j & 31));
  };
  auto live = [&](uint32_t key) { return top >= 32 || (key >> top) == pf; };

  while (!(st && ns <= kRankCount) && top > 0) {
    const int bits = first_bin >= 0 ? first_bits : (top < 11 ? top : 11);
    const int sh = top - bits;
    const uint32_t nb = 1u << bits;
    uint32_t bin, above, cnt;
    if (first_bin >= 0) {
      bin = (uint32_t)first_bin;
      above = first_above;
      cnt = first_cnt;
      first_bin = -1;
    } else {
      for (int i = threadIdx.x; i < (int)nb; i += kTopkThreads) hist[i] = 0u;
      __syncthreads();
      for (int i = threadIdx.x; i < ns; i += kTopkThreads) {
        const uint32_t key = sk[i];
        if (live(key)) atomicAdd(&hist[(key >> sh) & (nb - 1)], 1u);
      }
      __syncthreads();
      find_bin(hist, (int)nb, r, misc + 48, misc + M_BIN);
      bin = misc[M_BIN];
      above = misc[M_ABOVE];
      cnt = misc[M_CNT];
    }
    r -= above;
    const bool compact = cnt <= (uint32_t)kListCap;
    uint32_t* dk = lists + buf * 2 * kListCap;
    uint32_t* dt = dk + kListCap;
    // One pass, four consecutive items per thread and load: items above the
    // bin are marked, the bin's items flagged (4 bits per load, in registers);
    // then one slot reservation per warp and the flagged items are copied.
    uint32_t keep = 0u;  // bit 4*it + u: item it*4*kTopkThreads + 4*threadIdx.x + u
#pragma unroll
    for (int it = 0; it < kSelectIters; ++it) {
      if (it * 4 * kTopkThreads < ns) {
        const int i0 = it * 4 * kTopkThreads + 4 * threadIdx.x;
        const uint4 kv = *reinterpret_cast<const uint4*>(sk + i0);
        const uint32_t kk[4] = {kv.x, kv.y, kv.z, kv.w};
        uint32_t up = 0u;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const bool lv = i0 + u < ns && live(kk[u]);
          const uint32_t dg = (kk[u] >> sh) & (nb - 1);
          if (lv && dg > bin) up |= 1u << u;
          if (lv && dg == bin) keep |= 1u << (4 * it + u);
        }
        if (kCls) {
          if (kSeqTok && !st) {
            // tokens i0..i0+3; eight lanes make one 32-token mask word
            uint32_t wm = up << (4 * (lane & 7));
            wm |= __shfl_xor_sync(0xffffffffu, wm, 1);
            wm |= __shfl_xor_sync(0xffffffffu, wm, 2);
            wm |= __shfl_xor_sync(0xffffffffu, wm, 4);
            const int j = i0 - 4 * (lane & 7) - c0;
            if ((lane & 7) == 0 && wm && j >= 0 && j < len) gtm[j >> 5] |= wm;
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if ((up >> u) & 1u) on_sure(i0 + u);
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if ((up >> u) & 1u) mark(gtm, token(i0 + u));
          }
        }
      }
    }
    if (compact) {
      const uint32_t c = __popc(keep);
      uint32_t incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      uint32_t base = 0u;
      if (lane == 31 && incl) base = atomicAdd(&misc[M_LIST], incl);
      base = __shfl_sync(0xffffffffu, base, 31) + incl - c;
      while (keep) {
        const int b = __ffs(keep) - 1;
        keep &= keep - 1u;
        const int i = (b >> 2) * 4 * kTopkThreads + 4 * threadIdx.x + (b & 3);
        dk[base] = sk[i];
        if (kCls) dt[base] = (uint32_t)token(i);
        ++base;
      }
      // zero keys (below every key of a non-NaN score) pad the list to a
      // multiple of 64 for the rank count
      if (threadIdx.x < 64 && cnt + threadIdx.x < (uint32_t)kListCap) dk[cnt + threadIdx.x] = 0u;
    }
    __syncthreads();
    pf = (pf << bits) | bin;
    top = sh;
    if (compact) {
      sk = dk;
      st = dt;
      ns = (int)cnt;
      buf ^= 1;
      if (threadIdx.x == 0) misc[M_LIST] = 0u;  // next used after a barrier
    }
  }

  uint32_t thr;
  if (st && ns <= kRankCount) {
    rank_in_list(sk, ns, r, lists + buf * 2 * kListCap, misc);  // the list buffer not in use
    thr = misc[M_THR];
    need = misc[M_NEED];
  } else {  // every bit fixed: the live items all equal the prefix
    thr = pf;
    need = r;
  }
  if (kCls) {
    for (int i = threadIdx.x; i < ns; i += kTopkThreads) {
      const uint32_t key = sk[i];
      if (!live(key)) continue;
      if (key > thr)
        mark(gtm, token(i));
      else if (key == thr)
        mark(eqm, token(i));
    }
  }
  __syncthreads();
  return thr;
}

// The streaming passes of the kernel below.

// Sample pass (block-uniform): keys of the m sampled tokens into keys[], the
// histogram of their top 32 - hshift bits into hist; scores of this CTA's
// tokens when the whole head is the sample.
template <class Source>
__device__ __forceinline__ void sample_pass(const Source& src, int bh, int T, int m, bool whole,
                                         uint32_t* keys, uint32_t* hist, int hshift,
                                         float* scores_out, int c0, int len, const float* qs) {
  const int q32 = T >> 5;
  auto tok = [whole, q32](int j) {
    return whole ? j : ((int)((long long)(j >> 5) * q32 / kSampleBlocks) << 5) + (j & 31);
  };
  src.stream(bh, T, m, tok,
             [&](bool v, int j, uint32_t key, float s) {
               if (v) {
                 keys[j] = key;
                 if (whole && scores_out && j >= c0 && j < c0 + len) scores_out[j] = s;
               }
             },
             qs);
  // the histogram from shared memory once every key is in: no shared-memory
  // atomics between the loads of the stream
  __syncthreads();
  for (int j = threadIdx.x; j < m; j += kTopkThreads) atomicAdd(&hist[keys[j] >> hshift], 1u);
}

// Main pass over this CTA's tokens against the bracket [lo, hi].
template <class Source>
__device__ __forceinline__ void classify_pass(const Source& src, int bh, int T, int c0, int len,
                                           uint32_t lo, uint32_t hi, float* scores_out,
                                           uint32_t* gtm, uint32_t* eqm, uint32_t* cand_key,
                                           uint32_t* cand_tok, uint32_t* ncand,
                                           const float* qs) {
  const bool one = lo == hi;
  auto tok = [c0](int j) { return c0 + j; };
  src.stream(bh, T, len, tok,
             [&](bool v, int j, uint32_t key, float s) {
               if (!v) return;
               if (scores_out) scores_out[c0 + j] = s;
               const uint32_t bit = 1u << (j & 31);
               if (key > hi) {
                 atomicOr(&gtm[j >> 5], bit);
               } else if (key >= lo) {
                 if (one) {
                   atomicOr(&eqm[j >> 5], bit);
                 } else {
                   const uint32_t slot = atomicAdd(ncand, 1u);
                   if (slot < kCandCap) {
                     cand_key[slot] = key;
                     cand_tok[slot] = (uint32_t)j;
                   }
                 }
               }
             },
             qs);
}

// Refinement pass: histogram of digit d of this CTA's keys that carry the
// prefix pf of the digits above d.
template <class Source>
__device__ __forceinline__ void digit_hist_pass(const Source& src, int bh, int T, int c0, int len,
                                             int d, uint32_t pf, uint32_t* hist,
                                             const float* qs) {
  const int hs = d > 0 ? digit_shift(d - 1) : 0;
  const int sh = digit_shift(d);
  const uint32_t mask = (uint32_t)digit_bins(d) - 1u;
  auto tok = [c0](int j) { return c0 + j; };
  src.stream(bh, T, len, tok,
             [&](bool v, int, uint32_t key, float) {
               if (v && (d == 0 || (key >> hs) == pf)) atomicAdd(&hist[(key >> sh) & mask], 1u);
             },
             qs);
}

// The selection of one head by one CTA of its cluster (cs CTAs, this one of
// rank `rank`, shared memory `sm` laid out by TopkLayout(chunk, cs)).  The
// selected indices, ascending, go to dst_g (global, k entries) and/or dst_s
// (shared memory, k entries); either may be null.  qs_ready: the caller has
// already written the source's query values (TopkLayout::small + 64 onwards).
// on_sure: see NoSureHook (called only when T <= kSample).
template <class Source, class SureHook = NoSureHook>
__device__ __forceinline__ void topk_body(const Source& src, uint32_t* sm, int cs, int rank,
                                          int bh, int T, int k, int chunk, int32_t* dst_g,
                                          int32_t* dst_s, bool qs_ready = false,
                                          const SureHook& on_sure = SureHook()) {
  const TopkLayout L(chunk, cs);
  uint32_t* hist = sm;
  uint32_t* misc = sm + L.small;
  uint32_t* warp_gt = misc + 32;
  uint32_t* warp_eq = misc + 40;
  float* qs = reinterpret_cast<float*>(misc + 64);
  uint32_t* gtm = sm + L.masks;
  uint32_t* eqm = gtm + chunk / 32;
  uint32_t* cand_key = sm + L.X;  // also the sample keys while sampling
  uint32_t* cand_tok = cand_key + kCandCap;

  const int c0 = min(rank * chunk, T);
  const int len = min(chunk, T - c0);
  const int groups = (len + 31) >> 5;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* scores_out = src.scores_out(bh, T);

  for (int i = threadIdx.x; i < L.small + 64; i += kTopkThreads) sm[i] = 0u;
  for (int i = threadIdx.x; i < 2 * (chunk / 32); i += kTopkThreads) gtm[i] = 0u;
  if (cs == 1) {  // the wide sample histogram (below)
    uint4* z = reinterpret_cast<uint4*>(cand_tok);
    for (int i = threadIdx.x; i < kWideBins / 4; i += kTopkThreads) z[i] = make_uint4(0, 0, 0, 0);
  }
  if (!qs_ready) src.prepare(bh, qs);
  // every CTA of the cluster is running and its counters are zero before any
  // remote access
  cluster_or_cta_sync(cs);

  // ---- 1. sample ---------------------------------------------------------------
  // one CTA: a 13-bit histogram over the candidate-token half and the lists
  // (free until the bracket is known); a cluster: the 11-bit one
  const bool whole = T <= kSample;
  const int m = whole ? T : kSample;
  const bool wide = cs == 1;
  uint32_t* hist0 = wide ? cand_tok : hist;
  const int hbits = wide ? kWideBits : digit_bits(0);
  if (cs > 1 && !whole) {
    // a cluster: each CTA computes the keys of its share of the sample's
    // blocks, then copies the other shares from the other CTAs' shared memory
    cg::cluster_group cl = cg::this_cluster();
    const int nblk = m / 32;
    auto share = [&](int c, int& a, int& b) {
      a = (c * nblk / cs) * 32;
      b = ((c + 1) * nblk / cs) * 32;
    };
    int j0, j1;
    share(rank, j0, j1);
    const int q32 = T >> 5;
    src.stream(bh, T, j1 - j0,
               [&](int j) {
                 const int jj = j0 + j;
                 return ((int)((long long)(jj >> 5) * q32 / kSampleBlocks) << 5) + (jj & 31);
               },
               [&](bool v, int j, uint32_t key, float) {
                 if (v) cand_key[j0 + j] = key;
               },
               qs);
    cl.sync();  // every share is written
    for (int c = 0; c < cs; ++c) {
      if (c == rank) continue;
      int a, b;
      share(c, a, b);
      const uint4* rk = reinterpret_cast<const uint4*>(cl.map_shared_rank(cand_key, c));
      uint4* lk = reinterpret_cast<uint4*>(cand_key);
      for (int i = a / 4 + threadIdx.x; i < b / 4; i += kTopkThreads) lk[i] = rk[i];
    }
    cl.sync();  // every copy is done before any CTA reuses its keys
    for (int j = threadIdx.x; j < m; j += kTopkThreads)
      atomicAdd(&hist0[cand_key[j] >> (32 - hbits)], 1u);
  } else {
    sample_pass(src, bh, T, m, whole, cand_key, hist0, 32 - hbits, scores_out, c0, len, qs);
  }
  __syncthreads();

  // ---- 2. bracket ----------------------------------------------------------------
  uint32_t lo, hi;
  uint32_t* lists = sm + L.lists;
  uint32_t need_unused;
  if (whole) {
    // exact threshold over every key of the head; this CTA's tokens are
    // classified on the way
    if (wide)
      find_bins_wide<kWideBins / kTopkThreads>(hist0, (uint32_t)k, 0u, misc + 48, misc + M_BIN,
                                               misc + M_BIN);
    else
      find_bin(hist0, 2048, (uint32_t)k, misc + 48, misc + M_BIN);
    const int b0 = (int)misc[M_BIN];
    const uint32_t a0 = misc[M_ABOVE], n0 = misc[M_CNT];
    const uint32_t thr = list_select<true, true>(
        cand_key, [](int i) { return i; }, T, 32, 0u, (uint32_t)k, hbits, b0, a0, n0, hist,
        lists, misc, gtm, eqm, c0, len, need_unused, on_sure);
    lo = hi = thr;
  } else {
    const float e = (float)k * (float)m / (float)T;
    const float sd = sqrtf(e * (1.f - (float)k / (float)T));
    const float margin = kBracketSigmas * sd + 2.f;
    const int r_hi = (int)floorf(e - margin), r_lo = (int)ceilf(e + margin);
    const uint32_t rh = r_hi >= 1 ? (uint32_t)r_hi : 0u, rl = r_lo <= m ? (uint32_t)r_lo : 0u;
    if (wide)
      find_bins_wide<kWideBins / kTopkThreads>(hist0, rh, rl, misc + 48, misc + M_BIN,
                                               misc + M_BIN2);
    else
      find_bins(hist0, 2048, rh, rl, misc + 48, misc + M_BIN, misc + M_BIN2);
    const int bh0 = (int)misc[M_BIN], bl0 = (int)misc[M_BIN2];
    const uint32_t ah = misc[M_ABOVE], nh = misc[M_CNT], al = misc[M_ABOVE2], nl = misc[M_CNT2];
    auto no_tok = [](int) { return 0; };
    if (cs > 1) {
      // a cluster: CTA 0 selects hi and CTA 1 lo at the same time, and each
      // writes its key into every CTA's misc[M_HI + rank]
      cg::cluster_group cl = cg::this_cluster();
      uint32_t key = 0u;
      const bool mine = (rank == 0 && rh) || (rank == 1 && rl);
      if (rank == 0 && rh)
        key = list_select<false, false>(cand_key, no_tok, m, 32, 0u, rh, hbits, bh0, ah, nh, hist,
                                        lists, misc, gtm, eqm, c0, len, need_unused);
      else if (rank == 1 && rl)
        key = list_select<false, false>(cand_key, no_tok, m, 32, 0u, rl, hbits, bl0, al, nl, hist,
                                        lists, misc, gtm, eqm, c0, len, need_unused);
      if (mine && threadIdx.x == 0)
        for (int c = 0; c < cs; ++c) cl.map_shared_rank(misc, c)[M_HI + rank] = key;
      cl.sync();
      hi = rh ? misc[M_HI] : 0xffffffffu;
      lo = rl ? misc[M_LO] : 0u;
    } else {
      hi = rh ? list_select<false, false>(cand_key, no_tok, m, 32, 0u, rh, hbits, bh0, ah, nh,
                                          hist, lists, misc, gtm, eqm, c0, len, need_unused)
              : 0xffffffffu;
      lo = rl ? list_select<false, false>(cand_key, no_tok, m, 32, 0u, rl, hbits, bl0, al, nl,
                                          hist, lists, misc, gtm, eqm, c0, len, need_unused)
              : 0u;
    }
  }

  // ---- 3/4. stream and check; exact refinement if the bracket fails -----------
  int level = 0;  // refinement digits done
  uint32_t prefix = 0, krem = (uint32_t)k;
  for (;;) {
    const bool one = lo == hi;
    if (whole && level == 0) {
      // classified by the select above
    } else {
      classify_pass(src, bh, T, c0, len, lo, hi, level == 0 ? scores_out : nullptr, gtm, eqm,
                    cand_key, cand_tok, &misc[M_NCAND], qs);
    }
    __syncthreads();
    uint32_t n_gt = 0, n_eq = 0;
    for (int g = threadIdx.x; g < groups; g += kTopkThreads) {
      n_gt += __popc(gtm[g]);
      n_eq += __popc(eqm[g]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      n_gt += __shfl_xor_sync(0xffffffffu, n_gt, o);
      n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
    }
    if (lane == 0) {
      warp_gt[warp] = n_gt;
      warp_eq[warp] = n_eq;
    }
    __syncthreads();
    const uint32_t ncand = misc[M_NCAND];
    uint32_t mine[4] = {0u, 0u, ncand, ncand > (uint32_t)kCandCap ? 1u : 0u};
    for (int w = 0; w < kTopkWarps; ++w) {
      mine[0] += warp_gt[w];
      mine[1] += warp_eq[w];
    }
    cluster_totals(misc, mine, cs);
    const uint32_t tot_gt = misc[M_TOT], tot_eq = misc[M_TOT + 1];
    const uint32_t tot_cand = misc[M_TOT + 2], tot_ovf = misc[M_TOT + 3];
    const bool ok = tot_ovf == 0 && tot_gt < (uint32_t)k &&
                    (uint32_t)k <= tot_gt + (one ? tot_eq : tot_cand);
    __syncthreads();
    if (threadIdx.x == 0)
      for (int i = 0; i < 4; ++i) misc[M_TOT + i] = 0u;  // before the next cluster barrier
    if (ok) {
      krem = (uint32_t)k - tot_gt;
      break;
    }

    // Exact refinement.  The rank sought within the current bracket: k itself
    // while no prefix is fixed (the failed bracket came from the sample), else
    // k minus the keys above the prefix's range.
    krem = level == 0 ? (uint32_t)k : (uint32_t)k - tot_gt;
    const int d = level;
    for (int i = threadIdx.x; i < 2048; i += kTopkThreads) hist[i] = 0u;
    if (cs > 1)
      for (int i = threadIdx.x; i < 4096; i += kTopkThreads) sm[L.merged0 + i] = 0u;
    for (int i = threadIdx.x; i < 2 * (chunk / 32); i += kTopkThreads) gtm[i] = 0u;
    if (threadIdx.x == 0) misc[M_NCAND] = 0u;
    // every CTA has zeroed its merged copies before anyone adds into them
    cluster_or_cta_sync(cs);
    digit_hist_pass(src, bh, T, c0, len, d, prefix, hist, qs);
    __syncthreads();
    const uint32_t* h =
        cluster_hist(hist, sm + (d == 1 ? L.merged1 : L.merged0), digit_bins(d), cs);
    find_bin(h, digit_bins(d), krem, misc + 48, misc + M_BIN);
    prefix = (prefix << digit_bits(d)) | misc[M_BIN];
    ++level;
    lo = prefix << digit_shift(d);
    hi = lo | ((1u << digit_shift(d)) - 1u);
    __syncthreads();
  }

  // ---- 5. resolve within the bracket -------------------------------------------
  uint32_t need = krem;
  if (lo != hi && cs == 1) {
    // the candidates share the bits of lo and hi above their highest differing bit
    const uint32_t ncand = misc[M_NCAND];
    const int top = 32 - __clz(lo ^ hi);
    list_select<true, false>(
        cand_key, [&](int i) { return c0 + (int)cand_tok[i]; }, (int)ncand, top,
        top >= 32 ? 0u : lo >> top, krem, 0, -1, 0u, 0u, hist, lists, misc, gtm, eqm, c0, len,
        need);
  } else if (lo != hi) {
    // a cluster: radix select over the candidates with histograms merged over
    // the cluster, starting at the highest bit where lo and hi differ (every
    // candidate shares the bits above it)
    const uint32_t ncand = misc[M_NCAND];
    int t = 32 - __clz(lo ^ hi);
    uint32_t p = t >= 32 ? 0u : lo >> t, r = krem;
    for (int round = 0; t > 0; ++round) {
      const int bits = t < 11 ? t : 11;
      const int sh = t - bits;
      const int nb = 1 << bits;
      uint32_t* mg = sm + ((round & 1) ? L.merged1 : L.merged0);
      for (int i = threadIdx.x; i < nb; i += kTopkThreads) hist[i] = 0u;
      for (int i = threadIdx.x; i < nb; i += kTopkThreads) mg[i] = 0u;
      cluster_or_cta_sync(cs);
      for (uint32_t s = threadIdx.x; s < ncand; s += kTopkThreads) {
        const uint32_t key = cand_key[s];
        if (t >= 32 || (key >> t) == p) atomicAdd(&hist[(key >> sh) & (nb - 1)], 1u);
      }
      __syncthreads();
      const uint32_t* h = cluster_hist(hist, mg, nb, cs);
      find_bin(h, nb, r, misc + 48, misc + M_BIN);
      p = (p << bits) | misc[M_BIN];
      r -= misc[M_ABOVE];
      __syncthreads();
      t = sh;
    }
    need = r;
    for (uint32_t s = threadIdx.x; s < ncand; s += kTopkThreads) {
      const uint32_t key = cand_key[s], j = cand_tok[s];
      if (key > p)
        atomicOr(&gtm[j >> 5], 1u << (j & 31));
      else if (key == p)
        atomicOr(&eqm[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
  }

  // ---- 6. counts, cluster prefix, write ------------------------------------------
  const int gpw = (groups + kTopkWarps - 1) / kTopkWarps;
  const int g0 = min(warp * gpw, groups), g1 = min(g0 + gpw, groups);
  {
    uint32_t n_gt = 0, n_eq = 0;
    for (int g = g0 + lane; g < g1; g += 32) {
      n_gt += __popc(gtm[g]);
      n_eq += __popc(eqm[g]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      n_gt += __shfl_xor_sync(0xffffffffu, n_gt, o);
      n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
    }
    if (lane == 0) {
      warp_gt[warp] = n_gt;
      warp_eq[warp] = n_eq;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t a = 0, e = 0;
    for (int w = 0; w < kTopkWarps; ++w) {
      a += warp_gt[w];
      e += warp_eq[w];
    }
    if (cs > 1) {  // push this CTA's counts into every later CTA of the cluster
      cg::cluster_group cl = cg::this_cluster();
      for (int c = rank + 1; c < cs; ++c) {
        uint32_t* mm = cl.map_shared_rank(misc, c);
        atomicAdd(mm + M_GT_BEFORE, a);
        atomicAdd(mm + M_EQ_BEFORE, e);
      }
    }
  }
  cluster_or_cta_sync(cs);

  uint32_t gt_before = misc[M_GT_BEFORE], eq_before = misc[M_EQ_BEFORE];
  for (int w = 0; w < warp; ++w) {
    gt_before += warp_gt[w];
    eq_before += warp_eq[w];
  }

  // 32 groups per step, one per lane; warp scans give each group its first tie
  // rank and its first output position.
  uint32_t tie = eq_before;
  uint32_t out = gt_before + min(eq_before, need);
  for (int base = g0; base < g1; base += 32) {
    const int g = base + lane;
    const uint32_t gmask = g < g1 ? gtm[g] : 0u;
    const uint32_t emask = g < g1 ? eqm[g] : 0u;
    const uint32_t ne = __popc(emask);
    uint32_t ne_incl = ne;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, ne_incl, o);
      if (lane >= o) ne_incl += v;
    }
    const uint32_t my_tie = tie + ne_incl - ne;
    const uint32_t take = need > my_tie ? min(need - my_tie, ne) : 0u;  // ties kept here
    uint32_t takem = emask;  // the first `take` set bits of emask
    if (take < ne) {
      uint32_t rest = emask;
      for (uint32_t j = 0; j < take; ++j) rest &= rest - 1u;
      takem = emask ^ rest;
    }
    uint32_t selm = gmask | takem;
    const uint32_t n = __popc(selm);
    uint32_t n_incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, n_incl, o);
      if (lane >= o) n_incl += v;
    }
    uint32_t pos = out + n_incl - n;
    while (selm) {
      const int b = __ffs(selm) - 1;
      selm &= selm - 1u;
      if (pos < (uint32_t)k) {
        if (dst_g) dst_g[pos] = c0 + g * 32 + b;
        if (dst_s) dst_s[pos] = c0 + g * 32 + b;
      }
      ++pos;
    }
    tie += __shfl_sync(0xffffffffu, ne_incl, 31);
    out += __shfl_sync(0xffffffffu, n_incl, 31);
  }
}

// grid (CS, BH), cluster (CS, 1, 1).  chunk: tokens per CTA, a multiple of 32.
template <class Source>
__global__ void __launch_bounds__(kTopkThreads, 3)  // three CTAs per SM: up to 85 registers
k_topk(Source src, int32_t* __restrict__ idx, int T, int k, int chunk) {
  extern __shared__ __align__(16) uint32_t sm[];
  topk_body(src, sm, (int)gridDim.x, (int)blockIdx.x, (int)blockIdx.y, T, k, chunk,
            idx + (size_t)blockIdx.y * k, nullptr);
}

}  // namespace ds

namespace ds {

// ---- hierarchical top-k ------------------------------------------------------
// Page "A Training-free Sub-quadratic Cost Transformer Model Serving Framework
// With Hierarchically Pruned Attention" (Core idea: attention locality, nearby
// tokens score alike; Technical framework: a hierarchy of tokens searched
// tree-like for each query's important keys).  Reading: k contiguous parts of
// [0, T) are halved level by level (the first half takes the extra token);
// each part is scored by its first token's approximate score; the k best parts
// stay (score descending, start ascending); after the last level the k parts
// are single tokens.  One CTA per head: each level scores its 2k children from
// the label cache (one row each, LabelSource), selects k of them with the list
// select (ties in child order = start order), and compacts the kept children
// into the next level's parts.  About 2k*log2(T/k) label rows are read instead
// of T.
constexpr int kHierMaxK = 2048;

struct HierLayout {
  int nodes0, nodes1, words;  // part starts and ends, two buffers of kHierMaxK each
  __host__ __device__ explicit HierLayout(const TopkLayout& L) {
    nodes0 = L.words;
    nodes1 = nodes0 + 2 * kHierMaxK;
    words = nodes1 + 2 * kHierMaxK;
  }
  __host__ __device__ size_t bytes() const { return (size_t)words * 4; }
};

// grid (BH), block kTopkThreads; shared memory HierLayout(TopkLayout(2k rounded
// up to 32, 1)).  idx: [BH, k] out, ascending.
template <class Source>
__global__ void __launch_bounds__(kTopkThreads, 2)
k_hier_topk(Source src, int32_t* __restrict__ idx, int T, int k) {
  extern __shared__ __align__(16) uint32_t sm[];
  const int n = 2 * k;  // children per level
  const int chunk = (n + 31) & ~31;
  const TopkLayout L(chunk, 1);
  const HierLayout H(L);
  const int bh = blockIdx.x;
  uint32_t* hist = sm;
  uint32_t* misc = sm + L.small;
  float* qs = reinterpret_cast<float*>(misc + 64);
  uint32_t* gtm = sm + L.masks;
  uint32_t* eqm = gtm + chunk / 32;
  uint32_t* keys = sm + L.X;
  uint32_t* lists = sm + L.lists;
  int32_t* ps = reinterpret_cast<int32_t*>(sm + H.nodes0);  // part starts
  int32_t* pe = ps + kHierMaxK;                               // part ends
  int32_t* qs2 = reinterpret_cast<int32_t*>(sm + H.nodes1);
  int32_t* qe2 = qs2 + kHierMaxK;

  for (int i = threadIdx.x; i < L.small + 64; i += kTopkThreads) sm[i] = 0u;
  for (int i = threadIdx.x; i < k; i += kTopkThreads) {
    ps[i] = (int)(((long long)i * T) / k);
    pe[i] = (int)(((long long)(i + 1) * T) / k);
  }
  src.prepare(bh, qs);
  __syncthreads();

  int maxlen = (T + k - 1) / k;
  const int groups = chunk / 32;
  while (maxlen > 1) {
    // child j of part j/2: the first or second half, or nothing (a part of one
    // token has one child)
    auto child = [&](int j, int& b, int& e) {
      const int i = j >> 1;
      const int pb = ps[i], pe_ = pe[i];
      if (pe_ - pb > 1) {
        const int m = pb + (pe_ - pb + 1) / 2;
        b = (j & 1) ? m : pb;
        e = (j & 1) ? pe_ : m;
      } else {
        b = pb;
        e = (j & 1) ? pb : pe_;  // empty second child
      }
    };
    src.stream(bh, T, n,
               [&](int j) {
                 int b, e;
                 child(j, b, e);
                 return b;
               },
               [&](bool v, int j, uint32_t key, float) {
                 if (v) {
                   int b, e;
                   child(j, b, e);
                   keys[j] = e > b ? key : 0u;  // zero: below every key of a non-NaN score
                 }
               },
               qs);
    for (int i = threadIdx.x; i < 2 * groups; i += kTopkThreads) gtm[i] = 0u;
    __syncthreads();
    uint32_t need;
    list_select<true, true>(keys, [](int i) { return i; }, n, 32, 0u, (uint32_t)k, 0, -1, 0u,
                            0u, hist, lists, misc, gtm, eqm, 0, n, need);
    // kept children in child order: all above the threshold, and the first
    // `need` equal to it
    uint32_t ne = 0u, ng = 0u, gm = 0u, em = 0u;
    if (threadIdx.x < groups) {
      gm = gtm[threadIdx.x];
      em = eqm[threadIdx.x];
      ne = __popc(em);
    }
    const uint32_t tie = block_exclusive_scan(ne, misc + 48);
    __syncthreads();
    uint32_t sel = gm;
    if (threadIdx.x < groups && need > tie) {
      const uint32_t take = min(need - tie, ne);
      uint32_t rest = em;
      for (uint32_t t = 0; t < take; ++t) rest &= rest - 1u;
      sel |= em ^ rest;
    }
    ng = __popc(sel);
    uint32_t pos = block_exclusive_scan(ng, misc + 48);
    while (sel) {
      const int bit = __ffs(sel) - 1;
      sel &= sel - 1u;
      int b, e;
      child(threadIdx.x * 32 + bit, b, e);
      if (pos < (uint32_t)k) {
        qs2[pos] = b;
        qe2[pos] = e;
      }
      ++pos;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < k; i += kTopkThreads) {
      ps[i] = qs2[i];
      pe[i] = qe2[i];
    }
    __syncthreads();
    maxlen = (maxlen + 1) / 2;
  }
  for (int i = threadIdx.x; i < k; i += kTopkThreads) idx[(size_t)bh * k + i] = ps[i];
}

}  // namespace ds
