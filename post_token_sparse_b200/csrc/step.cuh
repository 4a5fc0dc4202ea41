// One whole decode step per query head in one launch: label row of the newest
// token, channel-sparse score + top-k selection, and exact attention over the
// kept tokens (Double Sparsity: channel sparsity picks the tokens -- Method
// details: Core idea, Key design -- and self-attention runs over them only --
// Abstract, Key points 2).
//
// One CTA of kTopkThreads threads per query head, for heads whose selection
// fits one CTA.  Phases, all on chip:
//   1. append   the r label channels of the newest token's K row (t = T-1) are
//               gathered into shared memory and written to the label cache;
//               the selection reads that row from shared memory, so the kernel
//               never reads back through the non-coherent load path a row it
//               wrote itself.  When the caller hands over the newest token's K
//               and V rows (K_new, V_new), they are also stored into the K and V
//               caches here, and the label channels and token T-1's attention
//               rows are read from K_new / V_new
//   2. select   heads of at most kStepWholeT tokens: every key in shared
//               memory, then an exact radix select (12-bit histogram of all
//               keys, 12- and 8-bit histograms of the boundary bin's keys) and
//               one block scan that places the kept tokens and ranks the ties
//               (select_whole below); longer heads: the top-k body of
//               topk.cuh.  The k indices land in shared memory (and in idx
//               when requested)
//   3. attend   8 warps each take a contiguous run of the kept rows through a
//               per-warp cp.async ring (as k_attend does), online softmax in the
//               log2 domain, warp then CTA merge -> O and lse.
#pragma once

#include "attend.cuh"
#include "select.cuh"
#include "topk.cuh"

namespace ds {

constexpr int kStepWarps = kTopkThreads / 32;  // 8
static_assert(kTopkThreads >= kHeadDim + 48,
              "threads d..d+31 store the new K and V rows, d+32..d+47 load the query row");
constexpr int kStepStages = 3;
constexpr int kStepMaxK = 8192;
constexpr int kStepWholeT = 4096;  // heads selected by select_whole: 16 tokens a thread
constexpr int kStepTokPerThread = kStepWholeT / kTopkThreads;
static_assert(kTopkThreads == kSelThreads, "select_whole uses the selector's block scan");
// shared memory of select_whole, in words: keys, histogram, scan scratch, results
constexpr int kWholeWords = kStepWholeT + 4096 + 16 + 16;
// bin tokens ranked by direct counting (above that: the remaining digits by histograms)
constexpr int kWholeList = 512;
static_assert(2 * kWholeList + kStepWholeT / 32 <= 4096, "list and bitmap fit the histogram");

struct StepParams {
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  const uint16_t* K_new;  // optional: the newest token's K and V rows [B*Hkv, d],
  const uint16_t* V_new;  // stored into the caches at T-1 by this kernel
  const int32_t* C;
  uint16_t* label;
  int32_t* idx;  // optional copy of the selected indices [BH, k]
  float* O;
  float* lse;    // optional
  int Hq, Hkv, T_cap, T, k, append;
  int prefetch;  // K and V are in device memory: rows sure to be kept are
                 // prefetched into L2 while the selection finishes
  float scale_log2;
};

// The K and V rows of the tokens the selection has already settled on are
// asked into L2 (two 128-byte lines per 256-byte row), so that the attention
// phase finds most of its rows there instead of waiting on HBM after the
// selection; the HBM reads overlap the selection's on-chip work.
struct PrefetchSureRows {
  const uint16_t* K;  // row 0 of this KV head; null: no prefetch
  const uint16_t* V;
  __device__ __forceinline__ void operator()(int t) const {
    if (K == nullptr) return;
    const char* k = reinterpret_cast<const char*>(K + (size_t)t * kHeadDim);
    const char* v = reinterpret_cast<const char*>(V + (size_t)t * kHeadDim);
    prefetch_l2_line(k);
    prefetch_l2_line(k + 128);
    prefetch_l2_line(v);
    prefetch_l2_line(v + 128);
  }
};

// Shared memory of the step kernel in 32-bit words: the selection's layout,
// overlaid afterwards by the attention ring and warp partials; then the new
// token's label row, the query row and the index list, which outlive the
// selection.
struct StepLayout {
  int over, q, idx, words;
  __host__ __device__ StepLayout(int chunk, int k) {
    int sel = TopkLayout(chunk, 1).words;
    const int whole = TopkLayout(chunk, 1).small + 192 + kWholeWords;  // after q at the
    if (sel < whole) sel = whole;                                         // label channels
    const int att = kStepWarps * kStepStages * kAttnStageU4 * 4 + kStepWarps * 132;
    int o = sel > att ? sel : att;
    o = (o + 3) & ~3;
    over = o;  // label row of the newest token (up to 128 bf16 = 64 words)
    o += 64;
    q = o;  // the query row (128 bf16)
    o += 64;
    idx = o;
    o += (k + 3) & ~3;
    words = o;
  }
  __host__ __device__ size_t bytes() const { return (size_t)words * 4; }
};

// The threads that run a phase (here the whole CTA): tid() is the index in the
// group, sync() a barrier over the group.
struct WholeCta {
  __device__ __forceinline__ int tid() const { return threadIdx.x; }
  __device__ __forceinline__ void sync() const { __syncthreads(); }
};

// Inclusive prefix over a group of kTopkThreads threads, in order; *total: the
// sum.  scratch: 8 words, not rewritten before the group's next barrier.
template <class Grp>
__device__ __forceinline__ uint32_t grp_scan(const Grp& gr, uint32_t v, uint32_t* scratch,
                                             uint32_t* total) {
  const int t = gr.tid(), lane = t & 31, w = t >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) scratch[w] = incl;
  gr.sync();
  uint32_t base = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < kTopkThreads / 32; ++i) {
    const uint32_t x = scratch[i];
    if (i < w) base += x;
    tot += x;
  }
  *total = tot;
  return base + incl;
}

// Attention of one query (head bh) over rows idx_s[0..n) of K and V (KV head
// bkv), by the kStepWarps warps of group gr; writes O[bh] and lse[bh].
template <class Grp = WholeCta, int kStages = kStepStages>
__device__ __forceinline__ void attend_rows(const StepParams& p, int bh, int bkv,
                                            const int32_t* idx_s, int n, uint4* ring,
                                            float* red, const uint4* qrow,
                                            const Grp& gr = Grp()) {
  const int warp = gr.tid() >> 5, lane = gr.tid() & 31;
  const int g = lane >> 3, c = lane & 7;
  float q[16];
  {
    const uint4 a = qrow[c], bq = qrow[8 + c];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      q[2 * i] = bf_lo(w[i]) * p.scale_log2;
      q[2 * i + 1] = bf_hi(w[i]) * p.scale_log2;
    }
  }
  const int rpw = ((n + kStepWarps - 1) / kStepWarps + 3) & ~3;
  const int w_begin = min(warp * rpw, n);
  const int w_end = min(w_begin + rpw, n);
  const int nsteps = (w_end - w_begin + 3) >> 2;
  const size_t kv_base = (size_t)bkv * p.T_cap * kHeadDim;
  const uint16_t* Kh = p.K + kv_base;
  const uint16_t* Vh = p.V + kv_base;
  uint4* my_ring = ring + warp * kStages * kAttnStageU4;

  // with K_new, token T-1's rows are read from there: another CTA of the KV
  // group may not have stored them into the caches yet
  const uint16_t* Knew = p.K_new ? p.K_new + (size_t)bkv * kHeadDim : nullptr;
  const uint16_t* Vnew = p.K_new ? p.V_new + (size_t)bkv * kHeadDim : nullptr;
  auto issue = [&](int step) {
    const int lr = w_begin + step * 4 + g;
    if (lr < w_end) {
      int t = idx_s[lr];
      t = min(max(t, 0), p.T - 1);
      const bool nw = Knew != nullptr && t == p.T - 1;
      const uint4* krow = reinterpret_cast<const uint4*>(nw ? Knew : Kh + (size_t)t * kHeadDim);
      const uint4* vrow = reinterpret_cast<const uint4*>(nw ? Vnew : Vh + (size_t)t * kHeadDim);
      uint4* st = my_ring + (step % kStages) * kAttnStageU4 + g * 32;
      cp_async16(st + c, krow + c);
      cp_async16(st + 8 + c, krow + 8 + c);
      cp_async16(st + 16 + c, vrow + c);
      cp_async16(st + 24 + c, vrow + 8 + c);
    }
  };
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < nsteps) issue(s);
    cp_async_commit();
  }
  float m = -INFINITY, l = 0.f;
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (int s = 0; s < nsteps; ++s) {
    if (s + kStages - 1 < nsteps) issue(s + kStages - 1);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    const uint4* st = my_ring + (s % kStages) * kAttnStageU4 + g * 32;
    const uint4 klo = st[c], khi = st[8 + c];
    float x = dot8(klo, q) + dot8(khi, q + 8);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    online_row(w_begin + s * 4 + g < w_end, x, m, l, acc, st[16 + c], st[24 + c]);
  }
  cp_async_wait<0>();
#pragma unroll
  for (int o = 8; o <= 16; o <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
    const float mn = fmaxf(m, m2);
    const float a1 = rescale(m, mn), a2 = rescale(m2, mn);
    l = l * a1 + l2 * a2;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float other = __shfl_xor_sync(0xffffffffu, acc[i], o);
      acc[i] = acc[i] * a1 + other * a2;
    }
    m = mn;
  }
  float* wr = red + warp * 132;
  if (g == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      wr[4 + c * 8 + i] = acc[i];
      wr[4 + 64 + c * 8 + i] = acc[8 + i];
    }
    if (c == 0) {
      wr[0] = m;
      wr[1] = l;
    }
  }
  gr.sync();
  if (gr.tid() < kHeadDim) {
    const int j = gr.tid();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kStepWarps; ++w) M = fmaxf(M, red[w * 132]);
    float L = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < kStepWarps; ++w) {
      const float a = rescale(red[w * 132], M);
      L = fmaf(red[w * 132 + 1], a, L);
      o = fmaf(red[w * 132 + 4 + j], a, o);
    }
    p.O[(size_t)bh * kHeadDim + j] = o / L;
    if (p.lse && j == 0) p.lse[bh] = (M + log2f(L)) * 0.69314718055994530942f;
  }
}

// In a histogram of nb (256 * q, q a multiple of 4 or 1) bins counted from the
// top, the bin b holding rank r (1 = largest): res[0] = b, res[1] = count
// above b.  Ends with a barrier.
template <class Grp>
__device__ __forceinline__ void whole_find_bin(const Grp& gr, const uint32_t* hist, int nb,
                                               uint32_t r, uint32_t* scan, uint32_t* res) {
  const int q = nb / kTopkThreads;
  const int lo = nb - (gr.tid() + 1) * q;  // this thread's bins lo .. lo+q-1
  uint32_t sum = 0;
#pragma unroll 1
  for (int i = 0; i < q; i += 4) {
    if (q >= 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(hist + lo + i);
      sum += v.x + v.y + v.z + v.w;
    } else {
      sum += hist[lo + i];
    }
  }
  uint32_t tot;
  const uint32_t incl = grp_scan(gr, sum, scan, &tot);
  uint32_t before = incl - sum;
  if (before < r && r <= incl) {
#pragma unroll 1
    for (int i = q - 1; i >= 0; --i) {
      const uint32_t c = hist[lo + i];
      if (before + c >= r) {
        res[0] = (uint32_t)(lo + i);
        res[1] = before;
        break;
      }
      before += c;
    }
  }
  gr.sync();
}

// Top-k of a head of T <= kStepWholeT tokens whose keys are keys[0..T) in
// shared memory: the k largest, ties to the lower token index, ascending into
// dst_s (shared) and dst_g (global, may be null).  Exact: the threshold key is
// fixed digit by digit (bits 31..20 over every key, 19..8 and 7..0 over the
// keys that share the digits above), then every key above it is kept with the
// first ties in token order.  The loops are kept rolled: each CTA runs this
// code once, so its size (instruction fetch) matters more than loop overhead.
template <class Grp>
__device__ __noinline__ void select_whole(const Grp gr, const uint32_t* keys, uint32_t* w, int T,
                                          int k, int32_t* dst_s, int32_t* dst_g) {
  uint32_t* hist = w;             // 4096 bins
  uint32_t* scan = w + 4096;      // 16 words
  uint32_t* res = w + 4096 + 16;  // 16 words
  const int t0 = gr.tid() * kStepTokPerThread;  // this thread's tokens t0 .. t0+15
  // the keys of this thread's tokens, four at a time (f(i, key, valid))
  auto my_keys = [&](auto&& f) {
#pragma unroll 1
    for (int i = 0; i < kStepTokPerThread; i += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(keys + t0 + i);
      const uint32_t kv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) f(i + u, kv[u], t0 + i + u < T);
    }
  };
  // first digit (bits 31..20) over every key: the bin b0 of the k-th key
#pragma unroll 1
  for (int i = gr.tid(); i < 4096; i += kTopkThreads) hist[i] = 0u;
  gr.sync();
#pragma unroll 1
  for (int t = gr.tid(); t < T; t += kTopkThreads) atomicAdd(&hist[keys[t] >> 20], 1u);
  gr.sync();
  whole_find_bin(gr, hist, 4096, (uint32_t)k, scan, res);
  const uint32_t b0 = res[0];
  const uint32_t need = (uint32_t)k - res[1];  // keys of bin b0 kept: 1 .. n0
  const uint32_t n0 = hist[b0];
  gr.sync();  // every thread has read res and hist[b0]
  uint32_t keep = 0u;  // this thread's kept tokens
  if (need == n0) {
    // every key of bin b0 is kept
    my_keys([&](int i, uint32_t key, bool ok) { keep |= (uint32_t)(ok && (key >> 20) >= b0) << i; });
  } else if (n0 <= (uint32_t)kWholeList) {
    // bin b0's keys listed in token order; each kept when fewer than `need` of
    // them are larger or equal and earlier (ties to the lower token)
    uint32_t* lkey = hist;                     // reused: the histogram is read
    uint32_t* ltok = hist + kWholeList;
    uint32_t* kept = hist + 2 * kWholeList;    // bitmap of the kept bin tokens
    uint32_t cm = 0u;
    my_keys([&](int i, uint32_t key, bool ok) {
      keep |= (uint32_t)(ok && (key >> 20) > b0) << i;
      cm |= (uint32_t)(ok && (key >> 20) == b0) << i;
    });
    uint32_t tot;
    uint32_t pos = grp_scan(gr, (uint32_t)__popc(cm), scan + 8, &tot) - (uint32_t)__popc(cm);
    for (int i = gr.tid(); i < kStepWholeT / 32; i += kTopkThreads) kept[i] = 0u;
#pragma unroll 1
    for (uint32_t m = cm; m; m &= m - 1u) {
      const int i = __ffs(m) - 1;
      lkey[pos] = keys[t0 + i];
      ltok[pos] = (uint32_t)(t0 + i);
      ++pos;
    }
    gr.sync();
#pragma unroll 1
    for (int i = gr.tid(); i < (int)n0; i += kTopkThreads) {
      const uint32_t ki = lkey[i];
      uint32_t ahead = 0u;
#pragma unroll 4
      for (int j = 0; j < (int)n0; ++j) {
        const uint32_t kj = lkey[j];
        ahead += (uint32_t)(kj > ki || (kj == ki && j < i));
      }
      if (ahead < need) atomicOr(&kept[ltok[i] >> 5], 1u << (ltok[i] & 31));
    }
    gr.sync();
    keep |= (kept[t0 >> 5] >> (t0 & 31)) & 0xffffu;
  } else {
    // many keys share bin b0: its remaining digits (bits 19..8, then 7..0) by
    // histograms of the keys that carry the prefix, then the ties in token order
    uint32_t r = need, pf = b0;
#pragma unroll 1
    for (int d = 1; d < 3; ++d) {
      const int sh = d == 1 ? 8 : 0;
      const int nb = d == 2 ? 256 : 4096;
      const int hs = d == 1 ? 20 : 8;  // bits above the digit
#pragma unroll 1
      for (int i = gr.tid(); i < nb; i += kTopkThreads) hist[i] = 0u;
      gr.sync();
#pragma unroll 1
      for (int t = gr.tid(); t < T; t += kTopkThreads) {
        const uint32_t key = keys[t];
        if ((key >> hs) == pf) atomicAdd(&hist[(key >> sh) & (uint32_t)(nb - 1)], 1u);
      }
      gr.sync();
      whole_find_bin(gr, hist, nb, r, scan + 8 * (d & 1), res);
      pf = (pf << (d == 2 ? 8 : 12)) | res[0];
      r -= res[1];
      gr.sync();
    }
    const uint32_t thr = pf, need_eq = r;  // the k-th key; ties with it kept: need_eq >= 1
    uint32_t eq = 0u;
    my_keys([&](int i, uint32_t key, bool ok) {
      keep |= (uint32_t)(ok && key > thr) << i;
      eq |= (uint32_t)(ok && key == thr) << i;
    });
    uint32_t tot;
    uint32_t rank = grp_scan(gr, (uint32_t)__popc(eq), scan, &tot) - (uint32_t)__popc(eq);
#pragma unroll 1
    for (uint32_t m = eq; m; m &= m - 1u) {
      if (rank < need_eq) keep |= 1u << (__ffs(m) - 1);
      ++rank;
    }
  }
  // the kept tokens, ascending
  uint32_t tot;
  uint32_t pos = grp_scan(gr, (uint32_t)__popc(keep), scan + 8, &tot) - (uint32_t)__popc(keep);
#pragma unroll 1
  for (uint32_t m = keep; m; m &= m - 1u) {
    const int i = __ffs(m) - 1;
    dst_s[pos] = t0 + i;
    if (dst_g) dst_g[pos] = t0 + i;
    ++pos;
  }
}

// grid (BH), block kTopkThreads.  chunk: T rounded up to a multiple of 32.
template <int R>
__global__ void __launch_bounds__(kTopkThreads, 2)
k_step(const StepParams p, int chunk) {
  extern __shared__ __align__(16) uint32_t sm[];
  const StepLayout SL(chunk, p.k);
  const int bh = blockIdx.x;
  const int G = p.Hq / p.Hkv;
  const int b = bh / p.Hq, h = bh % p.Hq;
  const int bkv = b * p.Hkv + h / G;
  uint16_t* over16 = reinterpret_cast<uint16_t*>(sm + SL.over);
  uint4* q_s = reinterpret_cast<uint4*>(sm + SL.q);
  int32_t* idx_s = reinterpret_cast<int32_t*>(sm + SL.idx);

  // 1. the newest token's label row, and q at the label channels (one load of
  //    each channel id serves both); with K_new, the newest token's K and V
  //    rows are stored into the caches by the KV group's first query head
  float* qs = reinterpret_cast<float*>(sm + TopkLayout(chunk, 1).small + 64);
  {
    const int t = p.T - 1;
    const size_t cache_row = ((size_t)bkv * p.T_cap + t) * kHeadDim;
    const uint16_t* krow = p.K_new ? p.K_new + (size_t)bkv * kHeadDim : p.K + cache_row;
    if (p.K_new && h % G == 0 && threadIdx.x >= kHeadDim && threadIdx.x < kHeadDim + 32) {
      const int i = threadIdx.x - kHeadDim;  // 16-byte chunk i % 16 of the K (i < 16) or V row
      const uint4* src = reinterpret_cast<const uint4*>(
          (i < 16 ? p.K_new : p.V_new) + (size_t)bkv * kHeadDim);
      uint4* dst = reinterpret_cast<uint4*>(const_cast<uint16_t*>(i < 16 ? p.K : p.V) + cache_row);
      dst[i & 15] = src[i & 15];
    }
    if (threadIdx.x >= kHeadDim + 32 && threadIdx.x < kHeadDim + 48) {
      // the query row, kept for the attention phase (the selection's barriers
      // publish it); its load overlaps the label channel loads
      const int i = threadIdx.x - kHeadDim - 32;
      q_s[i] = reinterpret_cast<const uint4*>(p.Q + (size_t)bh * kHeadDim)[i];
    }
    uint16_t* lrow = p.label + ((size_t)bh * p.T_cap + t) * R;
    for (int j = threadIdx.x; j < R; j += kTopkThreads) {
      int ch = p.C[h * R + j];
      if (ch < 0 || ch >= kHeadDim) {
        flag_status(1u);
        ch &= (kHeadDim - 1);
      }
      qs[j] = bf_at(p.Q + (size_t)bh * kHeadDim + ch);
      if (p.append) {
        const uint16_t v = krow[ch];
        over16[j] = v;
        lrow[j] = v;
      }
    }
  }

  // 2. selection (its first barrier publishes qs and the new row)
  // eight label loads in flight per thread (the selection CTAs of k_topk,
  // three per SM, keep four)
  LabelSource<R, 8> src{p.Q, p.C, p.label, nullptr, p.Hq, p.T_cap};
  if (p.append) {
    src.over_t = p.T - 1;
    src.over_row = reinterpret_cast<const uint4*>(over16);
  }
  int32_t* dst_g = p.idx ? p.idx + (size_t)bh * p.k : nullptr;
  const size_t kv = (size_t)bkv * p.T_cap * kHeadDim;
  const PrefetchSureRows pf{p.prefetch ? p.K + kv : nullptr, p.V + kv};
  if (p.T <= kStepWholeT) {
    // every key into shared memory (the first barrier inside publishes qs and
    // the new row), then the exact select
    // keys and the select's scratch after q at the label channels (qs)
    uint32_t* keys = sm + TopkLayout(chunk, 1).small + 192;
    for (int i = p.T + threadIdx.x; i < kStepWholeT; i += kTopkThreads) keys[i] = 0u;
    __syncthreads();
    src.stream(bh, p.T, p.T, [](int j) { return j; },
               [&](bool v, int j, uint32_t key, float) {
                 if (v) keys[j] = key;
               },
               qs);
    __syncthreads();
    select_whole(WholeCta(), keys, keys + kStepWholeT, p.T, p.k, idx_s, dst_g);
  } else {
    topk_body(src, sm, 1, 0, bh, p.T, p.k, chunk, dst_g, idx_s, true, pf);
  }
  __syncthreads();

  // 3. attention over the kept rows (the selection's shared memory is free now)
  uint4* ring = reinterpret_cast<uint4*>(sm);
  float* red = reinterpret_cast<float*>(ring + kStepWarps * kStepStages * kAttnStageU4);
  attend_rows(p, bh, bkv, idx_s, p.k, ring, red, q_s);
}

}  // namespace ds
