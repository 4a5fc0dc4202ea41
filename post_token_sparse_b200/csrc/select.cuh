// Per-head top-k for heads of moderate length (4096 < T <= 32768), from the
// label cache, in one launch with a workspace.
//
// Token selection keeps the tokens with the highest approximate activation
// (Double Sparsity, Method details: Key design); contract as for k_topk: the k
// largest scores, ties to the lower token index, -0 == +0, output ascending.
//
// Grid (tiles, heads): each CTA streams one tile of kSelTile tokens of one
// head's label rows (the HBM-bound part), computes every token's fp32 score
// exactly as k_score_vec does (optionally writing it out) and stores only the
// top 16 bits of its order-preserving key in the workspace (2 bytes a token).
// The head's last tile to finish (a per-head arrival counter) then selects the
// head from those prefixes, which are still in L2, while other CTAs keep
// streaming:
//   1. a bracket [lo, hi] on the prefixes from a 2048-token subsample (ranks
//      k*m/T -/+ (5 sd + 2), as k_topk brackets its sample);
//   2. one pass over each thread's run of tokens builds two register bit
//      masks: above the bracket, and inside it (the candidates);
//   3. the candidates (token order) give the 16-bit bin B16 of the k-th key;
//   4. B16's tokens have their exact keys recomputed from their label rows and
//      a radix select over the keys' low 16 bits gives the exact threshold;
//      kept tokens of B16 are marked, ties in token order up to the rank needed;
//   5. each thread writes its kept tokens, ascending.
// The prefixes' L2 lines are then discarded (no write-back of a buffer that is
// dead).  When the bracket misses, histograms of every prefix give B16 instead; when
// B16 holds more tokens than its list, their exact keys are recomputed in
// place (both slower, both exact).
#pragma once

#include "topk.cuh"

namespace ds {

constexpr int kSelThreads = kTopkThreads;  // 8 warps: LabelSource's slicing
constexpr int kSelTile = 16384;            // tokens scored by one CTA
constexpr int kSelMaxT = 32768;            // 128 tokens per selector thread at most
constexpr int kSelMaxRun = kSelMaxT / kSelThreads;
constexpr int kSelListCap = 4096;          // candidates (and B16's tokens) held in lists
constexpr int kSelSmallBin = 64;           // B16's tokens ranked by one warp up to this
constexpr int kSelSample = 2048;           // prefixes sampled for the bracket
constexpr int kSelSlots = 8;               // label loads in flight per thread
static_assert(kSelThreads == 256, "the selector's scans and 256-bin histograms take 256 threads");

// Tokens of each selector thread: a power of two >= T/256 (at least 8: whole
// 16-byte prefix runs), so that a token's place is found by shifts.
__host__ __device__ inline int sel_per(int T) {
  int per = 8;
  while (per * kSelThreads < T) per <<= 1;
  return per;
}
__host__ __device__ inline int sel_tpad(int T) { return sel_per(T) * kSelThreads; }

// Workspace: one arrival counter per head at a fixed place (zero between
// calls), then each head's prefixes, T_pad 16-bit words.
__host__ __device__ inline size_t sel_ws_bytes(int BH, int T) {
  const size_t b = kCounterBytes + (size_t)BH * sel_tpad(T) * 2;
  return (b + 255) & ~size_t(255);
}

// Prefixes are stored transposed: selector thread ct owns tokens
// [ct*per, (ct+1)*per), and its i-th run of 8 sits in 16-byte word
// i*256 + ct, so that a warp's 16-byte loads are consecutive.  Index of token
// t's prefix, in 16-bit units.
__device__ __forceinline__ int key_slot(int t, int per) {
  const int lg = 31 - __clz(per);
  const int ct = t >> lg, j = t & (per - 1);
  return (((j >> 3) * kSelThreads + ct) << 3) + (j & 7);
}

struct SelParams {
  const uint16_t* Q;
  const int32_t* C;
  const uint16_t* label;
  float* scores;        // optional [BH, T]
  int32_t* idx;         // [BH, k]
  uint32_t* arrivals;   // [BH]
  uint16_t* prefixes;   // [BH, T_pad]
  int BH, Hq, T_cap, T, k;
};

enum { S_BIN = 0, S_ABV = 1, S_CNT = 2, S_LAST = 3 };

// The fp32 score of one label row computed by one thread in exactly the order
// of lane_group_score: 8-channel chunk sums, then pairwise as the butterfly
// adds them.
template <int R>
__device__ __forceinline__ float exact_row_score(const uint16_t* row, const float* qs) {
  constexpr int NC = R / 8;
  float a[NC];
  const uint4* r4 = reinterpret_cast<const uint4*>(row);
#pragma unroll
  for (int c = 0; c < NC; ++c) a[c] = chunk_dot(__ldg(r4 + c), qs + 8 * c);
#pragma unroll
  for (int st = 1; st < NC; st <<= 1)
#pragma unroll
    for (int i = 0; i < NC; i += 2 * st) a[i] = a[i] + a[i + st];
  return a[0];
}

// Exact keys of the n tokens tok[0..n) into key[], the CTA's threads taking
// items tid, tid+256, ...: a batch of items' label rows is loaded before any
// is used, so that their loads are in flight together.
template <int R>
__device__ __forceinline__ void exact_keys(const uint16_t* lab, const float* qs,
                                           const uint32_t* tok, uint32_t* key, int n) {
  constexpr int NC = R / 8;
  constexpr int kBatch = NC >= 8 ? 1 : 8 / NC;
  for (int i0 = threadIdx.x; i0 < n; i0 += kBatch * kSelThreads) {
    uint4 x[kBatch][NC];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int i = i0 + b * kSelThreads;
      const uint4* r4 = reinterpret_cast<const uint4*>(lab + (size_t)(i < n ? tok[i] : 0) * R);
#pragma unroll
      for (int c = 0; c < NC; ++c) x[b][c] = i < n ? __ldg(r4 + c) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int i = i0 + b * kSelThreads;
      float a[NC];
#pragma unroll
      for (int c = 0; c < NC; ++c) a[c] = chunk_dot(x[b][c], qs + 8 * c);
#pragma unroll
      for (int st = 1; st < NC; st <<= 1)
#pragma unroll
        for (int j = 0; j < NC; j += 2 * st) a[j] = a[j] + a[j + st];
      if (i < n) key[i] = order_key(a[0]);
    }
  }
}

// Exact keys of a head's tokens for the selection's boundary bin: recomputed
// from the head's label rows (LabelKeys), or read from written scores
// (StoredKeys).
template <int R>
struct LabelKeys {
  const uint16_t* lab;
  const float* qs;
  __device__ __forceinline__ uint32_t key(int t) const {
    return order_key(exact_row_score<R>(lab + (size_t)t * R, qs));
  }
  __device__ __forceinline__ void keys(const uint32_t* tok, uint32_t* key, int n) const {
    exact_keys<R>(lab, qs, tok, key, n);
  }
};
struct StoredKeys {
  const float* sc;  // the head's scores; read around L1 (another kernel may have written them)
  __device__ __forceinline__ uint32_t key(int t) const { return order_key(__ldcg(sc + t)); }
  __device__ __forceinline__ void keys(const uint32_t* tok, uint32_t* key, int n) const {
    constexpr int kB = 4;
    for (int i0 = threadIdx.x; i0 < n; i0 += kB * kSelThreads) {
      float v[kB];
#pragma unroll
      for (int j = 0; j < kB; ++j) {
        const int i = i0 + j * kSelThreads;
        v[j] = i < n ? __ldcg(sc + tok[i]) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < kB; ++j) {
        const int i = i0 + j * kSelThreads;
        if (i < n) key[i] = order_key(v[j]);
      }
    }
  }
};

// Inclusive prefix over the CTA's threads in order; *total: the sum.
// scratch: 8 words, not rewritten before the caller's next barrier.
__device__ __forceinline__ uint32_t blk_scan(uint32_t v, uint32_t* scratch, uint32_t* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) scratch[w] = incl;
  __syncthreads();
  uint32_t base = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < kSelThreads / 32; ++i) {
    const uint32_t x = scratch[i];
    if (i < w) base += x;
    tot += x;
  }
  *total = tot;
  return base + incl;
}

// In a 256-bin histogram (bins counted from the top), the bin b holding rank r
// (1 = largest): misc[S_BIN] = b, misc[S_ABV] = count above it, misc[S_CNT] =
// its count.  Ends with a barrier.
__device__ __forceinline__ void blk_find_bin(const uint32_t* hist, uint32_t r, uint32_t* scratch,
                                             uint32_t* misc) {
  const uint32_t c = hist[255 - threadIdx.x];
  uint32_t tot;
  const uint32_t incl = blk_scan(c, scratch, &tot);
  if (c > 0 && incl - c < r && r <= incl) {
    misc[S_BIN] = 255u - threadIdx.x;
    misc[S_ABV] = incl - c;
    misc[S_CNT] = c;
  }
  __syncthreads();
}

// The 16-bit key of rank r among n keys (key_of(i) & 0xffff, i < n) by two
// 8-bit histogram levels; *above / *eq: counts above and equal to it.
template <class KeyOf>
__device__ __forceinline__ uint32_t blk_select16(KeyOf key_of, int n, uint32_t r, uint32_t* hist,
                                                 uint32_t* scratch, uint32_t* misc,
                                                 uint32_t* above, uint32_t* eq) {
  hist[threadIdx.x] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += kSelThreads)
    atomicAdd(&hist[(key_of(i) >> 8) & 255u], 1u);
  __syncthreads();
  blk_find_bin(hist, r, scratch, misc);
  const uint32_t b1 = misc[S_BIN], a1 = misc[S_ABV];
  hist[threadIdx.x] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += kSelThreads) {
    const uint32_t key = key_of(i) & 0xffffu;
    if ((key >> 8) == b1) atomicAdd(&hist[key & 255u], 1u);
  }
  __syncthreads();
  blk_find_bin(hist, r - a1, scratch + 8, misc);
  *above = a1 + misc[S_ABV];
  *eq = misc[S_CNT];
  return (b1 << 8) | misc[S_BIN];
}

// Prefix words a thread loads before using any: while the SM's other CTAs
// stream, an L2 round trip takes about a microsecond, and the callers'
// shared-memory stores would otherwise keep each load behind the previous
// word's work.  Eight spill registers where the label rows are wide.
constexpr int kRunBatch = 4;

// Calls f(i, w) for each 16-byte word i = 0 .. per/8-1 of this thread's run,
// read around L1 (the prefixes were written by other CTAs): w holds the
// prefixes of tokens 8i .. 8i+7, two a word, the lower token low.
template <class F>
__device__ __forceinline__ void for_my_words(const uint16_t* pref, int per, F&& f) {
  const uint4* p4 = reinterpret_cast<const uint4*>(pref);
  const int words = per / 8;
#pragma unroll
  for (int i0 = 0; i0 < kSelMaxRun / 8; i0 += kRunBatch) {
    if (i0 < words) {
      uint4 v[kRunBatch];
#pragma unroll
      for (int b = 0; b < kRunBatch; ++b)
        v[b] = i0 + b < words ? __ldcg(p4 + (i0 + b) * kSelThreads + threadIdx.x)
                              : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int b = 0; b < kRunBatch; ++b) {
        if (i0 + b < words) {
          const uint32_t w[4] = {v[b].x, v[b].y, v[b].z, v[b].w};
          f(i0 + b, w);
        }
      }
    }
  }
}

// Calls f(j, prefix) for j = 0 .. per-1 of this thread's run (j: the token's
// offset in the run).
template <class F>
__device__ __forceinline__ void for_my_run(const uint16_t* pref, int per, F&& f) {
  for_my_words(pref, per, [&](int i, const uint32_t (&w)[4]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) f(8 * i + e, (w[e >> 1] >> (16 * (e & 1))) & 0xffffu);
  });
}

// Per-thread candidate entries kept during the mask pass: (16-bit key << 16) |
// offset in the run, entry c of thread t at word c * kSelThreads + t, in the
// candidate lists' storage (free until the boundary bin is known).
constexpr int kSelOwnCands = 2 * kSelListCap / kSelThreads;  // 32

struct SelSmem {
  float qs[128];
  uint32_t hist[256];
  uint32_t misc[8];
  uint32_t scan[16];
  uint16_t smp[kSelSample];  // the bracket's subsample of prefixes
  uint32_t ltok[kSelListCap];  // ltok and lkey adjacent: the candidate entries
  uint32_t lkey[kSelListCap];  // of the mask pass use both
  uint32_t selb[kSelMaxT / 32];  // kept tokens found through the lists
};

// The 16-bit keys of ranks ra and rb (0: not wanted, the output untouched)
// among the n keys of list[]: both from the same two 8-bit histogram passes.
__device__ __forceinline__ void blk_select16_pair(const uint16_t* list, int n, uint32_t ra,
                                                  uint32_t rb, SelSmem& s, uint32_t* out_a,
                                                  uint32_t* out_b) {
  uint32_t* h2 = s.ltok;  // [2][256]: the second level of both ranks (free here)
  s.hist[threadIdx.x] = 0u;
  h2[threadIdx.x] = 0u;
  h2[256 + threadIdx.x] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += kSelThreads) atomicAdd(&s.hist[list[i] >> 8], 1u);
  __syncthreads();
  // both ranks' bins from one scan
  const uint32_t c = s.hist[255 - threadIdx.x];
  uint32_t tot;
  const uint32_t incl = blk_scan(c, s.scan, &tot);
  if (c > 0) {
    if (ra && incl - c < ra && ra <= incl) {
      s.misc[0] = 255u - threadIdx.x;
      s.misc[1] = incl - c;
    }
    if (rb && incl - c < rb && rb <= incl) {
      s.misc[4] = 255u - threadIdx.x;
      s.misc[5] = incl - c;
    }
  }
  __syncthreads();
  const uint32_t ba = s.misc[0], aa = s.misc[1], bb = s.misc[4], ab = s.misc[5];
  for (int i = threadIdx.x; i < n; i += kSelThreads) {
    const uint32_t key = list[i];
    if (ra && (key >> 8) == ba) atomicAdd(&h2[key & 255u], 1u);
    if (rb && (key >> 8) == bb) atomicAdd(&h2[256 + (key & 255u)], 1u);
  }
  __syncthreads();
  const uint32_t ca = h2[255 - threadIdx.x], cb = h2[256 + 255 - threadIdx.x];
  const uint32_t inca = blk_scan(ca, s.scan + 8, &tot);
  __syncthreads();
  const uint32_t incb = blk_scan(cb, s.scan, &tot);
  if (ra && ca > 0 && inca - ca < ra - aa && ra - aa <= inca) *out_a = (ba << 8) | (255u - threadIdx.x);
  if (rb && cb > 0 && incb - cb < rb - ab && rb - ab <= incb) *out_b = (bb << 8) | (255u - threadIdx.x);
  // every thread takes the results from the two that found them
  if (ra && ca > 0 && inca - ca < ra - aa && ra - aa <= inca) s.misc[2] = *out_a;
  if (rb && cb > 0 && incb - cb < rb - ab && rb - ab <= incb) s.misc[6] = *out_b;
  __syncthreads();
  if (ra) *out_a = s.misc[2];
  if (rb) *out_b = s.misc[6];
  __syncthreads();
}

// Selection of head bh from its prefixes, by the whole CTA; ks gives the exact
// keys of the boundary bin's tokens.
template <class KS>
__device__ void select_head(const SelParams& p, int bh, SelSmem& s, const KS& ks) {
  const int T = p.T, per = sel_per(T), tp = per * kSelThreads;
  const int t0 = threadIdx.x * per;
  const uint16_t* pref = p.prefixes + (size_t)bh * tp;
  const uint32_t k = (uint32_t)p.k;
  auto exact_key = [&](int t) { return ks.key(t); };
  auto in_t = [&](int j) { return t0 + j < T; };

  for (int i = threadIdx.x; i < tp / 32; i += kSelThreads) s.selb[i] = 0u;

  // 1. bracket from a subsample of the prefixes
  const int stride = tp / kSelSample;
  const int mv = (T + stride - 1) / stride;  // sampled tokens below T
  const float e = (float)k * (float)mv / (float)T;
  const float sd = sqrtf(e * (1.f - (float)k / (float)T));
  const float margin = kBracketSigmas * sd + 2.f;
  const int r_hi = (int)floorf(e - margin), r_lo = (int)ceilf(e + margin);
  // the subsample in shared memory (one batch of loads)
  {
    uint16_t v[kSelSample / kSelThreads];
#pragma unroll
    for (int j = 0; j < kSelSample / kSelThreads; ++j) {
      const int i = threadIdx.x + j * kSelThreads;
      v[j] = i < mv ? __ldcg(pref + key_slot(i * stride, per)) : (uint16_t)0;
    }
#pragma unroll
    for (int j = 0; j < kSelSample / kSelThreads; ++j) s.smp[threadIdx.x + j * kSelThreads] = v[j];
  }
  __syncthreads();
  uint32_t hi = 0xffffffffu, lo = 0u;
  blk_select16_pair(s.smp, mv, r_hi >= 1 ? (uint32_t)r_hi : 0u, r_lo <= mv ? (uint32_t)r_lo : 0u,
                    s, &hi, &lo);

  // 2. register masks of this thread's run: above the bracket, inside it; the
  // candidates (inside it) also kept as entries of this thread
  uint32_t am[4] = {0u, 0u, 0u, 0u}, cm[4] = {0u, 0u, 0u, 0u};
  uint32_t* own = s.ltok;  // kSelOwnCands entries a thread (ltok, then lkey)
  uint32_t n_own = 0;
  const uint32_t span = hi - lo;  // lo <= hi: the candidates are key - lo <= span
  for_my_words(pref, per, [&](int i, const uint32_t (&w)[4]) {
    uint32_t g8 = 0u, c8 = 0u;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t key = (w[e >> 1] >> (16 * (e & 1))) & 0xffffu;
      g8 |= (uint32_t)(key > hi) << e;
      c8 |= (uint32_t)(key - lo <= span) << e;
    }
    am[i >> 2] |= g8 << (8 * (i & 3));
    cm[i >> 2] |= c8 << (8 * (i & 3));
    while (c8) {  // the word's candidates (a few percent of the tokens) as entries
      const int e = __ffs(c8) - 1;
      c8 &= c8 - 1u;
      const int q = e >> 1;
      const uint32_t ww = q == 0 ? w[0] : q == 1 ? w[1] : q == 2 ? w[2] : w[3];
      const uint32_t key = (ww >> (16 * (e & 1))) & 0xffffu;
      if (n_own < (uint32_t)kSelOwnCands)
        own[n_own * kSelThreads + threadIdx.x] = (key << 16) | (uint32_t)(8 * i + e);
      ++n_own;
    }
  });
  // tokens at or past T (stale prefix slots) leave both masks; entries made for
  // them follow the valid ones and are never read (nc counts valid ones only)
  {
    const int nv = T - t0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int nb = nv - 32 * w;
      const uint32_t vm = nb >= 32 ? 0xffffffffu : nb <= 0 ? 0u : (1u << nb) - 1u;
      am[w] &= vm;
      cm[w] &= vm;
    }
  }
  const uint32_t na = __popc(am[0]) + __popc(am[1]) + __popc(am[2]) + __popc(am[3]);
  const uint32_t nc = __popc(cm[0]) + __popc(cm[1]) + __popc(cm[2]) + __popc(cm[3]);
  uint32_t tot;
  const uint32_t incl = blk_scan(na | (nc << 16), s.scan, &tot);
  const uint32_t n_above = tot & 0xffffu, n_cand = tot >> 16;
  const bool listed = n_cand <= (uint32_t)kSelListCap && n_above < k && k <= n_above + n_cand;
  // every thread kept all its candidates as entries: the bin B16 is found from
  // them, without reading the prefixes again
  const bool owned = listed && !__syncthreads_or(nc > (uint32_t)kSelOwnCands);
  __syncthreads();

  // 3. the bin B16 of the k-th key
  uint32_t B16, ngt16, neq;
  uint32_t bm[4] = {0u, 0u, 0u, 0u};  // this thread's tokens of B16
  auto set_bit = [](uint32_t (&m)[4], int j) {
    const uint32_t b = 1u << (j & 31);
    const int w = j >> 5;
    m[0] |= w == 0 ? b : 0u;
    m[1] |= w == 1 ? b : 0u;
    m[2] |= w == 2 ? b : 0u;
    m[3] |= w == 3 ? b : 0u;
  };
  if (owned && hi - lo < 256u) {
    // the bracket spans fewer than 256 prefix values: one histogram of key - lo
    s.hist[threadIdx.x] = 0u;
    __syncthreads();
    for (uint32_t c = 0; c < nc; ++c)
      atomicAdd(&s.hist[(own[c * kSelThreads + threadIdx.x] >> 16) - lo], 1u);
    __syncthreads();
    blk_find_bin(s.hist, k - n_above, s.scan, s.misc);
    B16 = lo + s.misc[S_BIN];
    ngt16 = n_above + s.misc[S_ABV];
    neq = s.misc[S_CNT];
  } else if (owned) {
    // two 8-bit levels over the entries, each thread adding its own
    s.hist[threadIdx.x] = 0u;
    __syncthreads();
    for (uint32_t c = 0; c < nc; ++c) atomicAdd(&s.hist[own[c * kSelThreads + threadIdx.x] >> 24], 1u);
    __syncthreads();
    blk_find_bin(s.hist, k - n_above, s.scan, s.misc);
    const uint32_t b1 = s.misc[S_BIN], a1 = s.misc[S_ABV];
    s.hist[threadIdx.x] = 0u;
    __syncthreads();
    for (uint32_t c = 0; c < nc; ++c) {
      const uint32_t e = own[c * kSelThreads + threadIdx.x];
      if ((e >> 24) == b1) atomicAdd(&s.hist[(e >> 16) & 255u], 1u);
    }
    __syncthreads();
    blk_find_bin(s.hist, k - n_above - a1, s.scan + 8, s.misc);
    B16 = (b1 << 8) | s.misc[S_BIN];
    ngt16 = n_above + a1 + s.misc[S_ABV];
    neq = s.misc[S_CNT];
  }
  if (owned) {
    // this thread's candidates above B16 join its mask; those in B16 are marked
    for (uint32_t c = 0; c < nc; ++c) {
      const uint32_t e = own[c * kSelThreads + threadIdx.x];
      const uint32_t key16 = e >> 16;
      const int j = (int)(e & 0xffffu);
      if (key16 > B16) set_bit(am, j);
      if (key16 == B16) set_bit(bm, j);
    }
  } else if (listed) {
    // the candidates in token order: the 16-byte prefix words that hold any are
    // loaded again, all at once
    uint32_t pos = (incl - (na | (nc << 16))) >> 16;
    const uint4* p4 = reinterpret_cast<const uint4*>(pref);
#pragma unroll
    for (int i = 0; i < kSelMaxRun / 8; ++i) {
      const uint32_t bits8 = (cm[i >> 2] >> (8 * (i & 3))) & 255u;
      if (i < per / 8 && bits8) {
        const uint4 v = __ldcg(p4 + i * kSelThreads + threadIdx.x);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e8 = 0; e8 < 8; ++e8) {
          if ((bits8 >> e8) & 1u) {
            s.ltok[pos] = (uint32_t)(t0 + 8 * i + e8);
            s.lkey[pos] = (w[e8 >> 1] >> (16 * (e8 & 1))) & 0xffffu;
            ++pos;
          }
        }
      }
    }
    __syncthreads();
    uint32_t above_c;
    B16 = blk_select16([&](int i) { return s.lkey[i]; }, (int)n_cand, k - n_above, s.hist,
                       s.scan, s.misc, &above_c, &neq);
    ngt16 = n_above + above_c;
    // candidates above B16 join the bitmap
    for (uint32_t i = threadIdx.x; i < n_cand; i += kSelThreads) {
      const uint32_t t = s.ltok[i];
      if (s.lkey[i] > B16) atomicOr(&s.selb[t >> 5], 1u << (t & 31));
    }
  } else {
    // the bracket missed: histograms of every prefix
    s.hist[threadIdx.x] = 0u;
    __syncthreads();
    for_my_run(pref, per, [&](int j, uint32_t key) {
      if (in_t(j)) atomicAdd(&s.hist[key >> 8], 1u);
    });
    __syncthreads();
    blk_find_bin(s.hist, k, s.scan, s.misc);
    const uint32_t b1 = s.misc[S_BIN], a1 = s.misc[S_ABV];
    s.hist[threadIdx.x] = 0u;
    __syncthreads();
    for_my_run(pref, per, [&](int j, uint32_t key) {
      if (in_t(j) && (key >> 8) == b1) atomicAdd(&s.hist[key & 255u], 1u);
    });
    __syncthreads();
    blk_find_bin(s.hist, k - a1, s.scan + 8, s.misc);
    B16 = (b1 << 8) | s.misc[S_BIN];
    ngt16 = a1 + s.misc[S_ABV];
    neq = s.misc[S_CNT];
    // this thread's tokens above B16
    am[0] = am[1] = am[2] = am[3] = 0u;
    for_my_run(pref, per, [&](int j, uint32_t key) {
      am[j >> 5] |= (uint32_t)(in_t(j) && key > B16) << (j & 31);
    });
  }
  __syncthreads();

  // 4. B16's tokens: all kept, or the exact threshold among them
  const uint32_t need = k - ngt16;  // 1 <= need <= neq
  if (owned) {
    // marked above
  } else if (listed) {
    // B16 lies inside the bracket: its tokens are candidates of this thread's
    // own run, in the list slice this thread wrote
    const uint32_t pos0 = (incl - (na | (nc << 16))) >> 16;
    for (uint32_t i = pos0; i < pos0 + nc; ++i)
      if (s.lkey[i] == B16) {
        const int j = (int)s.ltok[i] - t0;
        bm[j >> 5] |= 1u << (j & 31);
      }
  } else {
    for_my_run(pref, per, [&](int j, uint32_t key) {
      bm[j >> 5] |= (uint32_t)(in_t(j) && key == B16) << (j & 31);
    });
  }
  if (need == neq) {
#pragma unroll
    for (int w = 0; w < 4; ++w) am[w] |= bm[w];
  } else if (neq <= (uint32_t)kSelListCap) {
    // B16's tokens in token order, their exact keys, the threshold over the
    // keys' low 16 bits, then the kept ones (ties in order up to the rank needed)
    const uint32_t nb = __popc(bm[0]) + __popc(bm[1]) + __popc(bm[2]) + __popc(bm[3]);
    uint32_t pos = blk_scan(nb, s.scan, &tot) - nb;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t bits = bm[w];
      while (bits) {
        s.ltok[pos++] = (uint32_t)(t0 + 32 * w + __ffs(bits) - 1);
        bits &= bits - 1u;
      }
    }
    __syncthreads();
    ks.keys(s.ltok, s.lkey, (int)neq);
    __syncthreads();
    if (neq <= (uint32_t)kSelSmallBin) {
      // few tokens: one warp ranks each by the keys above it and the equal keys
      // before it in token order, and keeps the need first
      if (threadIdx.x < 32) {
        for (uint32_t i = threadIdx.x; i < neq; i += 32) {
          const uint32_t ki = s.lkey[i];
          uint32_t rank = 0;
          for (uint32_t j = 0; j < neq; ++j) {
            const uint32_t kj = s.lkey[j];
            rank += (uint32_t)(kj > ki) | ((uint32_t)(kj == ki) & (uint32_t)(j < i));
          }
          if (rank < need) {
            const uint32_t t = s.ltok[i];
            atomicOr(&s.selb[t >> 5], 1u << (t & 31));
          }
        }
      }
    } else {
      uint32_t above_e, eq_e;
      const uint32_t thr =
          (B16 << 16) | blk_select16([&](int i) { return s.lkey[i]; }, (int)neq, need, s.hist,
                                     s.scan, s.misc, &above_e, &eq_e);
      const uint32_t need_eq = need - above_e;
      const int per_t = ((int)neq + kSelThreads - 1) / kSelThreads;
      const int s0 = min((int)threadIdx.x * per_t, (int)neq), s1 = min(s0 + per_t, (int)neq);
      uint32_t nt = 0;
      for (int i = s0; i < s1; ++i) nt += s.lkey[i] == thr;
      uint32_t rank = blk_scan(nt, s.scan, &tot) - nt;
      for (int i = s0; i < s1; ++i) {
        const uint32_t key = s.lkey[i], t = s.ltok[i];
        bool keep = key > thr;
        if (key == thr) keep = rank++ < need_eq;
        if (keep) atomicOr(&s.selb[t >> 5], 1u << (t & 31));
      }
    }
  } else {
    // more tokens in B16 than the list holds: exact keys recomputed in place
    uint32_t rank = need, pf = 0u;
    for (int d = 0; d < 2; ++d) {
      s.hist[threadIdx.x] = 0u;
      __syncthreads();
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t bits = bm[w];
        while (bits) {
          const uint32_t key = exact_key(t0 + 32 * w + __ffs(bits) - 1);
          bits &= bits - 1u;
          if (d == 0)
            atomicAdd(&s.hist[(key >> 8) & 255u], 1u);
          else if (((key >> 8) & 255u) == pf)
            atomicAdd(&s.hist[key & 255u], 1u);
        }
      }
      __syncthreads();
      blk_find_bin(s.hist, rank, s.scan + 8 * d, s.misc);
      rank -= s.misc[S_ABV];
      pf = d == 0 ? s.misc[S_BIN] : (pf << 8) | s.misc[S_BIN];
    }
    const uint32_t thr = (B16 << 16) | pf, need_eq = rank;
    // ties in token order: this thread's count first
    uint32_t nt = 0, gtw[4] = {0u, 0u, 0u, 0u}, eqw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t bits = bm[w];
      while (bits) {
        const int j = 32 * w + __ffs(bits) - 1;
        bits &= bits - 1u;
        const uint32_t key = exact_key(t0 + j);
        gtw[w] |= (uint32_t)(key > thr) << (j & 31);
        eqw[w] |= (uint32_t)(key == thr) << (j & 31);
      }
      nt += __popc(eqw[w]);
    }
    uint32_t rk = blk_scan(nt, s.scan, &tot) - nt;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      am[w] |= gtw[w];
      uint32_t bits = eqw[w];
      while (bits) {
        const int j = 32 * w + __ffs(bits) - 1;
        bits &= bits - 1u;
        if (rk++ < need_eq) am[w] |= 1u << (j & 31);
      }
    }
  }
  __syncthreads();

  // the prefixes are read for the last time: drop their L2 lines without
  // writing them back (the next call writes them again)
  {
    const char* pb = reinterpret_cast<const char*>(pref);
    if ((reinterpret_cast<uintptr_t>(pb) & 127) == 0)  // whole 128-byte lines only
      for (int i = threadIdx.x; i < tp * 2 / 128; i += kSelThreads)
        asm volatile("discard.global.L2 [%0], 128;" ::"l"(pb + (size_t)i * 128) : "memory");
  }

  // 5. write this thread's kept tokens, ascending
  uint32_t sel[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t m = 0u;
    if (per >= 32) {
      if (32 * w < per) m = s.selb[(t0 >> 5) + w];
    } else if (w == 0) {
      m = (s.selb[t0 >> 5] >> (t0 & 31)) & ((1u << per) - 1u);
    }
    sel[w] = am[w] | m;
  }
  const uint32_t cnt = __popc(sel[0]) + __popc(sel[1]) + __popc(sel[2]) + __popc(sel[3]);
  uint32_t out = blk_scan(cnt, s.scan, &tot) - cnt;
  int32_t* dst = p.idx + (size_t)bh * p.k;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t bits = sel[w];
    while (bits) {
      const int t = t0 + 32 * w + __ffs(bits) - 1;
      bits &= bits - 1u;
      if (out < k) dst[out] = t;
      ++out;
    }
  }
}

// grid (ceil(T / kSelTile), BH), kSelThreads threads.
// select_head compiled as a function of its own: with R >= 64 the streaming
// loop's label rows fill the registers, and the selection inlined beside it
// made the loop spill (R = 128: 676 bytes of spill loads against 8 apart).
template <class KS>
__device__ __noinline__ void select_head_apart(const SelParams& p, int bh, SelSmem& s,
                                               const KS& ks) {
  select_head(p, bh, s, ks);
}

template <int R>
__global__ void __launch_bounds__(kSelThreads, 3)
k_score_select(const SelParams p) {
  __shared__ SelSmem s;
  const int bh = blockIdx.y;
  const int per = sel_per(p.T);
  const int tile0 = blockIdx.x * kSelTile;
  const int n = min(kSelTile, p.T - tile0);
  uint16_t* pref = p.prefixes + (size_t)bh * per * kSelThreads;
  float* so = p.scores ? p.scores + (size_t)bh * p.T : nullptr;

  LabelSource<R, kSelSlots> src{p.Q, p.C, p.label, nullptr, p.Hq, p.T_cap};
  src.prepare(bh, s.qs);
  __syncthreads();
  src.stream(bh, p.T, n, [tile0](int j) { return tile0 + j; },
             [&](bool v, int j, uint32_t key, float sc) {
               if (v) {
                 pref[key_slot(tile0 + j, per)] = (uint16_t)(key >> 16);
                 if (so) so[tile0 + j] = sc;
               }
             },
             s.qs);
  // the head's last tile to finish selects it
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0)
    s.misc[S_LAST] = atomicAdd(&p.arrivals[bh], 1u) == gridDim.x - 1 ? 1u : 0u;
  __syncthreads();
  if (s.misc[S_LAST] == 0u) return;
  __threadfence();
  const LabelKeys<R> ks{p.label + (size_t)bh * p.T_cap * R, s.qs};
  if constexpr (R >= 64)
    select_head_apart(p, bh, s, ks);  // keeps the wide streaming loop's registers
  else
    select_head(p, bh, s, ks);
  if (threadIdx.x == 0) p.arrivals[bh] = 0u;  // zero again for the next call
}

// ---- top-k over written scores in one launch ---------------------------------
//
// The same selection over a [BH, T] score array (ds_topk's contract): grid
// (ceil(T / kScoresTile), BH); each CTA turns one tile of scores into 16-bit
// key prefixes, and the head's last tile selects, taking the boundary bin's
// exact keys from the scores.  The scores are small (4 bytes a token), so the
// tiles are short and the selections of all heads overlap.
constexpr int kScoresTile = 4096;

__global__ void __launch_bounds__(kSelThreads, 3)
k_scores_select(const SelParams p) {
  __shared__ SelSmem s;
  const int bh = blockIdx.y;
  const int T = p.T, per = sel_per(T);
  uint16_t* pref = p.prefixes + (size_t)bh * per * kSelThreads;
  const float* sc = p.scores + (size_t)bh * T;
  const int t_end = min(T, (int)(blockIdx.x + 1) * kScoresTile);
#pragma unroll 4
  for (int t = blockIdx.x * kScoresTile + threadIdx.x; t < t_end; t += kSelThreads)
    pref[key_slot(t, per)] = (uint16_t)(order_key(__ldg(sc + t)) >> 16);
  // the head's last tile to finish selects it
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0)
    s.misc[S_LAST] = atomicAdd(&p.arrivals[bh], 1u) == gridDim.x - 1 ? 1u : 0u;
  __syncthreads();
  if (s.misc[S_LAST] == 0u) return;
  __threadfence();
  select_head(p, bh, s, StoredKeys{sc});
  if (threadIdx.x == 0) p.arrivals[bh] = 0u;  // zero again for the next call
}

}  // namespace ds
