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
//   2. select   the top-k body of topk.cuh; the k indices land in shared memory
//               (and in idx when requested)
//   3. attend   8 warps each take a contiguous run of the kept rows through a
//               per-warp cp.async ring (as k_attend does), online softmax in the
//               log2 domain, warp then CTA merge -> O and lse.
#pragma once

#include "attend.cuh"
#include "topk.cuh"

namespace ds {

constexpr int kStepWarps = kTopkThreads / 32;  // 8
static_assert(kTopkThreads >= kHeadDim + 48,
              "threads d..d+31 store the new K and V rows, d+32..d+47 load the query row");
constexpr int kStepStages = 3;
constexpr int kStepMaxK = 8192;

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
    const int sel = TopkLayout(chunk, 1).words;
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

// Attention of one query (head bh) over rows idx_s[0..n) of K and V (KV head
// bkv), by kStepWarps warps; writes O[bh] and lse[bh].
__device__ __forceinline__ void attend_rows(const StepParams& p, int bh, int bkv,
                                            const int32_t* idx_s, int n, uint4* ring,
                                            float* red, const uint4* qrow) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
  uint4* my_ring = ring + warp * kStepStages * kAttnStageU4;

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
      uint4* st = my_ring + (step % kStepStages) * kAttnStageU4 + g * 32;
      cp_async16(st + c, krow + c);
      cp_async16(st + 8 + c, krow + 8 + c);
      cp_async16(st + 16 + c, vrow + c);
      cp_async16(st + 24 + c, vrow + 8 + c);
    }
  };
#pragma unroll
  for (int s = 0; s < kStepStages - 1; ++s) {
    if (s < nsteps) issue(s);
    cp_async_commit();
  }
  float m = -INFINITY, l = 0.f;
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (int s = 0; s < nsteps; ++s) {
    if (s + kStepStages - 1 < nsteps) issue(s + kStepStages - 1);
    cp_async_commit();
    cp_async_wait<kStepStages - 1>();
    const uint4* st = my_ring + (s % kStepStages) * kAttnStageU4 + g * 32;
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
  __syncthreads();
  if (threadIdx.x < kHeadDim) {
    const int j = threadIdx.x;
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
  const size_t kv = (size_t)bkv * p.T_cap * kHeadDim;
  const PrefetchSureRows pf{p.prefetch ? p.K + kv : nullptr, p.V + kv};
  topk_body(src, sm, 1, 0, bh, p.T, p.k, chunk, p.idx ? p.idx + (size_t)bh * p.k : nullptr,
            idx_s, true, pf);
  __syncthreads();

  // 3. attention over the kept rows (the selection's shared memory is free now)
  uint4* ring = reinterpret_cast<uint4*>(sm);
  float* red = reinterpret_cast<float*>(ring + kStepWarps * kStepStages * kAttnStageU4);
  attend_rows(p, bh, bkv, idx_s, p.k, ring, red, q_s);
}

}  // namespace ds
