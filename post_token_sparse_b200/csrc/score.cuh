// Channel-sparse approximate scores: s[b,h,t] = sum_j q[b,h,C[h,j]] * label[b,h,t,j].
//
// Double Sparsity, Method details: Key design -- tokens are ranked by their
// activation under the calibrated channels.  HBM-bound: every label row is read
// once with coalesced 16-byte loads (L1 bypassed); q[C] lives in shared memory
// as fp32 and is read by broadcast.  Products of two bf16 values are exact in
// fp32; they are summed in fp32 in channel order j = 0..r-1.
#pragma once

#include "common.cuh"

namespace ds {

constexpr int kScoreThreads = 256;

// 16-byte chunks of one label row, and rows per thread per pass
template <int R>
struct ScoreShape {
  static constexpr int kLanes = R / 8;                 // lanes (16-byte chunks) per row
  static constexpr int kRowsPerInstr = 32 / kLanes;    // rows per warp load
  static constexpr int kSlots = 4;                     // loads in flight per thread
  static constexpr int kTokensPerCta = (kScoreThreads / 32) * kSlots * kRowsPerInstr;
};

// fp32 q[C] for one head into shared memory (channel ids masked into range)
__device__ __forceinline__ void load_qc(const uint16_t* __restrict__ Q,
                                        const int32_t* __restrict__ C, int bh, int h, int r,
                                        float* qs) {
  for (int j = threadIdx.x; j < r; j += blockDim.x) {
    int c = C[h * r + j];
    if (c < 0 || c >= kHeadDim) {
      flag_status(1u);
      c &= (kHeadDim - 1);
    }
    qs[j] = bf_at(Q + (size_t)bh * kHeadDim + c);
  }
}

// Scores are summed in a fixed order shared by every kernel that computes
// them, so the fused score+select path and this one give identical fp32
// values: each 16-byte chunk (8 channels) is summed sequentially, then the
// r/8 chunk sums are added pairwise ((c0+c1)+(c2+c3))+... -- the order a
// butterfly of xor-shuffles produces when r/8 lanes share a row.
__device__ __forceinline__ float chunk_dot(const uint4& x, const float* q) {
  float a = bf_lo(x.x) * q[0];
  a = fmaf(bf_hi(x.x), q[1], a);
  a = fmaf(bf_lo(x.y), q[2], a);
  a = fmaf(bf_hi(x.y), q[3], a);
  a = fmaf(bf_lo(x.z), q[4], a);
  a = fmaf(bf_hi(x.z), q[5], a);
  a = fmaf(bf_lo(x.w), q[6], a);
  a = fmaf(bf_hi(x.w), q[7], a);
  return a;
}

// r/8 consecutive lanes hold the chunks of one row: butterfly sum of the chunk dots.
template <int R>
__device__ __forceinline__ float lane_group_score(const uint4& x, const float* qs, int chunk) {
  float a = chunk_dot(x, qs + 8 * chunk);
#pragma unroll
  for (int st = 1; st < R / 8; st <<= 1) a = a + __shfl_xor_sync(0xffffffffu, a, st);
  return a;
}

// grid: (ceil(T / kTokensPerCta), B*Hq).  R is a multiple of 8 (rows are whole
// uint4s).  r/8 lanes share a row, so every warp load reads 512 contiguous bytes.
template <int R>
__global__ void __launch_bounds__(kScoreThreads)
k_score_vec(const uint16_t* __restrict__ Q, const int32_t* __restrict__ C,
            const uint16_t* __restrict__ label, float* __restrict__ scores, int Hq, int T_cap,
            int T) {
  using S = ScoreShape<R>;
  __shared__ __align__(16) float qs[R];
  const int bh = blockIdx.y, h = bh % Hq;
  load_qc(Q, C, bh, h, R, qs);
  __syncthreads();

  const uint4* lab = reinterpret_cast<const uint4*>(label + (size_t)bh * T_cap * R);
  float* out = scores + (size_t)bh * T;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk = lane % S::kLanes;
  // token of slot i of this lane
  auto token = [&](int i) {
    return blockIdx.x * S::kTokensPerCta + (warp * S::kSlots + i) * S::kRowsPerInstr +
           lane / S::kLanes;
  };
  uint4 v[S::kSlots];
#pragma unroll
  for (int i = 0; i < S::kSlots; ++i) {
    const int t = token(i);
    if (t < T) v[i] = ldg_stream(lab + (size_t)t * S::kLanes + chunk);
  }
#pragma unroll
  for (int i = 0; i < S::kSlots; ++i) {
    const int t = token(i);
    const float s = lane_group_score<R>(v[i], qs, chunk);  // all lanes take part
    if (t < T && chunk == 0) out[t] = s;
  }
}

// Any r (rows need not be 16-byte aligned): one token per thread, scalar loads.
__global__ void __launch_bounds__(kScoreThreads)
k_score_any(const uint16_t* __restrict__ Q, const int32_t* __restrict__ C,
            const uint16_t* __restrict__ label, float* __restrict__ scores, int Hq, int T_cap,
            int T, int r) {
  __shared__ float qs[kHeadDim];
  const int bh = blockIdx.y, h = bh % Hq;
  load_qc(Q, C, bh, h, r, qs);
  __syncthreads();
  const int t = blockIdx.x * kScoreThreads + threadIdx.x;
  if (t >= T) return;
  const uint16_t* row = label + ((size_t)bh * T_cap + t) * r;
  float a = 0.f;
  for (int j = 0; j < r; ++j) a = fmaf(bf_at(row + j), qs[j], a);
  scores[(size_t)bh * T + t] = a;
}

}  // namespace ds

namespace ds {

// Group scores for grouped KV heads: sg[b,g,t] = sum over the G query heads
// h = g*G .. g*G+G-1 of s[b,h,t], each s computed exactly as k_score_vec
// computes it and the sum taken in head order in fp32 (group-shared
// selection: one top-k per KV group, so that each selected K/V row is read
// once for all of the group's query heads).
// With Kc (the K cache, [B, Hkv, T_cap, d]) the newest token's label rows are
// appended first, as ds_label_append(.., T-1, 1) writes them: the CTA whose
// tile holds token T-1 gathers them from K into shared memory and the label
// cache, and scores that token from shared memory.
// grid: (ceil(T / kTokensPerCta), B*Hkv); dynamic shared memory G*R floats,
// then (with Kc) G*R bf16.
template <int R>
__global__ void __launch_bounds__(kScoreThreads)
k_group_score(const uint16_t* __restrict__ Q, const int32_t* __restrict__ C, uint16_t* label,
              float* __restrict__ sg, int Hq, int Hkv, int T_cap, int T,
              const uint16_t* __restrict__ Kc) {
  using S = ScoreShape<R>;
  extern __shared__ __align__(16) float qg[];  // [G][R]
  const int G = Hq / Hkv;
  uint16_t* newrow = reinterpret_cast<uint16_t*>(qg + G * R);  // [G][R] with Kc
  const int bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv;
  const int t_new = T - 1;
  const bool app = Kc != nullptr && t_new / S::kTokensPerCta == (int)blockIdx.x;
  for (int i = threadIdx.x; i < G * R; i += blockDim.x) {
    const int hh = i / R, j = i % R;
    const int h = g * G + hh;
    int c = C[h * R + j];
    if (c < 0 || c >= kHeadDim) {
      flag_status(1u);
      c &= (kHeadDim - 1);
    }
    qg[i] = bf_at(Q + (size_t)(b * Hq + h) * kHeadDim + c);
    if (app) {
      const uint16_t v = Kc[((size_t)bg * T_cap + t_new) * kHeadDim + c];
      newrow[i] = v;
      label[((size_t)(b * Hq + h) * T_cap + t_new) * R + j] = v;
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk = lane % S::kLanes;
  auto token = [&](int i) {
    return blockIdx.x * S::kTokensPerCta + (warp * S::kSlots + i) * S::kRowsPerInstr +
           lane / S::kLanes;
  };
  float acc[S::kSlots];
  // two heads' rows loaded before either is used (twice the loads in flight)
  for (int hh = 0; hh < G; hh += 2) {
    const bool two = hh + 1 < G;
    const uint4* lab0 =
        reinterpret_cast<const uint4*>(label + (size_t)(b * Hq + g * G + hh) * T_cap * R);
    const uint4* lab1 = lab0 + (size_t)T_cap * S::kLanes;
    uint4 v0[S::kSlots], v1[S::kSlots];
#pragma unroll
    for (int i = 0; i < S::kSlots; ++i) {
      const int t = token(i);
      v0[i] = t < T ? ldg_stream(lab0 + (size_t)t * S::kLanes + chunk) : make_uint4(0, 0, 0, 0);
      v1[i] = two && t < T ? ldg_stream(lab1 + (size_t)t * S::kLanes + chunk)
                           : make_uint4(0, 0, 0, 0);
      if (app && t == t_new) {  // the row just appended, from shared memory
        const uint4* nr = reinterpret_cast<const uint4*>(newrow);
        v0[i] = nr[(hh * R) / 8 + chunk];
        if (two) v1[i] = nr[((hh + 1) * R) / 8 + chunk];
      }
    }
#pragma unroll
    for (int i = 0; i < S::kSlots; ++i) {
      // head order: acc + s(hh), then + s(hh+1); all lanes take part
      const float s0 = lane_group_score<R>(v0[i], qg + hh * R, chunk);
      acc[i] = hh == 0 ? s0 : acc[i] + s0;
      if (two) {
        const float s1 = lane_group_score<R>(v1[i], qg + (hh + 1) * R, chunk);
        acc[i] = acc[i] + s1;
      }
    }
  }
  float* out = sg + (size_t)bg * T;
#pragma unroll
  for (int i = 0; i < S::kSlots; ++i) {
    const int t = token(i);
    if (t < T && chunk == 0) out[t] = acc[i];
  }
}

}  // namespace ds

namespace ds {

// Block informativeness for block-granular selection (page "Jenga: Enhancing
// LLM Long-Context Fine-tuning with Contextual Token Sparsity", Core method 1:
// a token's informativeness counts positive scores only; a block's is the
// largest of its tokens').  sb[bh, j] = max over t in block j (bs tokens,
// clipped to T) of max(s[bh, t], 0), s computed exactly as k_score_vec does.
// grid: (ceil(T / kTokensPerCta), BH); bs a power of two <= 64 (it divides the
// tile); scores staged in shared memory, then one warp reduces 32 tokens (or
// one 64-token block) per pass.
template <int R>
__global__ void __launch_bounds__(kScoreThreads)
k_block_score(const uint16_t* __restrict__ Q, const int32_t* __restrict__ C,
              const uint16_t* __restrict__ label, float* __restrict__ sb, int Hq, int T_cap, int T,
              int bs) {
  using S = ScoreShape<R>;
  __shared__ __align__(16) float qs[R];
  __shared__ float sc[S::kTokensPerCta];
  const int bh = blockIdx.y, h = bh % Hq;
  load_qc(Q, C, bh, h, R, qs);
  __syncthreads();
  const uint4* lab = reinterpret_cast<const uint4*>(label + (size_t)bh * T_cap * R);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk = lane % S::kLanes;
  const int t0 = blockIdx.x * S::kTokensPerCta;
  auto row = [&](int i) { return (warp * S::kSlots + i) * S::kRowsPerInstr + lane / S::kLanes; };
  uint4 v[S::kSlots];
#pragma unroll
  for (int i = 0; i < S::kSlots; ++i) {
    const int t = t0 + row(i);
    v[i] = t < T ? ldg_stream(lab + (size_t)t * S::kLanes + chunk) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < S::kSlots; ++i) {
    const float s = lane_group_score<R>(v[i], qs, chunk);  // all lanes take part
    if (chunk == 0) sc[row(i)] = t0 + row(i) < T ? fmaxf(s, 0.f) : 0.f;
  }
  __syncthreads();
  const int nblk = (T + bs - 1) / bs;
  float* out = sb + (size_t)bh * nblk;
  const int step = bs > 32 ? bs : 32;  // tokens per warp pass
  for (int base = warp * step; base < S::kTokensPerCta; base += kScoreThreads / 32 * step) {
    float x = sc[base + lane];
    if (bs > 32) x = fmaxf(x, sc[base + 32 + lane]);
    const int seg = bs > 32 ? 32 : bs;  // lanes reduced together
    for (int o = 1; o < seg; o <<= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    const int j = (t0 + base + lane) / bs;
    if ((lane & (seg - 1)) == 0 && (bs > 32 ? lane == 0 : true) && j < nblk) out[j] = x;
  }
}

}  // namespace ds
