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

// One thread, whole row in registers (the same tree as the lane butterfly).
template <int R>
__device__ __forceinline__ float row_score(const uint4 (&v)[R / 8], const float* qs) {
  float part[R / 8];
#pragma unroll
  for (int c = 0; c < R / 8; ++c) part[c] = chunk_dot(v[c], qs + 8 * c);
#pragma unroll
  for (int st = 1; st < R / 8; st <<= 1)
#pragma unroll
    for (int c = 0; c < R / 8; c += 2 * st) part[c] = part[c] + part[c + st];
  return part[0];
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
