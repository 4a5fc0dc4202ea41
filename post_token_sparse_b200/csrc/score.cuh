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
  static constexpr int kChunks = R / 8;                         // uint4 per row
  static constexpr int kRowsPerThread = kChunks >= 4 ? 1 : 4 / kChunks;
  static constexpr int kTokensPerCta = kScoreThreads * kRowsPerThread;
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

// Score of one label row whose chunks are already in registers.  Summation is
// sequential over j so the result does not depend on R's blocking.
template <int R>
__device__ __forceinline__ float row_score(const uint4 (&v)[R / 8], const float* qs) {
  float a = 0.f;
#pragma unroll
  for (int c = 0; c < R / 8; ++c) {
    const uint4 x = v[c];
    const float* q = qs + 8 * c;
    a = fmaf(bf_lo(x.x), q[0], a);
    a = fmaf(bf_hi(x.x), q[1], a);
    a = fmaf(bf_lo(x.y), q[2], a);
    a = fmaf(bf_hi(x.y), q[3], a);
    a = fmaf(bf_lo(x.z), q[4], a);
    a = fmaf(bf_hi(x.z), q[5], a);
    a = fmaf(bf_lo(x.w), q[6], a);
    a = fmaf(bf_hi(x.w), q[7], a);
  }
  return a;
}

// grid: (ceil(T / kTokensPerCta), B*Hq).  R is a multiple of 8 (rows are whole uint4s).
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
  const int tbase = blockIdx.x * S::kTokensPerCta + threadIdx.x;

  uint4 v[S::kRowsPerThread][S::kChunks];
#pragma unroll
  for (int i = 0; i < S::kRowsPerThread; ++i) {
    const int t = tbase + i * kScoreThreads;
    if (t < T) {
#pragma unroll
      for (int c = 0; c < S::kChunks; ++c) v[i][c] = ldg_stream(lab + (size_t)t * S::kChunks + c);
    }
  }
#pragma unroll
  for (int i = 0; i < S::kRowsPerThread; ++i) {
    const int t = tbase + i * kScoreThreads;
    if (t < T) out[t] = row_score<R>(v[i], qs);
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
