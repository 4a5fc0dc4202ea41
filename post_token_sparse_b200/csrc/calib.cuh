// Offline channel calibration: per query head, the r channels whose share
// q_c * k_c of the attention logit has the largest mean magnitude over a
// calibration set (Double Sparsity, Method details: Core idea and Technical
// framework -- the channel pattern is static, so it is fixed offline; the page
// leaves the criterion open and this is its plainest reading).
//
//   I[h,c] = 1/(B*Nq*T) * sum_b (sum_n |q[b,h,n,c]|) * (sum_t |k[b,g(h),t,c]|)
//
// (|q k| = |q| |k|, so the mean over all (query, token) pairs of a sequence is
// a product of two column sums.)  Two launches:
//   k_absum         column sums of |x| over a chunk of rows of one head, for
//                   the keys and the calibration queries in one grid:
//                   HBM-bound, every row read once with 16-byte loads; fixed
//                   summation order
//   k_calib_select  per query head: combine the chunk sums (fixed order), the
//                   importance of its 128 channels, their ranks (importance
//                   descending, channel ascending) and the r kept, ascending.
#pragma once

#include "common.cuh"

namespace ds {

constexpr int kAbsumThreads = 256;
constexpr int kAbsumRows = 512;  // rows per CTA
constexpr int kAbsumRowLanes = kHeadDim / 8;                   // 16 threads per row
constexpr int kAbsumRowsPerPass = kAbsumThreads / kAbsumRowLanes;  // 16

__device__ __forceinline__ void abs_acc8(float* a, const uint4& v) {
  a[0] += fabsf(bf_lo(v.x));
  a[1] += fabsf(bf_hi(v.x));
  a[2] += fabsf(bf_lo(v.y));
  a[3] += fabsf(bf_hi(v.y));
  a[4] += fabsf(bf_lo(v.z));
  a[5] += fabsf(bf_hi(v.z));
  a[6] += fabsf(bf_lo(v.w));
  a[7] += fabsf(bf_hi(v.w));
}

// Two row sets in one launch: heads j < nx of x (rows [0, n), head stride
// x_stride elements) and heads j < ny of y (rows [0, m), stride y_stride).
// grid (max(ceil(n/kAbsumRows), ceil(m/kAbsumRows)), nx + ny).
// outx[j][chunk][c] / outy[j][chunk][c] = sum over the chunk's rows of |.[c]|.
__global__ void __launch_bounds__(kAbsumThreads)
k_absum(const uint16_t* __restrict__ x, size_t x_stride, int n, int nx, float* __restrict__ outx,
        const uint16_t* __restrict__ y, size_t y_stride, int m, float* __restrict__ outy) {
  __shared__ float part[kAbsumRowsPerPass][kHeadDim + 4];
  const bool is_x = (int)blockIdx.y < nx;
  const int j = is_x ? blockIdx.y : blockIdx.y - nx;
  const int rows = is_x ? n : m;
  const int nchunks = (rows + kAbsumRows - 1) / kAbsumRows;
  const int chunk = blockIdx.x;
  if (chunk >= nchunks) return;  // block-uniform
  const uint16_t* src = is_x ? x + (size_t)j * x_stride : y + (size_t)j * y_stride;
  float* out = (is_x ? outx : outy) + ((size_t)j * nchunks + chunk) * kHeadDim;
  const int sub = threadIdx.x % kAbsumRowLanes;   // channels 8*sub .. 8*sub+7
  const int roff = threadIdx.x / kAbsumRowLanes;  // row offset within a pass
  const int r0 = chunk * kAbsumRows;
  const int r1 = min(r0 + kAbsumRows, rows);
  const uint4* base = reinterpret_cast<const uint4*>(src);
  float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  constexpr int kU = 4;  // loads in flight per thread
  for (int r = r0 + roff; r < r1; r += kU * kAbsumRowsPerPass) {
    uint4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int rr = r + u * kAbsumRowsPerPass;
      v[u] = rr < r1 ? ldg_stream(base + (size_t)rr * kAbsumRowLanes + sub) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) abs_acc8(a, v[u]);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[roff][8 * sub + i] = a[i];
  __syncthreads();
  if (threadIdx.x < kHeadDim) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < kAbsumRowsPerPass; ++q) s += part[q][threadIdx.x];
    out[threadIdx.x] = s;
  }
}

// Sum of n chunk partials (stride kHeadDim floats), four running sums then
// combined: a fixed order.
__device__ __forceinline__ float sum_chunks(const float* p, int n) {
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  int i = 0;
  for (; i + 4 <= n; i += 4) {
    s0 += p[(size_t)i * kHeadDim];
    s1 += p[(size_t)(i + 1) * kHeadDim];
    s2 += p[(size_t)(i + 2) * kHeadDim];
    s3 += p[(size_t)(i + 3) * kHeadDim];
  }
  for (; i < n; ++i) s0 += p[(size_t)i * kHeadDim];
  return (s0 + s1) + (s2 + s3);
}

// grid (Hq), block kHeadDim.  pk: [B*Hkv][nck][d] key sums; pq: [B*Hq][ncq][d]
// query sums.  C: [Hq, r] out; importance: [Hq, d] out (nullable).
__global__ void __launch_bounds__(kHeadDim)
k_calib_select(const float* __restrict__ pk, int nck, const float* __restrict__ pq, int ncq,
               int B, int Hq, int Hkv, int r, float inv_pairs, int32_t* __restrict__ C,
               float* __restrict__ importance) {
  __shared__ float I[kHeadDim];
  __shared__ uint32_t warp_sel[kHeadDim / 32];
  const int h = blockIdx.x, c = threadIdx.x;
  const int g = h / (Hq / Hkv);
  float acc = 0.f;
  for (int b = 0; b < B; ++b) {
    const float ks = sum_chunks(pk + (size_t)(b * Hkv + g) * nck * kHeadDim + c, nck);
    const float qs = sum_chunks(pq + (size_t)(b * Hq + h) * ncq * kHeadDim + c, ncq);
    acc = fmaf(qs, ks, acc);
  }
  const float mine = acc * inv_pairs;
  I[c] = mine;
  if (importance) importance[(size_t)h * kHeadDim + c] = mine;
  __syncthreads();
  // rank: channels with larger importance, or equal importance and a lower id
  int rank = 0;
#pragma unroll 8
  for (int o = 0; o < kHeadDim; ++o) {
    const float x = I[o];
    rank += (x > mine || (x == mine && o < c)) ? 1 : 0;
  }
  const bool keep = rank < r;
  const uint32_t bal = __ballot_sync(0xffffffffu, keep);
  const int warp = c >> 5, lane = c & 31;
  if (lane == 0) warp_sel[warp] = (uint32_t)__popc(bal);
  __syncthreads();
  if (keep) {
    int pos = __popc(bal & lanemask_lt());
    for (int w = 0; w < warp; ++w) pos += (int)warp_sel[w];
    C[(size_t)h * r + pos] = c;
  }
}

}  // namespace ds
