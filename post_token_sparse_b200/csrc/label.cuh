// Label-cache append: label[b,h,t,j] = K[b,g(h),t,C[h,j]] for t in [t0, t0+n).
//
// Channel sparsity (Double Sparsity, Method details: Core idea): each query
// head keeps a contiguous copy of its r calibrated K channels so that scoring
// streams r*2 bytes per token instead of a 256-byte K row.
//
// One CTA per (32-token tile, batch, KV head): the tile's K rows are read once
// with coalesced 16-byte loads into shared memory and every query head of the
// group gathers its channels from there.
#pragma once

#include "common.cuh"

namespace ds {

constexpr int kLabelTile = 32;
constexpr int kLabelThreads = 256;

__global__ void __launch_bounds__(kLabelThreads)
k_label_append(const uint16_t* __restrict__ K, const int32_t* __restrict__ C,
               uint16_t* __restrict__ label, int Hq, int Hkv, int T_cap, int r, int t0, int n) {
  __shared__ uint4 ks[kLabelTile * (kRowBytes / 16)];  // 8 KB
  extern __shared__ int32_t cs[];                       // [G, r] channel ids

  const int G = Hq / Hkv;
  const int bg = blockIdx.y;  // b * Hkv + g
  const int b = bg / Hkv, g = bg % Hkv;
  const int tile0 = t0 + blockIdx.x * kLabelTile;
  const int rows = min(kLabelTile, t0 + n - tile0);

  // channel ids of the group's query heads; out-of-range ids are masked and flagged
  for (int i = threadIdx.x; i < G * r; i += blockDim.x) {
    int c = C[(g * G) * r + i];
    if (c < 0 || c >= kHeadDim) {
      flag_status(1u);
      c &= (kHeadDim - 1);
    }
    cs[i] = c;
  }
  const uint4* src = reinterpret_cast<const uint4*>(K + ((size_t)bg * T_cap + tile0) * kHeadDim);
  for (int i = threadIdx.x; i < rows * (kRowBytes / 16); i += blockDim.x) ks[i] = src[i];
  __syncthreads();

  const uint16_t* kt = reinterpret_cast<const uint16_t*>(ks);
  // outputs of one query head for this tile are contiguous: rows * r elements
  for (int hh = 0; hh < G; ++hh) {
    uint16_t* dst = label + ((size_t)(b * Hq + g * G + hh) * T_cap + tile0) * r;
    const int32_t* ch = cs + hh * r;
    for (int i = threadIdx.x; i < rows * r; i += blockDim.x) {
      int t = i / r, j = i - t * r;
      dst[i] = kt[t * kHeadDim + ch[j]];
    }
  }
}

}  // namespace ds
