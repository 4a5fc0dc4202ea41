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

namespace ds {

// KV-cache append of one decode step: K[b,g,t,:] = K_new[b,g,:] and the same
// for V.  The new rows may be read from page-locked host memory mapped into
// the device (the step's inputs arriving from the host need no copy of their
// own).  grid (B*Hkv), 32 threads: lanes 0-15 copy the K row, 16-31 the V row,
// 16 bytes each.
__global__ void __launch_bounds__(32)
k_kv_append(const uint16_t* __restrict__ K_new, const uint16_t* __restrict__ V_new,
            uint16_t* __restrict__ K, uint16_t* __restrict__ V, int T_cap, int t) {
  const int bg = blockIdx.x, lane = threadIdx.x;
  const bool isv = lane >= 16;
  const uint4* src = reinterpret_cast<const uint4*>((isv ? V_new : K_new) + (size_t)bg * kHeadDim);
  uint4* dst = reinterpret_cast<uint4*>((isv ? V : K) + ((size_t)bg * T_cap + t) * kHeadDim);
  dst[lane & 15] = src[lane & 15];
}

}  // namespace ds
