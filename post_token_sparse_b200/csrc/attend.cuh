// Decode attention over a set of K/V rows: the selected tokens (sparse) or all
// T tokens (dense).
//
// Token sparsity (Double Sparsity, Abstract; Key points 2): exact softmax
// attention computed over the important tokens only.  HBM-bound: every
// selected row is 256 B of K plus 256 B of V, read once.
//
// Grid (G, S, B*Hkv): the G query heads sharing one KV head are neighbours in
// launch order (their dense K/V reads meet in L2), and each head's rows are
// cut into S splits.  A CTA has kAttnWarps warps; every warp owns a
// contiguous run of its split's rows and walks it 4 rows per step.  Lane
// (g = lane/8, c = lane%8) handles row g of the step and the 16-byte chunks c
// and c+8 of that row (dims 8c..8c+7 and 64+8c..64+8c+7) of both K and V.
//
// Staging: each lane copies exactly the bytes it later reads with cp.async
// into a per-warp ring of kAttnStages steps, so the pipeline needs neither
// block barriers nor cross-lane hand-off: cp.async.wait_group is the only
// wait.  Per row: 8 paired FMAs + 3 xor-shuffles for the logit, an
// online-softmax update (running max m, sum l, log2 domain; the accumulator
// rescaled only when the warp meets a new maximum), 8 paired FMAs into the
// accumulator.
// Warps then merge through shared memory; with S > 1 each split writes
// (m, l, unnormalised o) to the workspace and the head's last split to finish
// (found by an arrival counter) combines them.
#pragma once

#include "common.cuh"

namespace ds {

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = kAttnWarps * 32;
static_assert(kAttnThreads == kHeadDim, "the merges give thread j output dim j");
constexpr int kAttnStages = 4;
constexpr int kAttnStageU4 = 4 * 32;  // 4 rows x (16 uint4 of K + 16 uint4 of V) = 2 KB
constexpr int kPartialStride = 132;   // floats per split partial: m, l, pad, pad, o[128]
constexpr int kMaxRowsPerSplitSparse = 2048;

struct AttnParams {
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* idx;  // null: dense (rows 0..T-1)
  float* O;
  float* lse;      // optional
  float* partial;      // [BH, S, kPartialStride] when S > 1
  uint32_t* arrivals;  // [BH] split-arrival counters (zero between calls) when S > 1
  int idx_per_group;   // idx rows per KV head ([B*Hkv, rows]) instead of per query head
  int block;           // > 0: idx holds block ids ([.., rows/block]); row r is token
                       // idx[r/block]*block + r%block, rows at or past T skipped
  int Hq, Hkv, T_cap, T;
  int rows;           // k (sparse) or T (dense)
  int rows_per_split; // multiple of 4
  float scale_log2;   // softmax scale * log2(e)
};

__device__ __forceinline__ int nb_total(const AttnParams& p) {
  return (p.T + p.block - 1) / p.block;
}

// d0 += a0*b0 and d1 += a1*b1, each rounded once: one paired fp32 FMA.
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " mov.b64 rd, {%0, %1};\n fma.rn.f32x2 rd, ra, rb, rd;\n mov.b64 {%0, %1}, rd;\n}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// dot product of 8 bf16 values with 8 fp32 values: even and odd elements
// accumulated side by side, then added
__device__ __forceinline__ float dot8(const uint4& v, const float* q) {
  float e = bf_lo(v.x) * q[0], o = bf_hi(v.x) * q[1];
  fma2(e, o, bf_lo(v.y), bf_hi(v.y), q[2], q[3]);
  fma2(e, o, bf_lo(v.z), bf_hi(v.z), q[4], q[5]);
  fma2(e, o, bf_lo(v.w), bf_hi(v.w), q[6], q[7]);
  return e + o;
}

// acc[0..8) += p * v (8 bf16 values)
__device__ __forceinline__ void axpy8(float* acc, float p, const uint4& v) {
  fma2(acc[0], acc[1], p, p, bf_lo(v.x), bf_hi(v.x));
  fma2(acc[2], acc[3], p, p, bf_lo(v.y), bf_hi(v.y));
  fma2(acc[4], acc[5], p, p, bf_lo(v.z), bf_hi(v.z));
  fma2(acc[6], acc[7], p, p, bf_lo(v.w), bf_hi(v.w));
}

// One row of the online softmax for one lane: running max m and sum l (log2
// domain) and the lane's 16 output dims acc, with the row's logit x and its V
// chunks.  The accumulator is rescaled only when some lane of the warp meets a
// new maximum (a warp-uniform branch, rare after the first rows).  Every lane
// of the warp calls it; valid: the lane's row exists.
__device__ __forceinline__ void online_row(bool valid, float x, float& m, float& l, float* acc,
                                           const uint4& vlo, const uint4& vhi) {
  const bool grow = valid && x > m;
  if (__any_sync(0xffffffffu, grow)) {
    const float a = grow ? exp2f(m - x) : 1.f;  // 0 when m is still -inf
    if (grow) {
      l *= a;
      m = x;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] *= a;
  }
  if (valid) {
    const float pw = exp2f(x - m);
    l += pw;
    axpy8(acc, pw, vlo);
    axpy8(acc + 8, pw, vhi);
  }
}

// weight of a partial with running max m against a common max mn (0 if empty)
__device__ __forceinline__ float rescale(float m, float mn) {
  return m == -INFINITY ? 0.f : exp2f(m - mn);
}

template <bool kSparse>
__global__ void __launch_bounds__(kAttnThreads)
k_attend(const AttnParams p) {
  extern __shared__ __align__(16) uint4 smem_u4[];
  uint4* ring = smem_u4;                                                 // [warps][stages][128]
  float* red = reinterpret_cast<float*>(ring + kAttnWarps * kAttnStages * kAttnStageU4);
  int32_t* idx_s = reinterpret_cast<int32_t*>(red + kAttnWarps * 132);   // [rows_per_split]

  const int G = p.Hq / p.Hkv;
  const int bkv = blockIdx.z;  // b * Hkv + g
  const int b = bkv / p.Hkv;
  const int h = (bkv % p.Hkv) * G + blockIdx.x;
  const int bh = b * p.Hq + h;
  // Split s of KV head bkv runs in grid slot (s - 5*bkv) mod S: CTAs resident
  // together then work on different key ranges of their heads, instead of every
  // head's same range (head strides in K and V are large powers of two).
  const int S = gridDim.y;
  const int split = (int)((blockIdx.y + 5u * (unsigned)bkv) % (unsigned)S);
  const int r0 = split * p.rows_per_split;
  const int nrows = min(p.rows_per_split, p.rows - r0);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 3, c = lane & 7;

  // this lane's query chunks, issued before the index staging so that the two
  // loads overlap
  const uint4* qrow = reinterpret_cast<const uint4*>(p.Q + (size_t)bh * kHeadDim);
  const uint4 qa = qrow[c], qb = qrow[8 + c];

  // rows of this warp: [w_begin, w_end) relative to r0
  const int rpw = ((nrows + kAttnWarps - 1) / kAttnWarps + 3) & ~3;
  const int w_begin = min(warp * rpw, nrows);
  const int w_end = min(w_begin + rpw, nrows);
  const int nsteps = (w_end - w_begin + 3) >> 2;

  if constexpr (kSparse) {
    // each warp stages the token ids of its own rows (no block barrier: a warp
    // starts its gathers as soon as its own ids are in)
    if (p.block) {
      const int nb = p.rows / p.block;
      const int32_t* src = p.idx + (size_t)bh * nb;
      for (int i = w_begin + lane; i < w_end; i += 32) {
        const int r = r0 + i;
        int b = src[r / p.block];
        if (b < 0 || b >= nb_total(p)) {
          flag_status(2u);
          b = min(max(b, 0), nb_total(p) - 1);
        }
        const int t = b * p.block + r % p.block;
        idx_s[i] = t < p.T ? t : -1;  // the short last block
      }
    } else {
      const int32_t* src = p.idx + (size_t)(p.idx_per_group ? bkv : bh) * p.rows + r0;
      for (int i = w_begin + lane; i < w_end; i += 32) {
        int t = src[i];
        if (t < 0 || t >= p.T) {
          flag_status(2u);
          t = min(max(t, 0), p.T - 1);
        }
        idx_s[i] = t;
      }
    }
    __syncwarp();
  }

  // this lane's 16 query values, pre-scaled into the log2 domain
  float q[16];
  {
    const uint32_t w[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      q[2 * i] = bf_lo(w[i]) * p.scale_log2;
      q[2 * i + 1] = bf_hi(w[i]) * p.scale_log2;
    }
  }

  const size_t kv_base = (size_t)bkv * p.T_cap * kHeadDim;
  const uint16_t* Kh = p.K + kv_base;
  const uint16_t* Vh = p.V + kv_base;
  uint4* my_ring = ring + warp * kAttnStages * kAttnStageU4;

  auto issue = [&](int step) {
    const int lr = w_begin + step * 4 + g;  // row within the split
    if (lr < w_end) {
      int t = kSparse ? idx_s[lr] : r0 + lr;
      if (kSparse && t < 0) t = 0;  // a skipped row: any valid address
      const uint4* krow = reinterpret_cast<const uint4*>(Kh + (size_t)t * kHeadDim);
      const uint4* vrow = reinterpret_cast<const uint4*>(Vh + (size_t)t * kHeadDim);
      uint4* st = my_ring + (step % kAttnStages) * kAttnStageU4 + g * 32;
      cp_async16(st + c, krow + c);
      cp_async16(st + 8 + c, krow + 8 + c);
      cp_async16(st + 16 + c, vrow + c);
      cp_async16(st + 24 + c, vrow + 8 + c);
    }
  };

#pragma unroll
  for (int s = 0; s < kAttnStages - 1; ++s) {
    if (s < nsteps) issue(s);
    cp_async_commit();
  }

  float m = -INFINITY, l = 0.f;
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;

  for (int n = 0; n < nsteps; ++n) {
    if (n + kAttnStages - 1 < nsteps) issue(n + kAttnStages - 1);
    cp_async_commit();
    cp_async_wait<kAttnStages - 1>();

    const uint4* st = my_ring + (n % kAttnStages) * kAttnStageU4 + g * 32;
    const uint4 klo = st[c], khi = st[8 + c];
    float x = dot8(klo, q) + dot8(khi, q + 8);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    const int lr = w_begin + n * 4 + g;
    const bool valid = lr < w_end && (!kSparse || idx_s[lr] >= 0);
    online_row(valid, x, m, l, acc, st[16 + c], st[24 + c]);
  }
  cp_async_wait<0>();

  // merge the four row slots of the warp (lanes with equal c)
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
  // warp partials -> shared memory: red[w*132 + {0: m, 1: l, 4..131: o}]
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

  // thread j merges dim j over the warps
  const int j = threadIdx.x;
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, red[w * 132]);
  float L = 0.f, o = 0.f;
#pragma unroll
  for (int w = 0; w < kAttnWarps; ++w) {
    const float a = rescale(red[w * 132], M);
    L = fmaf(red[w * 132 + 1], a, L);
    o = fmaf(red[w * 132 + 4 + j], a, o);
  }
  if (S == 1) {
    p.O[(size_t)bh * kHeadDim + j] = o / L;
    if (p.lse && j == 0) p.lse[bh] = (M + log2f(L)) * 0.69314718055994530942f;
  } else {
    // publish this split's partial; the last split of the head to arrive
    // merges all of them and resets the head's counter for the next call
    float* part = p.partial + ((size_t)bh * S + split) * kPartialStride;
    part[4 + j] = o;
    if (j == 0) {
      part[0] = M;
      part[1] = L;
    }
    __threadfence();
    __syncthreads();
    __shared__ uint32_t last;
    if (j == 0) last = atomicAdd(&p.arrivals[bh], 1u) == (uint32_t)(S - 1);
    __syncthreads();
    if (last) {
      __threadfence();
      const float* all = p.partial + (size_t)bh * S * kPartialStride;
      // the splits' (m, l) side by side in shared memory (the ring is free),
      // each split's weight once, then every dim's weighted sum with its
      // loads independent of one another
      float* ms = reinterpret_cast<float*>(ring);  // [S] m, then [S] weight
      float* wt = ms + S;
      for (int s = j; s < S; s += kAttnThreads) ms[s] = __ldcg(all + s * kPartialStride);
      __syncthreads();
      float Mg = -INFINITY;
      for (int s = 0; s < S; ++s) Mg = fmaxf(Mg, ms[s]);
      for (int s = j; s < S; s += kAttnThreads) wt[s] = rescale(ms[s], Mg);
      __syncthreads();
      float Lg = 0.f, og = 0.f;
#pragma unroll 8
      for (int s = 0; s < S; ++s) {
        Lg = fmaf(__ldcg(all + s * kPartialStride + 1), wt[s], Lg);
        og = fmaf(__ldcg(all + s * kPartialStride + 4 + j), wt[s], og);
      }
      p.O[(size_t)bh * kHeadDim + j] = og / Lg;
      if (p.lse && j == 0) p.lse[bh] = (Mg + log2f(Lg)) * 0.69314718055994530942f;
      if (j == 0) p.arrivals[bh] = 0u;
    }
  }
}

}  // namespace ds
