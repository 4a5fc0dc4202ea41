// Decode attention over a set of K/V rows: the selected tokens (sparse) or all
// T tokens (dense).
//
// Token sparsity (Double Sparsity, Abstract; Key points 2): exact softmax
// attention computed over the important tokens only.  HBM-bound: every
// selected row is 256 B of K plus 256 B of V, read once.
//
// Work split: the rows of all heads, head after head, form one sequence of
// R = heads * rows rows, and warp u of the grid takes the contiguous range
// [u*per, (u+1)*per).  The grid is one CTA of kAttnWarps warps per SM, so
// every warp has the same number of rows and the same age on its SM (the
// warp schedulers favour older CTAs: ranges handed to CTAs of different ages
// finish far apart), and a warp walks straight from the end of one head into
// the next without waiting for anyone.  A head covered by one warp is written
// directly.  Otherwise each warp's partial (running max m, sum l, unnormalised
// o) goes to shared memory, the CTA's last warp on the head (a shared-memory
// arrival counter) merges them by their log-sum-exp weights, and when the head
// spans several CTAs the CTAs' merged partials meet in global memory, where
// the last CTA to arrive (a per-head arrival counter) merges those.
//
// Inside a warp: steps of 4 rows of one head; lane (g = lane/8, c = lane%8)
// handles row g of the step and the 16-byte chunks c and c+8 of that row (dims
// 8c..8c+7 and 64+8c..64+8c+7) of both K and V.  Each lane copies exactly the
// bytes it later reads with cp.async into a per-warp ring of kAttnStages steps,
// so the pipeline needs neither block barriers nor cross-lane hand-off of row
// data.  The query row of a head and (sparse) the token ids are staged by
// cp.async into small per-warp buffers ahead of use.  Per row: 8 paired FMAs +
// 3 xor-shuffles for the logit, an online-softmax update (log2 domain; the
// accumulator is rescaled only when the warp meets a new maximum), 8 paired FMAs
// into the accumulator.
#pragma once

#include "common.cuh"

namespace ds {

constexpr int kAttnWarps = 16;  // one CTA per SM (128 registers a thread)
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kAttnStages = 4;
constexpr int kAttnStageU4 = 4 * 32;  // 4 rows x (16 uint4 of K + 16 uint4 of V) = 2 KB
constexpr int kAttnCtas = 148;        // the B200's SMs: the row ranges are planned for them
constexpr int kAttnMaxUnits = kAttnCtas * kAttnWarps;
constexpr int kAttnMinRows = 16;      // rows per warp at least
constexpr int kPartialStride = 132;   // floats per partial: m, l, pad, pad, o[128]
constexpr int kIdxChunkSteps = 8;     // token ids staged 8 steps (32 rows) at a time
constexpr int kLocalHeads = 32;       // heads one CTA's range can touch (<= kAttnWarps + 1)
static_assert(kLocalHeads >= kAttnWarps + 1, "a CTA's range of < W*rows rows spans <= W+1 heads");
// Arrival counters sit at the start of the workspace, one per head for up to
// 65536 heads, so that their place never depends on the sizes of a call.
constexpr size_t kCounterBytes = 65536 * 4;

// shared memory of one warp, in uint4: ring, query slots, token-id chunks,
// then two partials (the warp's first and last head)
constexpr int kWarpRingU4 = kAttnStages * kAttnStageU4;
constexpr int kWarpQU4 = kAttnStages * 16;
constexpr int kWarpIdxU4 = 2 * 32 / 4;
constexpr int kWarpPartU4 = 2 * kPartialStride / 4;
constexpr int kWarpU4 = kWarpRingU4 + kWarpQU4 + kWarpIdxU4 + kWarpPartU4;
constexpr size_t kAttnSmemBytes = (size_t)kAttnWarps * kWarpU4 * 16 + kLocalHeads * 4;

// Row ranges of the warps.  per: rows per warp (a multiple of 4); units: warps
// with rows; slots: partial slots the call may use (0: every head is covered by
// one warp, no workspace).  Depends only on the sizes.
struct AttnPlan {
  int per;
  int units;
  int slots;
};

__host__ __device__ inline AttnPlan attn_plan(int heads, int rows) {
  const long long R = (long long)heads * rows;
  long long per = (R + kAttnMaxUnits - 1) / kAttnMaxUnits;
  if (per < kAttnMinRows) per = kAttnMinRows;
  per = (per + 3) & ~3LL;
  AttnPlan pl;
  if (per >= rows) {
    // whole heads per warp: no head is shared, nothing to merge
    const long long hpw = per / rows;
    pl.per = (int)(hpw * rows);
    pl.units = (int)((heads + hpw - 1) / hpw);
    pl.slots = 0;
  } else {
    pl.per = (int)per;
    pl.units = (int)((R + per - 1) / per);
    // slot of (CTA c, head h) is c + h
    pl.slots = (pl.units + kAttnWarps - 1) / kAttnWarps + heads;
  }
  return pl;
}

__host__ __device__ inline size_t attn_workspace_bytes(const AttnPlan& pl) {
  if (pl.slots == 0) return 0;
  const size_t b = kCounterBytes + (size_t)pl.slots * kPartialStride * sizeof(float);
  return (b + 255) & ~size_t(255);
}

struct AttnParams {
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* idx;  // null: dense (rows 0..T-1)
  float* O;
  float* lse;          // optional
  uint32_t* arrivals;  // [heads] arrival counters (zero between calls) when slots > 0
  float* partial;      // [slots, kPartialStride] when slots > 0
  int idx_per_group;   // idx rows per KV head ([B*Hkv, rows]) instead of per query head
  int block;           // > 0: idx holds block ids ([.., rows/block]); row r is token
                       // idx[r/block]*block + r%block, rows at or past T skipped
  int heads;           // B * Hq
  int Hq, Hkv, T_cap, T;
  int rows;            // per head: k (sparse) or T (dense)
  int per;             // rows per warp (attn_plan)
  int units;
  float scale_log2;    // softmax scale * log2(e)
};

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

// Merges the four row slots of a warp (lanes with equal c): afterwards every
// lane holds the warp's m, l and its chunk's 16 accumulated dims.
__device__ __forceinline__ void merge_row_slots(float& m, float& l, float* acc) {
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
}

// Position of a warp in its row range: head h, first row r of the current
// step, end of the warp's rows in h, and whether the step is the warp's first
// in h.  Steps of 4 rows never cross a head.
struct RowCursor {
  int h, r, end;
  bool first;
  __device__ __forceinline__ void begin(long long a, long long b, int rows) {
    h = (int)(a / rows);
    r = (int)(a - (long long)h * rows);
    const long long e = b - (long long)h * rows;
    end = (int)(e < rows ? e : rows);
    first = true;
  }
  __device__ __forceinline__ void next(long long b, int rows) {
    r += 4;
    first = false;
    if (r >= end) {
      ++h;
      r = 0;
      const long long e = b - (long long)h * rows;
      end = (int)(e < rows ? (e > 0 ? e : 0) : rows);
      first = true;
    }
  }
  __device__ __forceinline__ bool valid() const { return r < end; }
  __device__ __forceinline__ bool last() const { return r + 4 >= end; }
};

// Weighted sum of n partials (m, l, o) for one head, by one warp: part(i)
// gives the address of partial i (shared memory, or global memory written by
// other CTAs, read around L1 with kGlobal).  Every lane returns the common max
// M, the merged sum L and dims 4*lane..4*lane+3 of the merged unnormalised o.
template <bool kGlobal, class Part>
__device__ __forceinline__ void merge_partials(Part part, int n, int lane, float& M, float& L,
                                               float4& og) {
  auto ld = [](const float* p) { return kGlobal ? __ldcg(p) : *p; };
  M = -INFINITY;
  for (int i = lane; i < n; i += 32) M = fmaxf(M, ld(part(i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  L = 0.f;
  og = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i0 = 0; i0 < n; i0 += 32) {
    // weights of partials i0..i0+31, one per lane
    const int i = i0 + lane;
    const float wl = i < n ? rescale(ld(part(i)), M) : 0.f;
    L = fmaf(i < n ? ld(part(i) + 1) : 0.f, wl, L);
    const int cnt = min(32, n - i0);
    constexpr int kF = 4;
    for (int e0 = 0; e0 < cnt; e0 += kF) {
      float4 v[kF];
#pragma unroll
      for (int e = 0; e < kF; ++e) {
        const float* pp = part(i0 + min(e0 + e, cnt - 1)) + 4 + 4 * lane;
        v[e] = kGlobal ? __ldcg(reinterpret_cast<const float4*>(pp))
                       : *reinterpret_cast<const float4*>(pp);
      }
#pragma unroll
      for (int e = 0; e < kF; ++e) {
        const float w = __shfl_sync(0xffffffffu, wl, (e0 + e) & 31);
        if (e0 + e < cnt) {
          og.x = fmaf(v[e].x, w, og.x);
          og.y = fmaf(v[e].y, w, og.y);
          og.z = fmaf(v[e].z, w, og.z);
          og.w = fmaf(v[e].w, w, og.w);
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
}

// O[h] and lse[h] from a merged (M, L, o): lane j writes dims 4j..4j+3.
__device__ __forceinline__ void write_head(const AttnParams& p, int h, int lane, float M, float L,
                                          const float4& og) {
  const float inv = 1.f / L;
  reinterpret_cast<float4*>(p.O + (size_t)h * kHeadDim)[lane] =
      make_float4(og.x * inv, og.y * inv, og.z * inv, og.w * inv);
  if (p.lse && lane == 0) p.lse[h] = (M + log2f(L)) * 0.69314718055994530942f;
}

template <bool kSparse>
__global__ void __launch_bounds__(kAttnThreads, 1)
k_attend(const AttnParams p) {
  extern __shared__ __align__(16) uint4 smem_u4[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * kAttnWarps + warp;
  uint4* wbase = smem_u4 + warp * kWarpU4;
  uint4* ring = wbase;
  uint4* qslot = wbase + kWarpRingU4;
  int32_t* idxr = reinterpret_cast<int32_t*>(wbase + kWarpRingU4 + kWarpQU4);
  float* wpart_all = reinterpret_cast<float*>(smem_u4 + kWarpRingU4 + kWarpQU4 + kWarpIdxU4);
  uint32_t* lctr = reinterpret_cast<uint32_t*>(smem_u4 + kAttnWarps * kWarpU4);
  // this warp's partial of head h: slot 0 if h is the first head of warp w's
  // range, else slot 1
  auto wpart = [&](int w, int slot) { return wpart_all + (size_t)w * kWarpU4 * 4 + slot * kPartialStride; };
  if (threadIdx.x < kLocalHeads) lctr[threadIdx.x] = 0u;
  __syncthreads();           // the only block barrier: idle warps may leave after it
  if (u >= p.units) return;
  const int g = lane >> 3, c = lane & 7;
  const int G = p.Hq / p.Hkv;

  const long long R = (long long)p.heads * p.rows;
  const long long a = (long long)u * p.per;
  const long long b = a + p.per < R ? a + p.per : R;
  auto kv_head = [&](int h) { return (h / p.Hq) * p.Hkv + (h % p.Hq) / G; };
  const int nb = p.block ? p.rows / p.block : 0;               // block ids per idx row
  const int nb_all = p.block ? (p.T + p.block - 1) / p.block : 0;

  // token ids of 8 steps (32 rows) into chunk buffer `buf`: lane i copies the id
  // of row (i & 3) of step (i >> 2), found by walking a copy of the cursor
  auto stage_ids = [&](RowCursor& d, int buf) {
    int eh = -1, er = 0;
#pragma unroll
    for (int j = 0; j < kIdxChunkSteps; ++j) {
      if (d.valid() && (lane >> 2) == j && d.r + (lane & 3) < d.end) {
        eh = d.h;
        er = d.r + (lane & 3);
      }
      if (d.valid()) d.next(b, p.rows);
    }
    if (eh >= 0) {
      const int row = p.idx_per_group ? kv_head(eh) : eh;
      const int32_t* src = p.block ? p.idx + (size_t)row * nb + er / p.block
                                   : p.idx + (size_t)row * p.rows + er;
      const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(idxr + buf * 32 + lane));
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s), "l"(src) : "memory");
    }
  };

  RowCursor ic, cc, dc;  // issue, consume and id-staging cursors
  ic.begin(a, b, p.rows);
  cc = ic;
  // first K/V row of the issue cursor's KV head (recomputed only when it moves
  // to another head)
  long long kvrow = (long long)kv_head(ic.h) * p.T_cap;
  uint32_t vbits = 0;  // bit j: this lane's row of step (consumed + j) is valid

  // issue the copies of step s (cursor ic); returns the lane's row validity
  auto issue = [&](int s) -> uint32_t {
    if (!ic.valid()) return 0u;
    const int row = ic.r + g;
    bool v = row < ic.end;
    int t = row;
    if constexpr (kSparse) {
      const int raw = idxr[((s >> 3) & 1) * 32 + (s & 7) * 4 + g];
      if (p.block) {
        int bl = raw;
        if (v && (bl < 0 || bl >= nb_all)) {
          flag_status(2u);
          bl = min(max(bl, 0), nb_all - 1);
        }
        t = bl * p.block + row % p.block;
        v = v && t < p.T;  // the short last block
      } else {
        t = raw;
        if (v && (t < 0 || t >= p.T)) {
          flag_status(2u);
          t = min(max(t, 0), p.T - 1);
        }
      }
    }
    const int slot = s % kAttnStages;
    if (v) {
      const size_t kv = (size_t)(kvrow + t) * kHeadDim;
      const uint4* krow = reinterpret_cast<const uint4*>(p.K + kv);
      const uint4* vrow = reinterpret_cast<const uint4*>(p.V + kv);
      uint4* st = ring + slot * kAttnStageU4 + g * 32;
      cp_async16(st + c, krow + c);
      cp_async16(st + 8 + c, krow + 8 + c);
      cp_async16(st + 16 + c, vrow + c);
      cp_async16(st + 24 + c, vrow + 8 + c);
    }
    if (ic.first && lane < 16)
      cp_async16(qslot + slot * 16 + lane,
                 reinterpret_cast<const uint4*>(p.Q + (size_t)ic.h * kHeadDim) + lane);
    ic.next(b, p.rows);
    if (ic.first && ic.valid()) kvrow = (long long)kv_head(ic.h) * p.T_cap;
    return v ? 1u : 0u;
  };

  if constexpr (kSparse) {
    dc = ic;
    stage_ids(dc, 0);
    stage_ids(dc, 1);
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
  }
#pragma unroll
  for (int s = 0; s < kAttnStages - 1; ++s) {
    vbits |= issue(s) << s;
    cp_async_commit();
  }

  float q[16];
  float m = -INFINITY, l = 0.f;
  float acc[16];
  for (int n = 0; cc.valid(); ++n) {
    const int s_in = n + kAttnStages - 1;
    // the previous step's reads of the query slots and id chunks (written by
    // other lanes) are done before this step's copies overwrite them
    __syncwarp();
    if constexpr (kSparse) {
      // ids of steps s_in+8 .. s_in+15 into the buffer the previous chunk used
      if ((s_in & 7) == 0 && s_in >= 8) stage_ids(dc, ((s_in >> 3) + 1) & 1);
    }
    vbits |= issue(s_in) << (kAttnStages - 1);
    cp_async_commit();
    cp_async_wait<kAttnStages - 1>();
    __syncwarp();

    const int slot = n % kAttnStages;
    if (cc.first) {
      const uint4 qa = qslot[slot * 16 + c], qb = qslot[slot * 16 + 8 + c];
      const uint32_t w[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        q[2 * i] = bf_lo(w[i]) * p.scale_log2;
        q[2 * i + 1] = bf_hi(w[i]) * p.scale_log2;
      }
      m = -INFINITY;
      l = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    }
    const uint4* st = ring + slot * kAttnStageU4 + g * 32;
    const uint4 klo = st[c], khi = st[8 + c];
    float x = dot8(klo, q) + dot8(khi, q + 8);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    online_row((vbits & 1u) != 0u, x, m, l, acc, st[16 + c], st[24 + c]);
    vbits >>= 1;

    if (cc.last()) {
      // the warp's rows of head cc.h are done
      const int h = cc.h;
      merge_row_slots(m, l, acc);
      const int f = (int)((long long)h * p.rows / p.per);
      const int lw = (int)(((long long)(h + 1) * p.rows - 1) / p.per);
      if (f == lw) {
        float* o = p.O + (size_t)h * kHeadDim;
        if (g == 0) {
          const float inv = 1.f / l;
          float4* o4 = reinterpret_cast<float4*>(o);
          o4[2 * c] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
          o4[2 * c + 1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
          o4[16 + 2 * c] = make_float4(acc[8] * inv, acc[9] * inv, acc[10] * inv, acc[11] * inv);
          o4[16 + 2 * c + 1] =
              make_float4(acc[12] * inv, acc[13] * inv, acc[14] * inv, acc[15] * inv);
        }
        if (p.lse && lane == 0) p.lse[h] = (m + log2f(l)) * 0.69314718055994530942f;
      } else {
        // this warp's partial into shared memory; the CTA's last warp on the
        // head merges the CTA's partials
        const long long hrow = (long long)h * p.rows;
        auto slot_of = [&](int w) { return (long long)w * p.per >= hrow ? 0 : 1; };
        float* part = wpart(warp, slot_of(u));
        if (g == 0) {
          float4* o4 = reinterpret_cast<float4*>(part + 4);
          o4[2 * c] = make_float4(acc[0], acc[1], acc[2], acc[3]);
          o4[2 * c + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
          o4[16 + 2 * c] = make_float4(acc[8], acc[9], acc[10], acc[11]);
          o4[16 + 2 * c + 1] = make_float4(acc[12], acc[13], acc[14], acc[15]);
        }
        if (lane == 0) {
          part[0] = m;
          part[1] = l;
        }
        const int cta0 = blockIdx.x * kAttnWarps;
        const int lo = max(f, cta0), hi = min(min(lw, cta0 + kAttnWarps - 1), p.units - 1);
        const int hbase = (int)((long long)cta0 * p.per / p.rows);
        __threadfence_block();
        __syncwarp();
        uint32_t old = 0;
        if (lane == 0) old = atomicAdd(&lctr[h - hbase], 1u);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == (uint32_t)(hi - lo)) {
          __threadfence_block();
          float M, L;
          float4 og;
          merge_partials<false>(
              [&](int i) -> const float* { return wpart(lo + i - cta0, slot_of(lo + i)); },
              hi - lo + 1, lane, M, L, og);
          const int cf = f / kAttnWarps, cl = lw / kAttnWarps;
          if (cf == cl) {
            write_head(p, h, lane, M, L, og);
          } else {
            // the head spans CTAs: publish the CTA's partial; the last CTA merges
            float* gp = p.partial + (size_t)(blockIdx.x + h) * kPartialStride;
            reinterpret_cast<float4*>(gp + 4)[lane] = og;
            if (lane == 0) {
              gp[0] = M;
              gp[1] = L;
            }
            __threadfence();
            __syncwarp();
            uint32_t old2 = 0;
            if (lane == 0) old2 = atomicAdd(&p.arrivals[h], 1u);
            old2 = __shfl_sync(0xffffffffu, old2, 0);
            if (old2 == (uint32_t)(cl - cf)) {
              __threadfence();
              const float* g0 = p.partial + (size_t)(cf + h) * kPartialStride;
              merge_partials<true>(
                  [&](int i) -> const float* { return g0 + (size_t)i * kPartialStride; },
                  cl - cf + 1, lane, M, L, og);
              write_head(p, h, lane, M, L, og);
              if (lane == 0) p.arrivals[h] = 0u;  // zero again for the next call
            }
          }
        }
      }
    }
    cc.next(b, p.rows);
  }
  cp_async_wait<0>();
}

}  // namespace ds
