// Decode attention for grouped KV heads: the G (2..8) query heads of one KV
// head attend over the same K/V rows (all T tokens, or the group's shared
// token set), so each row is read from HBM once and applied to all G heads.
//
// Grouped-query attention shares one KV head among G query heads (the
// Llama-2-70B shapes of Double Sparsity, Evaluation highlights); with a
// group-shared selection (Double Sparsity, Method details: GQA) the G heads
// also share the selected rows.  Per row the work is G dot products and G
// weighted sums of 128 dims: at HBM rate for G = 8 that is more fp32 FMAs
// than the CUDA cores issue comfortably, so both products run on the tensor
// cores as small matrix products (mma.sync m16n8k16, bf16 in, fp32
// accumulate; G <= 8 is below the smallest tcgen05 tile, and the kernel is
// bound by HBM, not by the tensor pipe):
//   S^T[16 rows x 8 heads]  = K[16 rows x 128] . Q^T[128 x 8 heads]
//   O^T[128 x 8 heads]     += V^T[128 x 16 rows] . P^T[16 rows x 8 heads]
// Q^T lives in registers for the whole group; K and V tiles come from shared
// memory by ldmatrix (V transposed on the way); P^T goes from the S^T
// accumulator layout to the B-operand layout with movmatrix.  P is split into
// a bf16 high part and a bf16 remainder, two products, so the weights keep
// fp32 accuracy (2^-16 relative) although the tensor core takes bf16.
//
// Work split as in k_attend: the rows of all groups form one sequence and
// warp u takes the range [u*per, (u+1)*per), one CTA of kGrpWarps warps per
// SM.  Steps of 16 rows never cross a group.  A group covered by one warp is
// written directly; otherwise each warp leaves its partial (per head: max m,
// sum l, unnormalised o) in shared memory (the partial of its range's first
// group in a slot of its own, that of its last group in its ring, which is
// idle by then), the CTA's last warp on the group (a shared-memory arrival
// counter) merges the CTA's partials, and when the group spans CTAs the CTA
// partials (global slot CTA + group) are merged by the last CTA to arrive (a
// per-group arrival counter).
//
// Shared memory: per warp a ring of kGrpStages steps, each 16 K rows then 16
// V rows of 256 bytes; the 16-byte chunk c of row r sits at chunk c ^ (r & 7)
// so that the 8 rows an ldmatrix reads fall in 8 different bank groups.
#pragma once

#include "attend.cuh"

namespace ds {

constexpr int kGrpWarps = 8;
constexpr int kGrpThreads = kGrpWarps * 32;
constexpr int kGrpStages = 3;
constexpr int kGrpRows = 16;                 // rows per step: one k16 of the P.V product
constexpr int kGrpStageU4 = kGrpRows * 32;   // 16 K rows + 16 V rows = 8 KB
constexpr int kGrpMaxG = 8;                  // query heads per group (the mma's N)
constexpr int kGrpMaxUnits = kAttnCtas * kGrpWarps;
constexpr int kGrpPartStride = kGrpMaxG * kPartialStride;  // floats per partial slot
constexpr int kGrpLocal = 16;  // groups one CTA's range can touch (<= kGrpWarps + 1)
static_assert(kGrpLocal >= kGrpWarps + 1, "a CTA's range of < W*rows rows spans <= W+1 groups");
constexpr size_t kGrpRingBytes = (size_t)kGrpWarps * kGrpStages * kGrpStageU4 * 16;
constexpr size_t kGrpPartBytes = (size_t)kGrpWarps * kGrpPartStride * 4;  // first-group partials
constexpr size_t kGrpSmemBytes = kGrpRingBytes + kGrpPartBytes + kGrpLocal * 4;
static_assert(kGrpSmemBytes <= 227 * 1024, "one CTA per SM");
static_assert(kGrpPartStride * 4 <= kGrpStages * kGrpStageU4 * 16, "a partial fits a ring");

// Row ranges of the warps over `groups` groups of `rows` rows (AttnPlan's
// rule with 16-row steps): per, a multiple of 16 unless it is a whole number
// of groups; slots = 0 when no group is shared by two warps.
__host__ __device__ inline AttnPlan grp_plan(int groups, int rows) {
  const long long R = (long long)groups * rows;
  long long per = (R + kGrpMaxUnits - 1) / kGrpMaxUnits;
  if (per < kGrpRows) per = kGrpRows;
  per = (per + kGrpRows - 1) / kGrpRows * kGrpRows;
  AttnPlan pl;
  if (per >= rows) {
    const long long gpw = per / rows;
    pl.per = (int)(gpw * rows);
    pl.units = (int)((groups + gpw - 1) / gpw);
    pl.slots = 0;
  } else {
    pl.per = (int)per;
    pl.units = (int)((R + per - 1) / per);
    // CTA slots: slot of CTA c and group h is c + h
    pl.slots = (pl.units + kGrpWarps - 1) / kGrpWarps + groups;
  }
  return pl;
}

__host__ __device__ inline size_t grp_workspace_bytes(const AttnPlan& pl) {
  if (pl.slots == 0) return 0;
  const size_t b = kCounterBytes + (size_t)pl.slots * kGrpPartStride * sizeof(float);
  return (b + 255) & ~size_t(255);
}

// Weighted sum of n partials of one head by one lane: addr(i) is partial i
// (m, l, pad, pad, o[128]), in shared memory or (kGlobal) in global memory
// written by other CTAs; the lane takes dims d0..d0+31.  M: common max, L:
// merged sum, acc: merged o.
template <bool kGlobal, class Addr>
__device__ __forceinline__ void grp_merge(Addr addr, int n, int d0, float& M, float& L,
                                          float4 (&acc)[8]) {
  auto ld = [](const float* q) { return kGlobal ? __ldcg(q) : *q; };
  M = -INFINITY;
#pragma unroll 4
  for (int i = 0; i < n; ++i) M = fmaxf(M, ld(addr(i)));
  L = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
  for (int i = 0; i < n; ++i) {
    const float* sp = addr(i);
    const float w = rescale(ld(sp), M);
    L = fmaf(ld(sp + 1), w, L);
    const float4* o4 = reinterpret_cast<const float4*>(sp + 4 + d0);
    float4 v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = kGlobal ? __ldcg(o4 + e) : o4[e];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      acc[e].x = fmaf(v[e].x, w, acc[e].x);
      acc[e].y = fmaf(v[e].y, w, acc[e].y);
      acc[e].z = fmaf(v[e].z, w, acc[e].z);
      acc[e].w = fmaf(v[e].w, w, acc[e].w);
    }
  }
}

struct GrpParams {
  const uint16_t* Q;   // [B, Hq, 128]
  const uint16_t* K;   // [B, Hkv, T_cap, 128]
  const uint16_t* V;
  const int32_t* idx;  // [groups, rows] shared token ids (sparse), null (dense)
  float* O;            // [B, Hq, 128]
  float* lse;          // [B, Hq] or null
  uint32_t* arrivals;  // [groups] (zero between calls) when slots > 0
  float* partial;      // [slots, kGrpPartStride] when slots > 0
  int groups;          // B * Hkv
  int G, Hq, Hkv, T_cap, T;
  int rows;            // per group: k (sparse) or T (dense)
  int per, units;
  float scale_log2;
};

// Position of a warp in its range, in steps of 16 rows that never cross a
// group (RowCursor's walk with a longer step).
struct GrpCursor {
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
    r += kGrpRows;
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
  __device__ __forceinline__ bool last() const { return r + kGrpRows >= end; }
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// d += a . b for one m16n8k16 tile, bf16 operands, fp32 accumulators
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// 8x8 bf16 matrix held one row pair per lane, transposed across the warp
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// {lo, hi} -> bf16x2 (lo in the low half), round to nearest even
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
// 16-byte copy that writes zeros (reads nothing) when !v
__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, bool v) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const uint32_t n = v ? 16u : 0u;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(n)
               : "memory");
}

// grid: ceil(units / kGrpWarps) CTAs of kGrpThreads, kGrpSmemBytes dynamic
// shared memory.
template <bool kSparse>
__global__ void __launch_bounds__(kGrpThreads, 1)
k_attend_group(const GrpParams p) {
  extern __shared__ __align__(128) uint4 smem_grp[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * kGrpWarps + warp;
  float* part0 = reinterpret_cast<float*>(reinterpret_cast<char*>(smem_grp) + kGrpRingBytes);
  uint32_t* lctr =
      reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(smem_grp) + kGrpRingBytes + kGrpPartBytes);
  if (threadIdx.x < kGrpLocal) lctr[threadIdx.x] = 0u;
  __syncthreads();  // the only block barrier: idle warps may leave after it
  if (u >= p.units) return;
  uint4* ring = smem_grp + warp * kGrpStages * kGrpStageU4;
  const uint32_t ring_s = static_cast<uint32_t>(__cvta_generic_to_shared(ring));
  const int gq = lane >> 2, tq = lane & 3;  // mma fragment coordinates
  const int G = p.G;

  const long long R = (long long)p.groups * p.rows;
  const long long a = (long long)u * p.per;
  const long long b = a + p.per < R ? a + p.per : R;

  // copy layout: in copy i (0..7) lane copies chunk (lane & 15) of row
  // 2i + (lane >> 4), of K and of V: two whole rows per instruction
  const int crow = lane >> 4, cch = lane & 15;

  GrpCursor ic, cc, dc;  // issue, consume and id cursors (dc one step ahead of ic)
  ic.begin(a, b, p.rows);
  cc = ic;
  dc = ic;

  // token ids (sparse): lane l holds the id of row (l & 15) of a step
  auto load_ids = [&](const GrpCursor& d) -> int {
    int t = 0;
    if constexpr (kSparse) {
      if (d.valid() && d.r + (lane & 15) < d.end)
        t = __ldg(p.idx + (size_t)d.h * p.rows + d.r + (lane & 15));
    }
    return t;
  };
  // Q^T fragments of group h: lane (gq, tq) holds Q[head gq][16kk + 2tq ..] and
  // [16kk + 8 + 2tq ..] for kk = 0..7 (zero for gq >= G)
  auto load_q = [&](int h, uint32_t (&q)[16]) {
    const int bb = h / p.Hkv, kv = h - bb * p.Hkv;
    const bool v = gq < G;
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(
        p.Q + ((size_t)bb * p.Hq + (size_t)kv * G + (v ? gq : 0)) * kHeadDim);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      q[2 * kk] = v ? __ldg(q32 + kk * 8 + tq) : 0u;
      q[2 * kk + 1] = v ? __ldg(q32 + kk * 8 + 4 + tq) : 0u;
    }
  };

  uint32_t qnext[16];
  int qn_h = -1;  // group whose Q fragments qnext holds (-1: none pending)
  // ids of the next two steps to issue, loaded two steps ahead
  int ids_a = load_ids(dc);
  if (dc.valid()) dc.next(b, p.rows);
  int ids_b = load_ids(dc);
  if (dc.valid()) dc.next(b, p.rows);

  auto issue = [&](int s) {
    const int ids = ids_a;
    ids_a = ids_b;
    ids_b = load_ids(dc);
    if (dc.valid()) dc.next(b, p.rows);
    if (!ic.valid()) return;
    if (ic.first && qn_h < 0) {
      load_q(ic.h, qnext);
      qn_h = ic.h;
    }
    const int bb = ic.h / p.Hkv, kv = ic.h - bb * p.Hkv;
    const size_t base = ((size_t)bb * p.Hkv + kv) * p.T_cap;
    uint4* st = ring + (s % kGrpStages) * kGrpStageU4;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int row = 2 * i + crow;
      const bool v = ic.r + row < ic.end;
      int t = ic.r + row;
      if constexpr (kSparse) {
        t = __shfl_sync(0xffffffffu, ids, row);
        if (v && (t < 0 || t >= p.T)) {
          flag_status(2u);
          t = min(max(t, 0), p.T - 1);
        }
      }
      const size_t src = v ? (base + (size_t)t) * (kHeadDim / 8) + cch : 0;
      const int dst = row * 16 + (cch ^ (row & 7));
      cp_async16_zfill(st + dst, reinterpret_cast<const uint4*>(p.K) + src, v);
      cp_async16_zfill(st + 256 + dst, reinterpret_cast<const uint4*>(p.V) + src, v);
    }
    ic.next(b, p.rows);
  };

#pragma unroll
  for (int s = 0; s < kGrpStages - 1; ++s) {
    issue(s);
    cp_async_commit();
  }

  // ldmatrix row addresses (bytes from the stage start, before the chunk):
  // K: matrices (rows 0-7 | 8-15) x (chunk 2kk | 2kk+1) in the order of the
  // A fragment a0..a3; V (transposed): (chunk 2mt | 2mt+1) x (rows 0-7 | 8-15)
  const int krow = (lane & 7) + ((lane >> 3) & 1) * 8, kch = lane >> 4;
  const int vrow = (lane & 7) + (lane >> 4) * 8, vch = (lane >> 3) & 1;

  uint32_t q[16];
  float o[8][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads 2tq, 2tq+1
  for (int n = 0; cc.valid(); ++n) {
    if (cc.first) {
      if (qn_h == cc.h) {
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = qnext[i];
        qn_h = -1;
      } else {
        load_q(cc.h, q);
      }
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
    }
    // every lane's reads of the slot about to be refilled are done
    __syncwarp();
    issue(n + kGrpStages - 1);
    cp_async_commit();
    cp_async_wait<kGrpStages - 1>();
    __syncwarp();

    const uint32_t st = ring_s + (uint32_t)((n % kGrpStages) * kGrpStageU4 * 16);
    // S^T = K . Q^T
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t af[4];
      ldsm_x4(st + krow * 256 + (((2 * kk + kch) ^ (krow & 7)) << 4), af);
      mma_bf16(s4, af, q[2 * kk], q[2 * kk + 1]);
    }
    // logits in the log2 domain; rows past the step's end are masked
    const int nv = cc.end - cc.r;
    const float x0 = gq < nv ? s4[0] * p.scale_log2 : -INFINITY;      // row gq, head 2tq
    const float x1 = gq < nv ? s4[1] * p.scale_log2 : -INFINITY;      // row gq, head 2tq+1
    const float x2 = gq + 8 < nv ? s4[2] * p.scale_log2 : -INFINITY;  // row gq+8, head 2tq
    const float x3 = gq + 8 < nv ? s4[3] * p.scale_log2 : -INFINITY;
    float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
    for (int off = 4; off <= 16; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const bool g0 = mx0 > m0, g1 = mx1 > m1;
    if (__any_sync(0xffffffffu, g0 || g1)) {
      const float a0 = g0 ? exp2f(m0 - mx0) : 1.f;  // 0 while m is -inf
      const float a1 = g1 ? exp2f(m1 - mx1) : 1.f;
      if (g0) {
        l0 *= a0;
        m0 = mx0;
      }
      if (g1) {
        l1 *= a1;
        m1 = mx1;
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        o[mt][0] *= a0;
        o[mt][1] *= a1;
        o[mt][2] *= a0;
        o[mt][3] *= a1;
      }
    }
    const float p0 = exp2f(x0 - m0), p1 = exp2f(x1 - m1);
    const float p2 = exp2f(x2 - m0), p3 = exp2f(x3 - m1);
    l0 += p0 + p2;
    l1 += p1 + p3;
    // P^T (rows x heads) as the B operand: high bf16 parts and remainders
    const uint32_t h01 = pack_bf16(p0, p1), h23 = pack_bf16(p2, p3);
    const uint32_t r01 = pack_bf16(p0 - bf_lo(h01), p1 - bf_hi(h01));
    const uint32_t r23 = pack_bf16(p2 - bf_lo(h23), p3 - bf_hi(h23));
    const uint32_t bh0 = movm_t(h01), bh1 = movm_t(h23);
    const uint32_t br0 = movm_t(r01), br1 = movm_t(r23);
    // O^T += V^T . P^T
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t af[4];
      ldsm_x4_t(st + 4096 + vrow * 256 + (((2 * mt + vch) ^ (vrow & 7)) << 4), af);
      mma_bf16(o[mt], af, bh0, bh1);
      mma_bf16(o[mt], af, br0, br1);
    }

    if (cc.last()) {
      // the warp's rows of group h are done: sums over the 8 lanes of a head
      const int h = cc.h;
      float L0 = l0, L1 = l1;
#pragma unroll
      for (int off = 4; off <= 16; off <<= 1) {
        L0 += __shfl_xor_sync(0xffffffffu, L0, off);
        L1 += __shfl_xor_sync(0xffffffffu, L1, off);
      }
      const int bb = h / p.Hkv, kv = h - bb * p.Hkv;
      const size_t head0 = (size_t)bb * p.Hq + (size_t)kv * G;  // the group's first query head
      const int f = (int)((long long)h * p.rows / p.per);
      const int lw = (int)(((long long)(h + 1) * p.rows - 1) / p.per);
      const int ha = 2 * tq, hb = 2 * tq + 1;
      if (f == lw) {
        const float i0 = 1.f / L0, i1 = 1.f / L1;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int d0 = mt * 16 + gq;
          if (ha < G) {
            float* oa = p.O + (head0 + ha) * kHeadDim;
            oa[d0] = o[mt][0] * i0;
            oa[d0 + 8] = o[mt][2] * i0;
          }
          if (hb < G) {
            float* ob = p.O + (head0 + hb) * kHeadDim;
            ob[d0] = o[mt][1] * i1;
            ob[d0 + 8] = o[mt][3] * i1;
          }
        }
        if (p.lse && gq == 0) {
          if (ha < G) p.lse[head0 + ha] = (m0 + log2f(L0)) * 0.69314718055994530942f;
          if (hb < G) p.lse[head0 + hb] = (m1 + log2f(L1)) * 0.69314718055994530942f;
        }
      } else {
        // this warp's partial in shared memory: the range's last group in the
        // warp's ring (no copies are pending: the range has no later step),
        // its first group in the warp's own slot; the CTA's last warp on the
        // group merges the CTA's partials
        const long long hend = (long long)(h + 1) * p.rows;
        const int cta0 = blockIdx.x * kGrpWarps;
        // warp wg (of this CTA) ends its range in group h (ring) or goes on
        // past it (own slot)
        auto part_of = [&](int wg) -> float* {
          const long long e = (long long)(wg + 1) * p.per;
          const int wl = wg - cta0;
          return (e < R ? e : R) <= hend
                     ? reinterpret_cast<float*>(smem_grp + wl * kGrpStages * kGrpStageU4)
                     : part0 + (size_t)wl * kGrpPartStride;
        };
        if (b <= hend) {
          cp_async_wait<0>();
          __syncwarp();
        }
        float* part = part_of(u);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int d0 = mt * 16 + gq;
          if (ha < G) {
            part[ha * kPartialStride + 4 + d0] = o[mt][0];
            part[ha * kPartialStride + 4 + d0 + 8] = o[mt][2];
          }
          if (hb < G) {
            part[hb * kPartialStride + 4 + d0] = o[mt][1];
            part[hb * kPartialStride + 4 + d0 + 8] = o[mt][3];
          }
        }
        if (gq == 0) {
          if (ha < G) {
            part[ha * kPartialStride] = m0;
            part[ha * kPartialStride + 1] = L0;
          }
          if (hb < G) {
            part[hb * kPartialStride] = m1;
            part[hb * kPartialStride + 1] = L1;
          }
        }
        const int lo = max(f, cta0), hi = min(lw, cta0 + kGrpWarps - 1);
        const int hbase = (int)((long long)cta0 * p.per / p.rows);
        __threadfence_block();
        __syncwarp();
        uint32_t old = 0;
        if (lane == 0) old = atomicAdd(&lctr[h - hbase], 1u);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == (uint32_t)(hi - lo)) {
          __threadfence_block();
          // lane (j, quarter): head j, dims 32*quarter .. +31
          const int j = lane >> 2, d0 = (lane & 3) * 32;
          float M, L;
          float4 acc[8];
          if (j < G)
            grp_merge<false>([&](int i) -> const float* {
                               return part_of(lo + i) + j * kPartialStride;
                             },
                             hi - lo + 1, d0, M, L, acc);
          const int cf = f / kGrpWarps, cl = lw / kGrpWarps;
          float* cpart = p.partial;
          bool final_merge = cf == cl;
          if (!final_merge) {
            // the group spans CTAs: publish the CTA's partial; the last CTA merges
            float* gp = cpart + (size_t)(blockIdx.x + h) * kGrpPartStride + j * kPartialStride;
            if (j < G) {
              float4* o4 = reinterpret_cast<float4*>(gp + 4 + d0);
#pragma unroll
              for (int e = 0; e < 8; ++e) o4[e] = acc[e];
              if ((lane & 3) == 0) {
                gp[0] = M;
                gp[1] = L;
              }
            }
            __threadfence();
            __syncwarp();
            uint32_t old2 = 0;
            if (lane == 0) old2 = atomicAdd(&p.arrivals[h], 1u);
            old2 = __shfl_sync(0xffffffffu, old2, 0);
            if (old2 == (uint32_t)(cl - cf)) {
              __threadfence();
              if (j < G)
                grp_merge<true>([&](int i) -> const float* {
                            return cpart + (size_t)(cf + i + h) * kGrpPartStride +
                                   j * kPartialStride;
                          },
                          cl - cf + 1, d0, M, L, acc);
              if (lane == 0) p.arrivals[h] = 0u;  // zero again for the next call
              final_merge = true;
            }
          }
          if (final_merge && j < G) {
            const float inv = 1.f / L;
            float4* out = reinterpret_cast<float4*>(p.O + (head0 + j) * kHeadDim + d0);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              out[e] = make_float4(acc[e].x * inv, acc[e].y * inv, acc[e].z * inv,
                                   acc[e].w * inv);
            if (p.lse && (lane & 3) == 0)
              p.lse[head0 + j] = (M + log2f(L)) * 0.69314718055994530942f;
          }
        }
      }
    }
    cc.next(b, p.rows);
  }
  cp_async_wait<0>();
}

}  // namespace ds
