// Plain C++ oracle of Double-Sparsity-style decode attention, steps O1-O5:
// label gather, channel-sparse score, top-k, softmax attention over the kept
// rows, dense attention; plus the log-sum-exp merge of split attention, and the
// rows beside the path: offline channel calibration, group-shared selection,
// block-granular selection and the hierarchical top-k.
//
// TEST INFRASTRUCTURE ONLY: loaded by tests/ (through oracle/cxx.py) and by
// the CPU-baseline leg of bench.py, never by the library.  It shares no code
// with the CUDA path (no headers, helpers or tables): the two meet only at the
// seeded bf16 inputs drawn by dsgen.
//
// Source page: "Post-Training Sparse Attention with Double Sparsity".
//   token sparsity   self-attention over the important tokens only
//                    (Abstract; Key points 2)
//   channel sparsity a few calibrated feature channels identify those tokens
//                    (Abstract; Method details: Core idea, Technical framework)
//   token choice     keep the tokens with the higher activation under those
//                    channels (Method details: Key design)
// The page gives no formulas; the readings (shared with oracle/ds_oracle.py):
//   label   label[b,h,t,j] = K[b, h/(Hq/Hkv), t, C[h,j]]     (bf16 bits copied)
//   score   s[b,h,t] = sum_j q[b,h,C[h,j]] * label[b,h,t,j]  (unscaled; j in order)
//   top-k   the k tokens first in the order (score descending, index
//           ascending); -0 and +0 compare equal; output ascending
//   attend  l_i = scale * q . K_i; m = max l; w_i = exp(l_i - m) / sum exp(l - m);
//           o = sum_i w_i V_i; lse = m + log sum exp(l - m)
//   dense   attend with every token kept
//   merge   disjoint key chunks (o_c, lse_c) combine with weights exp(lse_c - M)
// and for the rows beside the path (readings shared with oracle/ds_oracle.py):
//   calibration  I[h,c] = mean over (calibration query n, token t < T) of the
//                same sequence of |q[b,h,n,c] * k[b,g(h),t,c]|; the r channels
//                of largest I (ties to the lower channel), ascending.  The
//                page leaves the criterion open (Method details: Key design).
//   group        sg[b,g,t] = sum of s[b,h,t] over the query heads h of KV group
//                g, in head order and in the scores' own precision; one top-k
//                per group; every head of the group attends over its set
//   block        (Jenga: Core method 1; Observation 2) per block of bs
//                consecutive tokens the largest max(s_t, 0); top-kb blocks;
//                attention over their tokens, clipped to T
//   hierarchy    (HiP: Core idea, Technical framework) k contiguous parts of
//                [0, T); while a part is longer than one token, each such part
//                splits at its middle (the first half one longer), the children
//                are ranked by the score of their first token (ties to the lower
//                start) and the first k are kept; the k starts are the result
//
// Every value is decoded exactly from its bf16 bits and every step runs in
// double precision (std::exp, std::log); the order of the top-k is decided by
// std::sort on the stated total order.  Plain loops, no blocking or fusion.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <thread>
#include <vector>

namespace {

// A bf16 value is the top half of a float32.
double bf16_value(uint16_t bits) {
  const uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

// Indices of the k entries of s[0..T) first in (s descending, index
// ascending), returned in ascending index order.
template <class S>
void topk_row(const S* s, int T, int k, int32_t* out) {
  std::vector<int32_t> order(T);
  std::iota(order.begin(), order.end(), 0);
  std::sort(order.begin(), order.end(), [s](int32_t a, int32_t b) {
    if (s[a] != s[b]) return s[a] > s[b];  // -0 == +0: equal, falls to the index
    return a < b;
  });
  std::sort(order.begin(), order.begin() + k);
  std::copy(order.begin(), order.begin() + k, out);
}

// Softmax attention of one query over rows idx[0..n) of one KV head.
// q: [d] bits; K, V: [T, d] bits.  o: [d]; w: [n] (may be null).
void attend_row(const uint16_t* q, const uint16_t* K, const uint16_t* V, const int32_t* idx,
                int n, int d, double scale, double* o, double* lse, double* w) {
  std::vector<double> l(n);
  for (int i = 0; i < n; ++i) {
    const uint16_t* krow = K + static_cast<int64_t>(idx[i]) * d;
    double dot = 0.0;
    for (int c = 0; c < d; ++c) dot += bf16_value(q[c]) * bf16_value(krow[c]);
    l[i] = scale * dot;
  }
  double m = -INFINITY;
  for (int i = 0; i < n; ++i) m = std::max(m, l[i]);
  double z = 0.0;
  for (int i = 0; i < n; ++i) {
    l[i] = std::exp(l[i] - m);
    z += l[i];
  }
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  for (int i = 0; i < n; ++i) {
    const double wi = l[i] / z;
    if (w) w[i] = wi;
    const uint16_t* vrow = V + static_cast<int64_t>(idx[i]) * d;
    for (int c = 0; c < d; ++c) o[c] += wi * bf16_value(vrow[c]);
  }
  *lse = m + std::log(z);
}

// Per block of bs tokens the largest max(s_t, 0), for rows of T scores.
template <class S>
void block_score_rows(const S* s, int64_t rows, int T, int bs, S* sb) {
  const int nb = (T + bs - 1) / bs;
  for (int64_t i = 0; i < rows; ++i)
    for (int j = 0; j < nb; ++j) {
      S m = 0;
      for (int t = j * bs; t < std::min((j + 1) * bs, T); ++t) m = std::max(m, s[i * T + t]);
      sb[i * nb + j] = m;
    }
}

// Ascending token ids of the blocks bidx[0..kb) of bs tokens each, clipped to
// T; returns their number.
int block_tokens_row(const int32_t* bidx, int kb, int bs, int T, int32_t* out) {
  std::vector<int32_t> blocks(bidx, bidx + kb);
  std::sort(blocks.begin(), blocks.end());
  int n = 0;
  for (int32_t j : blocks)
    for (int t = j * bs; t < std::min((j + 1) * bs, T); ++t) out[n++] = t;
  return n;
}

// The hierarchical search over one head's scores s[0..T) keeping k tokens.
template <class S>
void hier_row(const S* s, int T, int k, int32_t* out) {
  std::vector<std::pair<int, int>> parts;  // [begin, end)
  for (int i = 0; i < k; ++i)
    parts.emplace_back(static_cast<int>(static_cast<int64_t>(i) * T / k),
                       static_cast<int>(static_cast<int64_t>(i + 1) * T / k));
  auto longer = [](const std::pair<int, int>& p) { return p.second - p.first > 1; };
  while (std::any_of(parts.begin(), parts.end(), longer)) {
    std::vector<std::pair<int, int>> children;
    for (const auto& p : parts) {
      if (longer(p)) {
        const int m = p.first + (p.second - p.first + 1) / 2;
        children.emplace_back(p.first, m);
        children.emplace_back(m, p.second);
      } else {
        children.push_back(p);
      }
    }
    std::sort(children.begin(), children.end(),
              [s](const std::pair<int, int>& a, const std::pair<int, int>& b) {
                if (s[a.first] != s[b.first]) return s[a.first] > s[b.first];
                return a.first < b.first;
              });
    children.resize(k);
    std::sort(children.begin(), children.end());
    parts = children;
  }
  for (int i = 0; i < k; ++i) out[i] = parts[i].first;
}

}  // namespace

extern "C" {

// out[i] = exact value of the bf16 bits in[i].
void dso_bf16_to_f64(const uint16_t* in, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_value(in[i]);
}

// out[i] = in[i] rounded to float32 (the C++ conversion: nearest, ties to even).
void dso_to_f32(const double* in, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = static_cast<float>(in[i]);
}

// O1.  K [B, Hkv, T, d], C [Hq, r] -> label [B, Hq, T, r].
void dso_label(const uint16_t* K, const int32_t* C, int B, int Hq, int Hkv, int T, int d, int r,
               uint16_t* label) {
  const int G = Hq / Hkv;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hq; ++h) {
      const uint16_t* Kbg = K + (static_cast<int64_t>(b) * Hkv + h / G) * T * d;
      uint16_t* out = label + (static_cast<int64_t>(b) * Hq + h) * T * r;
      for (int t = 0; t < T; ++t)
        for (int j = 0; j < r; ++j)
          out[static_cast<int64_t>(t) * r + j] = Kbg[static_cast<int64_t>(t) * d + C[h * r + j]];
    }
}

// O2.  Q [B, Hq, d], C [Hq, r], label [B, Hq, T, r] -> s [B, Hq, T] (float64).
void dso_score(const uint16_t* Q, const int32_t* C, const uint16_t* label, int B, int Hq, int T,
               int d, int r, double* s) {
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hq; ++h) {
      const uint16_t* q = Q + (static_cast<int64_t>(b) * Hq + h) * d;
      const uint16_t* lab = label + (static_cast<int64_t>(b) * Hq + h) * T * r;
      double* out = s + (static_cast<int64_t>(b) * Hq + h) * T;
      for (int t = 0; t < T; ++t) {
        double acc = 0.0;
        for (int j = 0; j < r; ++j)
          acc += bf16_value(q[C[h * r + j]]) * bf16_value(lab[static_cast<int64_t>(t) * r + j]);
        out[t] = acc;
      }
    }
}

// O3.  s [rows, T] -> idx [rows, k]; 1 <= k <= T (checked by the caller).
void dso_topk_f64(const double* s, int64_t rows, int T, int k, int32_t* idx) {
  for (int64_t i = 0; i < rows; ++i) topk_row(s + i * T, T, k, idx + i * k);
}
void dso_topk_f32(const float* s, int64_t rows, int T, int k, int32_t* idx) {
  for (int64_t i = 0; i < rows; ++i) topk_row(s + i * T, T, k, idx + i * k);
}

// O4.  Q [B, Hq, d], K and V [B, Hkv, T, d], idx [B, Hq, k] -> O [B, Hq, d],
// lse [B, Hq], and the weights w [B, Hq, k] when w is not null.
void dso_attend(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const int32_t* idx,
                int B, int Hq, int Hkv, int T, int d, int k, double scale, double* O,
                double* lse, double* w) {
  const int G = Hq / Hkv;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hq; ++h) {
      const int64_t bh = static_cast<int64_t>(b) * Hq + h;
      const int64_t kv = (static_cast<int64_t>(b) * Hkv + h / G) * T * d;
      attend_row(Q + bh * d, K + kv, V + kv, idx + bh * k, k, d, scale, O + bh * d, lse + bh,
                 w ? w + bh * k : nullptr);
    }
}

// O5.  O4 with every token 0..T-1 kept.
void dso_dense(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int B, int Hq, int Hkv,
               int T, int d, double scale, double* O, double* lse) {
  std::vector<int32_t> all(static_cast<size_t>(B) * Hq * T);
  for (size_t i = 0; i < all.size(); ++i) all[i] = static_cast<int32_t>(i % T);
  dso_attend(Q, K, V, all.data(), B, Hq, Hkv, T, d, T, scale, O, lse, nullptr);
}

// Merge of n chunk results of one query: outs [n, d], lses [n] -> o [d], lse.
void dso_lse_merge(const double* outs, const double* lses, int n, int d, double* o, double* lse) {
  double M = -INFINITY;
  for (int c = 0; c < n; ++c) M = std::max(M, lses[c]);
  double z = 0.0;
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  for (int i = 0; i < n; ++i) {
    const double a = std::exp(lses[i] - M);
    z += a;
    for (int c = 0; c < d; ++c) o[c] += a * outs[static_cast<int64_t>(i) * d + c];
  }
  for (int c = 0; c < d; ++c) o[c] /= z;
  *lse = M + std::log(z);
}

// One query's attention over idx[0..n) cut into n_chunks consecutive chunks
// (the first n % n_chunks one longer; empty chunks dropped), then merged.
void dso_attend_split(const uint16_t* q, const uint16_t* K, const uint16_t* V,
                      const int32_t* idx, int n, int d, double scale, int n_chunks, double* o,
                      double* lse) {
  std::vector<double> outs, lses;
  int start = 0;
  for (int c = 0; c < n_chunks; ++c) {
    const int len = n / n_chunks + (c < n % n_chunks ? 1 : 0);
    if (len == 0) continue;
    outs.resize(outs.size() + d);
    lses.push_back(0.0);
    attend_row(q, K, V, idx + start, len, d, scale, outs.data() + outs.size() - d, &lses.back(),
               nullptr);
    start += len;
  }
  dso_lse_merge(outs.data(), lses.data(), static_cast<int>(lses.size()), d, o, lse);
}

// Calibration importance.  Qc [B, Hq, Nq, d], K [B, Hkv, T_cap, d] (tokens
// 0..T-1) -> I [Hq, d].  |q k| = |q| |k|, so per sequence the double sum over
// (n, t) is the product of the two single sums.
void dso_calib_importance(const uint16_t* Qc, const uint16_t* K, int B, int Hq, int Hkv, int Nq,
                          int T_cap, int T, int d, double* I) {
  const int G = Hq / Hkv;
  for (int i = 0; i < Hq * d; ++i) I[i] = 0.0;
  std::vector<double> ksum(static_cast<size_t>(Hkv) * d), qsum(d);
  for (int b = 0; b < B; ++b) {
    for (int g = 0; g < Hkv; ++g)
      for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int t = 0; t < T; ++t) {
          const int64_t row = (static_cast<int64_t>(b) * Hkv + g) * T_cap + t;
          acc += std::fabs(bf16_value(K[row * d + c]));
        }
        ksum[static_cast<size_t>(g) * d + c] = acc;
      }
    for (int h = 0; h < Hq; ++h) {
      for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int n = 0; n < Nq; ++n)
          acc += std::fabs(bf16_value(Qc[((static_cast<int64_t>(b) * Hq + h) * Nq + n) * d + c]));
        qsum[c] = acc;
      }
      const double* kg = ksum.data() + static_cast<size_t>(h / G) * d;
      for (int c = 0; c < d; ++c) I[h * d + c] += qsum[c] * kg[c];
    }
  }
  const double n = static_cast<double>(B) * Nq * T;
  for (int i = 0; i < Hq * d; ++i) I[i] /= n;
}

// Calibration choice: I [Hq, d] -> C [Hq, r], the r channels of largest
// importance (ties to the lower channel), ascending.
void dso_calib_select(const double* I, int Hq, int d, int r, int32_t* C) {
  dso_topk_f64(I, Hq, d, r, C);
}

// Group scores: s [B, Hq, T] -> sg [B, Hkv, T], the member heads' scores added
// in head order, in the scores' own precision.
void dso_group_score_f64(const double* s, int B, int Hq, int Hkv, int T, double* sg) {
  const int G = Hq / Hkv;
  for (int64_t i = 0; i < static_cast<int64_t>(B) * Hkv * T; ++i) sg[i] = 0.0;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hq; ++h)
      for (int t = 0; t < T; ++t)
        sg[(static_cast<int64_t>(b) * Hkv + h / G) * T + t] +=
            s[(static_cast<int64_t>(b) * Hq + h) * T + t];
}
void dso_group_score_f32(const float* s, int B, int Hq, int Hkv, int T, float* sg) {
  const int G = Hq / Hkv;
  for (int64_t i = 0; i < static_cast<int64_t>(B) * Hkv * T; ++i) sg[i] = 0.0f;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hq; ++h)
      for (int t = 0; t < T; ++t)
        sg[(static_cast<int64_t>(b) * Hkv + h / G) * T + t] +=
            s[(static_cast<int64_t>(b) * Hq + h) * T + t];
}

// Group attention: query head h attends over its group's set idx_g [B, Hkv, k].
void dso_group_attend(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                      const int32_t* idx_g, int B, int Hq, int Hkv, int T, int d, int k,
                      double scale, double* O, double* lse) {
  const int G = Hq / Hkv;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hq; ++h) {
      const int64_t bh = static_cast<int64_t>(b) * Hq + h;
      const int64_t bg = static_cast<int64_t>(b) * Hkv + h / G;
      attend_row(Q + bh * d, K + bg * T * d, V + bg * T * d, idx_g + bg * k, k, d, scale,
                 O + bh * d, lse + bh, nullptr);
    }
}

// Block scores: s [rows, T] -> sb [rows, ceil(T / bs)], per block the largest
// max(s_t, 0) (the last block may be short).
void dso_block_score_f64(const double* s, int64_t rows, int T, int bs, double* sb) {
  block_score_rows(s, rows, T, bs, sb);
}
void dso_block_score_f32(const float* s, int64_t rows, int T, int bs, float* sb) {
  block_score_rows(s, rows, T, bs, sb);
}

// Token ids of one head's blocks (ascending, clipped to T); returns the count.
int dso_block_tokens(const int32_t* bidx, int kb, int bs, int T, int32_t* out) {
  return block_tokens_row(bidx, kb, bs, T, out);
}

// Block attention: each head over the tokens of its blocks bidx [B, Hq, kb].
void dso_block_attend(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                      const int32_t* bidx, int B, int Hq, int Hkv, int T, int d, int kb, int bs,
                      double scale, double* O, double* lse) {
  const int G = Hq / Hkv;
  std::vector<int32_t> toks(static_cast<size_t>(kb) * bs);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hq; ++h) {
      const int64_t bh = static_cast<int64_t>(b) * Hq + h;
      const int64_t bg = static_cast<int64_t>(b) * Hkv + h / G;
      const int n = block_tokens_row(bidx + bh * kb, kb, bs, T, toks.data());
      attend_row(Q + bh * d, K + bg * T * d, V + bg * T * d, toks.data(), n, d, scale,
                 O + bh * d, lse + bh, nullptr);
    }
}

// Hierarchical top-k: s [rows, T] -> idx [rows, k]; 1 <= k <= T.
void dso_hier_topk_f64(const double* s, int64_t rows, int T, int k, int32_t* idx) {
  for (int64_t i = 0; i < rows; ++i) hier_row(s + i * T, T, k, idx + i * k);
}
void dso_hier_topk_f32(const float* s, int64_t rows, int T, int k, int32_t* idx) {
  for (int64_t i = 0; i < rows; ++i) hier_row(s + i * T, T, k, idx + i * k);
}

// The decode step of n independent heads spread over host threads (the CPU
// baseline: the same per-head steps, the heads shared out by a counter).  Head
// i has the query Qs[i] [d], channel ids Cs[i] [r], label rows Ls[i] [T, r] and
// its KV head's rows Ks[i], Vs[i] [T, d].  mode bit 1: O2 score in float64,
// rounded to float32, O3 top-k of k tokens, O4 attention over them -> O[i],
// lse[i]; mode bit 2: O5 dense attention over all T rows -> Od[i], lsed[i].
// nthreads <= 0 uses std::thread::hardware_concurrency().  Returns the number
// of threads used.
int dso_step_heads_mt(const uint16_t* Qs, const int32_t* Cs, const uint16_t* Ls,
                      const uint16_t* Ks, const uint16_t* Vs, int n, int T, int d, int r, int k,
                      double scale, int mode, int nthreads, double* O, double* lse, double* Od,
                      double* lsed) {
  if (nthreads <= 0) nthreads = static_cast<int>(std::thread::hardware_concurrency());
  if (nthreads <= 0) nthreads = 1;
  std::atomic<int> next{0};
  auto worker = [&]() {
    std::vector<double> s(T);
    std::vector<float> s32(T);
    std::vector<int32_t> idx(k), all;
    if (mode & 2) {
      all.resize(T);
      std::iota(all.begin(), all.end(), 0);
    }
    for (int i = next.fetch_add(1); i < n; i = next.fetch_add(1)) {
      const uint16_t* q = Qs + static_cast<int64_t>(i) * d;
      const int32_t* C = Cs + static_cast<int64_t>(i) * r;
      const uint16_t* K = Ks + static_cast<int64_t>(i) * T * d;
      const uint16_t* V = Vs + static_cast<int64_t>(i) * T * d;
      if (mode & 1) {
        const uint16_t* lab = Ls + static_cast<int64_t>(i) * T * r;
        for (int t = 0; t < T; ++t) {
          double acc = 0.0;
          for (int j = 0; j < r; ++j)
            acc += bf16_value(q[C[j]]) * bf16_value(lab[static_cast<int64_t>(t) * r + j]);
          s[t] = acc;
          s32[t] = static_cast<float>(acc);
        }
        topk_row(s32.data(), T, k, idx.data());
        attend_row(q, K, V, idx.data(), k, d, scale, O + static_cast<int64_t>(i) * d, lse + i,
                   nullptr);
      }
      if (mode & 2)
        attend_row(q, K, V, all.data(), T, d, scale, Od + static_cast<int64_t>(i) * d, lsed + i,
                   nullptr);
    }
  };
  std::vector<std::thread> pool;
  for (int t = 0; t < nthreads; ++t) pool.emplace_back(worker);
  for (auto& th : pool) th.join();
  return nthreads;
}

}  // extern "C"
