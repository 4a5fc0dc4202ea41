// Plain C++ oracle of Double-Sparsity-style decode attention, steps O1-O5:
// label gather, channel-sparse score, top-k, softmax attention over the kept
// rows, dense attention; plus the log-sum-exp merge of split attention.
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
//
// Every value is decoded exactly from its bf16 bits and every step runs in
// double precision (std::exp, std::log); the order of the top-k is decided by
// std::sort on the stated total order.  Plain loops, no blocking or fusion.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
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

}  // extern "C"
