/*
 * Seeded synthetic inputs for token-sparse decode attention.
 *
 * This generator is shared by the CPU oracle and the GPU path: both see the
 * same bf16 bit patterns.  It holds none of the attention method's
 * arithmetic; it only draws Q, K, V, the per-head channel permutation, and the
 * heavy-hitter token positions of the long-context workload.
 *
 * Random numbers: the splitmix64 sequence (Steele, Lea and Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014), read by counter:
 * draw(stream, i) is output number i+1 of splitmix64 started from `stream`,
 * i.e. mix64(stream + (i + 1) * gamma).  Any element can therefore be drawn
 * on its own, so a single (batch, head) slab can be regenerated without the
 * rest of the tensor.
 *
 * Normals: Box-Muller (Box and Muller, 1958) in double precision.  Element e
 * of a tensor uses the pair (draw(2p), draw(2p+1)) with p = e / 2 and takes
 * the cosine branch for even e and the sine branch for odd e.
 *
 * bf16: float32 rounded to nearest, ties to even, keeping the top 16 bits.
 *
 * Workload structure (stands in for Llama-2-shaped KV caches):
 *   - per query head h, a Fisher-Yates permutation pi_h of the d channels;
 *     its first n_out entries are h's outlier channels;
 *   - Q[b,h,c] ~ N(0,1), times 6 on h's outlier channels;
 *   - K[b,g,t,c] ~ N(0,1), times 6 on the union of the outlier channels of
 *     the query heads that share KV head g (each channel scaled once);
 *   - V ~ N(0,1);
 *   - calibration queries Qc[b,h,n,c] (n < Nq) drawn like Q from a stream of
 *     their own (the offline calibration set of the channel selection);
 *   - optionally n_hh heavy-hitter positions per query head h, where the
 *     channels of C_h (the first r entries of pi_h) of K are overwritten with
 *     6*sqrt(r)*q[C_h]/||q[C_h]||_2, so that those tokens score high.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define GAMMA 0x9E3779B97F4A7C15ull

enum { TID_Q = 1, TID_K = 2, TID_V = 3, TID_PERM = 4, TID_HH = 5, TID_QCAL = 6 };

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline uint64_t stream_of(uint64_t seed, uint64_t tensor_id) {
  return mix64(seed + GAMMA * (tensor_id + 1)) ^ (tensor_id << 56);
}

static inline uint64_t draw(uint64_t stream, uint64_t i) {
  return mix64(stream + (i + 1) * GAMMA);
}

/* uniform integer in [0, n), by the multiply-shift mapping of the top 32 bits */
static inline uint32_t draw_below(uint64_t stream, uint64_t i, uint32_t n) {
  return (uint32_t)(((draw(stream, i) >> 32) * (uint64_t)n) >> 32);
}

static inline double normal_at(uint64_t stream, uint64_t e) {
  uint64_t p = e >> 1;
  double u1 = ((double)((draw(stream, 2 * p) >> 11) + 1)) * 0x1.0p-53; /* (0,1] */
  double u2 = ((double)(draw(stream, 2 * p + 1) >> 11)) * 0x1.0p-53;  /* [0,1) */
  double rad = sqrt(-2.0 * log(u1));
  double ang = 6.283185307179586476925286766559 * u2;
  return (e & 1) ? rad * sin(ang) : rad * cos(ang);
}

/* out[i] = normal number e0 + i, for i in [0, n); each pair is computed once. */
static void normals(uint64_t stream, uint64_t e0, size_t n, double* out) {
  size_t i = 0;
  if (n && (e0 & 1)) out[i++] = normal_at(stream, e0);
  for (; i + 1 < n; i += 2) {
    uint64_t p = (e0 + i) >> 1;
    double u1 = ((double)((draw(stream, 2 * p) >> 11) + 1)) * 0x1.0p-53;
    double u2 = ((double)(draw(stream, 2 * p + 1) >> 11)) * 0x1.0p-53;
    double rad = sqrt(-2.0 * log(u1));
    double ang = 6.283185307179586476925286766559 * u2;
    out[i] = rad * cos(ang);
    out[i + 1] = rad * sin(ang);
  }
  if (i < n) out[i] = normal_at(stream, e0 + i);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t bias = 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)((u + bias) >> 16);
}

static inline double bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* ---- channel permutation -------------------------------------------------- */

/* perm[d]: Fisher-Yates shuffle of 0..d-1 for query head h. */
void dsgen_perm_head(uint64_t seed, int h, int d, int32_t* perm) {
  uint64_t s = stream_of(seed, TID_PERM);
  for (int c = 0; c < d; ++c) perm[c] = c;
  for (int i = d - 1; i >= 1; --i) {
    uint32_t j = draw_below(s, (uint64_t)h * (uint64_t)d + (uint64_t)i, (uint32_t)(i + 1));
    int32_t tmp = perm[i];
    perm[i] = perm[j];
    perm[j] = tmp;
  }
}

static int cmp_i32(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/* C[Hq, r]: the first r entries of each head's permutation, ascending. */
int dsgen_channels(uint64_t seed, int Hq, int d, int r, int32_t* C) {
  if (Hq <= 0 || d <= 0 || r <= 0 || r > d) return -1;
  int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)d);
  if (!perm) return -2;
  for (int h = 0; h < Hq; ++h) {
    dsgen_perm_head(seed, h, d, perm);
    memcpy(C + (size_t)h * r, perm, sizeof(int32_t) * (size_t)r);
    qsort(C + (size_t)h * r, (size_t)r, sizeof(int32_t), cmp_i32);
  }
  free(perm);
  return 0;
}

/* ---- slabs ------------------------------------------------------------------ */

typedef struct {
  uint64_t seed;
  int B, Hq, Hkv, d, T, n_out, r_hh, n_hh;
} dsgen_dims;

/* Q[b,h,0:d] */
static void q_slab(const dsgen_dims* D, int b, int h, uint16_t* out) {
  uint64_t s = stream_of(D->seed, TID_Q);
  int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)D->d);
  char* outlier = (char*)calloc((size_t)D->d, 1);
  dsgen_perm_head(D->seed, h, D->d, perm);
  for (int i = 0; i < D->n_out && i < D->d; ++i) outlier[perm[i]] = 1;
  uint64_t base = ((uint64_t)b * D->Hq + h) * (uint64_t)D->d;
  double* z = (double*)malloc(sizeof(double) * (size_t)D->d);
  normals(s, base, (size_t)D->d, z);
  for (int c = 0; c < D->d; ++c) {
    float f = (float)z[c];
    if (outlier[c]) f *= 6.0f;
    out[c] = f32_to_bf16_rne(f);
  }
  free(z);
  free(outlier);
  free(perm);
}

/* Heavy-hitter positions of query head h: the first n_hh entries of a partial
 * Fisher-Yates shuffle of 0..T-1. */
static void hh_positions(const dsgen_dims* D, int h, int32_t* pos) {
  uint64_t s = stream_of(D->seed, TID_HH);
  int32_t* a = (int32_t*)malloc(sizeof(int32_t) * (size_t)D->T);
  for (int t = 0; t < D->T; ++t) a[t] = t;
  for (int i = 0; i < D->n_hh; ++i) {
    uint32_t j = (uint32_t)i + draw_below(s, (uint64_t)h * (uint64_t)D->T + (uint64_t)i,
                                          (uint32_t)(D->T - i));
    int32_t tmp = a[i];
    a[i] = a[j];
    a[j] = tmp;
  }
  memcpy(pos, a, sizeof(int32_t) * (size_t)D->n_hh);
  free(a);
}

/* K[b,g,0:T,0:d] (which == TID_K) or V[b,g,0:T,0:d] (which == TID_V) */
static void kv_slab(const dsgen_dims* D, int which, int b, int g, uint16_t* out) {
  const int d = D->d, T = D->T, G = D->Hq / D->Hkv;
  uint64_t s = stream_of(D->seed, (uint64_t)which);
  char* outlier = (char*)calloc((size_t)d, 1);
  if (which == TID_K) {
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)d);
    for (int h = g * G; h < (g + 1) * G; ++h) {
      dsgen_perm_head(D->seed, h, d, perm);
      for (int i = 0; i < D->n_out && i < d; ++i) outlier[perm[i]] = 1;
    }
    free(perm);
  }
  uint64_t base = ((uint64_t)b * D->Hkv + g) * (uint64_t)T * (uint64_t)d;
  double* z = (double*)malloc(sizeof(double) * (size_t)d);
  for (int t = 0; t < T; ++t) {
    normals(s, base + (uint64_t)t * d, (size_t)d, z);
    for (int c = 0; c < d; ++c) {
      float f = (float)z[c];
      if (outlier[c]) f *= 6.0f;
      out[(size_t)t * d + c] = f32_to_bf16_rne(f);
    }
  }
  free(z);
  free(outlier);
  if (which == TID_K && D->n_hh > 0 && D->r_hh > 0) {
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)d);
    int32_t* pos = (int32_t*)malloc(sizeof(int32_t) * (size_t)D->n_hh);
    uint16_t* q = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)d);
    for (int h = g * G; h < (g + 1) * G; ++h) {
      dsgen_perm_head(D->seed, h, d, perm);
      qsort(perm, (size_t)D->r_hh, sizeof(int32_t), cmp_i32);
      q_slab(D, b, h, q);
      double nrm = 0.0;
      for (int j = 0; j < D->r_hh; ++j) {
        double v = bf16_to_f64(q[perm[j]]);
        nrm += v * v;
      }
      nrm = sqrt(nrm);
      if (nrm == 0.0) continue;
      double amp = 6.0 * sqrt((double)D->r_hh) / nrm;
      hh_positions(D, h, pos);
      for (int i = 0; i < D->n_hh; ++i) {
        uint16_t* row = out + (size_t)pos[i] * d;
        for (int j = 0; j < D->r_hh; ++j) {
          int c = perm[j];
          row[c] = f32_to_bf16_rne((float)(amp * bf16_to_f64(q[c])));
        }
      }
    }
    free(q);
    free(pos);
    free(perm);
  }
}

/* ---- public entry points -------------------------------------------------- */

static int check_dims(const dsgen_dims* D) {
  if (D->B <= 0 || D->Hq <= 0 || D->Hkv <= 0 || D->d <= 0 || D->T <= 0) return -1;
  if (D->Hq % D->Hkv) return -1;
  if (D->n_out < 0 || D->n_out > D->d) return -1;
  if (D->n_hh < 0 || D->n_hh > D->T) return -1;
  if (D->r_hh < 0 || D->r_hh > D->d) return -1;
  return 0;
}

int dsgen_q_slab(uint64_t seed, int B, int Hq, int Hkv, int d, int T, int n_out, int r_hh,
                 int n_hh, int b, int h, uint16_t* out) {
  dsgen_dims D = {seed, B, Hq, Hkv, d, T, n_out, r_hh, n_hh};
  if (check_dims(&D) || b < 0 || b >= B || h < 0 || h >= Hq) return -1;
  q_slab(&D, b, h, out);
  return 0;
}

/* which: 0 = K, 1 = V */
int dsgen_kv_slab(uint64_t seed, int B, int Hq, int Hkv, int d, int T, int n_out, int r_hh,
                  int n_hh, int which, int b, int g, uint16_t* out) {
  dsgen_dims D = {seed, B, Hq, Hkv, d, T, n_out, r_hh, n_hh};
  if (check_dims(&D) || b < 0 || b >= B || g < 0 || g >= Hkv || (which != 0 && which != 1))
    return -1;
  kv_slab(&D, which == 0 ? TID_K : TID_V, b, g, out);
  return 0;
}

typedef struct {
  const dsgen_dims* D;
  uint16_t *Q, *K, *V;
  int next; /* shared job counter */
  pthread_mutex_t mu;
} job_pool;

static void* worker(void* arg) {
  job_pool* P = (job_pool*)arg;
  const dsgen_dims* D = P->D;
  const int nq = D->B * D->Hq, nkv = D->B * D->Hkv;
  const int total = nq + 2 * nkv;
  for (;;) {
    pthread_mutex_lock(&P->mu);
    int j = P->next++;
    pthread_mutex_unlock(&P->mu);
    if (j >= total) break;
    if (j < nq) {
      if (P->Q) q_slab(D, j / D->Hq, j % D->Hq, P->Q + (size_t)j * D->d);
    } else {
      int kj = j - nq;
      int which = kj < nkv ? TID_K : TID_V;
      int s = kj % nkv;
      uint16_t* dst = which == TID_K ? P->K : P->V;
      if (dst)
        kv_slab(D, which, s / D->Hkv, s % D->Hkv, dst + (size_t)s * D->T * (size_t)D->d);
    }
  }
  return NULL;
}

/* Q[B,Hq,d], K[B,Hkv,T,d], V[B,Hkv,T,d] as bf16 bits; any of them may be NULL.
 * nthreads <= 0 uses every online core. */
int dsgen_qkv(uint64_t seed, int B, int Hq, int Hkv, int d, int T, int n_out, int r_hh, int n_hh,
              uint16_t* Q, uint16_t* K, uint16_t* V, int nthreads) {
  dsgen_dims D = {seed, B, Hq, Hkv, d, T, n_out, r_hh, n_hh};
  if (check_dims(&D)) return -1;
  if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  job_pool P;
  P.D = &D;
  P.Q = Q;
  P.K = K;
  P.V = V;
  P.next = 0;
  pthread_mutex_init(&P.mu, NULL);
  pthread_t th[256];
  for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &P);
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  pthread_mutex_destroy(&P.mu);
  return 0;
}

/* Calibration queries Qc[B,Hq,Nq,d] as bf16 bits: N(0,1), times 6 on each
 * head's outlier channels, element ((b*Hq + h)*Nq + n)*d + c of their stream. */
int dsgen_q_calib(uint64_t seed, int B, int Hq, int d, int n_out, int Nq, uint16_t* out) {
  if (B < 1 || Hq < 1 || d < 1 || Nq < 1 || n_out < 0 || n_out > d) return -1;
  uint64_t s = stream_of(seed, TID_QCAL);
  int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)d);
  char* outlier = (char*)malloc((size_t)d);
  double* z = (double*)malloc(sizeof(double) * (size_t)d * (size_t)Nq);
  for (int h = 0; h < Hq; ++h) {
    memset(outlier, 0, (size_t)d);
    dsgen_perm_head(seed, h, d, perm);
    for (int i = 0; i < n_out; ++i) outlier[perm[i]] = 1;
    for (int b = 0; b < B; ++b) {
      uint64_t base = ((uint64_t)b * Hq + h) * (uint64_t)Nq * (uint64_t)d;
      normals(s, base, (size_t)Nq * (size_t)d, z);
      uint16_t* o = out + base;
      for (int e = 0; e < Nq * d; ++e) {
        float f = (float)z[e];
        if (outlier[e % d]) f *= 6.0f;
        o[e] = f32_to_bf16_rne(f);
      }
    }
  }
  free(z);
  free(outlier);
  free(perm);
  return 0;
}

/* Heavy-hitter positions [Hq, n_hh] (in draw order, not sorted). */
int dsgen_hh_positions(uint64_t seed, int B, int Hq, int Hkv, int d, int T, int n_out, int r_hh,
                       int n_hh, int32_t* pos) {
  dsgen_dims D = {seed, B, Hq, Hkv, d, T, n_out, r_hh, n_hh};
  if (check_dims(&D)) return -1;
  for (int h = 0; h < Hq; ++h) hh_positions(&D, h, pos + (size_t)h * n_hh);
  return 0;
}
