/*
 * Seeded synthetic inputs for exact batched k-means (Lloyd) runs.
 *
 * This module is shared by the fp64 oracle's tests and by the GPU path's tests
 * and benchmark.  It holds NO k-means arithmetic: it only draws random numbers
 * and lays out points and initial-centroid indices.  The pages about
 * Flash-KMeans benchmark on random data ("Flash-KMeans" GitHub README, Usage:
 * points drawn with torch.randn; Large tensor Benchmark: inputs generated
 * randomly in CPU pinned memory), so every workload here is a seeded Gaussian
 * mixture or a plain standard normal.
 *
 * Random numbers: Philox4x32-10, the counter-based generator of Salmon,
 * Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3"
 * (SC'11), restated from its published definition (two 32x32->64 multiplies
 * per round, Weyl key schedule, ten rounds).  Normals come from the Box-Muller
 * transform; Gamma variates (for Dirichlet weights) from Marsaglia and Tsang,
 * "A simple method for generating gamma variables" (ACM TOMS 2000), with the
 * alpha<1 boost Gamma(a) = Gamma(a+1) * U^(1/a).
 *
 * Every value is a pure function of (seed, stream, counter), so generation is
 * parallel (OpenMP) and bit-reproducible regardless of thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

/* stream purposes (the high byte of key word 1) */
enum { P_MEANS = 1, P_NOISE = 2, P_LABEL = 3, P_GAMMA = 4, P_PERM = 5 };
/* dtype codes, identical to the library's public enum */
enum { DT_F32 = 0, DT_F16 = 1, DT_BF16 = 2 };
/* component-weight kinds */
enum { W_EQUAL = 0, W_DIRICHLET = 1, W_ZIPF = 2 };

static inline void philox_round(uint32_t c[4], const uint32_t k[2]) {
  uint64_t p0 = (uint64_t)PHILOX_M0 * c[0];
  uint64_t p1 = (uint64_t)PHILOX_M1 * c[2];
  uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
  uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
  uint32_t n0 = hi1 ^ c[1] ^ k[0];
  uint32_t n2 = hi0 ^ c[3] ^ k[1];
  c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
}

static inline void philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
  uint32_t k[2] = {key[0], key[1]};
  for (int r = 0; r < 10; ++r) {
    philox_round(c, k);
    k[0] += PHILOX_W0;
    k[1] += PHILOX_W1;
  }
  out[0] = c[0]; out[1] = c[1]; out[2] = c[2]; out[3] = c[3];
}

/* exported only so the tests can check the generator against published answers */
void fkmgen_philox(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  philox4x32_10(ctr, key, out);
}

static inline void make_key(uint64_t seed, int purpose, uint32_t batch, uint32_t key[2]) {
  key[0] = (uint32_t)seed;
  key[1] = ((uint32_t)(seed >> 32)) ^ ((uint32_t)purpose << 24) ^ (batch & 0xFFFFFFu);
}

static inline void draw(const uint32_t key[2], uint64_t i, uint32_t j, uint32_t out[4]) {
  uint32_t ctr[4] = {(uint32_t)i, (uint32_t)(i >> 32), j, 0u};
  philox4x32_10(ctr, key, out);
}

/* uniform double in the open interval (0,1) from two 32-bit words (53 bits) */
static inline double u53(uint32_t a, uint32_t b) {
  uint64_t m = ((uint64_t)(a >> 5) << 26) | (uint64_t)(b >> 6);
  return ((double)m + 0.5) * (1.0 / 9007199254740992.0);
}

/* two standard normals (Box-Muller) from one Philox block */
static inline void normal_pair(const uint32_t r[4], double* z0, double* z1) {
  double u1 = u53(r[0], r[1]);
  double u2 = u53(r[2], r[3]);
  double rad = sqrt(-2.0 * log(u1));
  double th = 6.283185307179586476925286766559 * u2;
  *z0 = rad * cos(th);
  *z1 = rad * sin(th);
}

/* element e of the normal stream (key): pairs share one Philox block */
static inline double normal_at(const uint32_t key[2], uint64_t e) {
  uint32_t r[4];
  draw(key, e >> 1, 0u, r);
  double z0, z1;
  normal_pair(r, &z0, &z1);
  return (e & 1) ? z1 : z0;
}

/* ---- storage rounding (input preparation: the rounded value IS the input) ---- */
static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

static inline uint16_t f32_to_f16_rne(float f) {
  _Float16 h = (_Float16)f;
  uint16_t u;
  memcpy(&u, &h, 2);
  return u;
}

static inline void store(void* out, int dtype, uint64_t idx, double v) {
  float f = (float)v;
  if (dtype == DT_F32) ((float*)out)[idx] = f;
  else if (dtype == DT_BF16) ((uint16_t*)out)[idx] = f32_to_bf16_rne(f);
  else ((uint16_t*)out)[idx] = f32_to_f16_rne(f);
}

/* Gamma(alpha) with alpha > 0, drawn with a per-variate counter stream */
static double gamma_draw(const uint32_t key[2], uint64_t var, double alpha) {
  double boost = 1.0;
  double a = alpha;
  uint32_t attempt = 0;
  if (alpha < 1.0) {
    uint32_t r[4];
    draw(key, var, 0xFFFFFFFFu, r);
    boost = pow(u53(r[0], r[1]), 1.0 / alpha);
    a = alpha + 1.0;
  }
  double d = a - 1.0 / 3.0;
  double c = 1.0 / sqrt(9.0 * d);
  for (;;) {
    uint32_t r[4];
    draw(key, var, attempt++, r);
    double z, z1;
    normal_pair(r, &z, &z1);
    double v = 1.0 + c * z;
    if (v <= 0.0) continue;
    v = v * v * v;
    uint32_t s[4];
    draw(key, var, 0x80000000u | attempt, s);
    double u = u53(s[0], s[1]);
    if (log(u) < 0.5 * z * z + d - d * v + d * log(v)) return d * v * boost;
  }
}

/* Component weights -> cumulative distribution (length n_comp). */
static void component_cdf(uint64_t seed, uint32_t batch, int n_comp, int wkind, double wparam,
                          double* cdf) {
  uint32_t key[2];
  make_key(seed, P_GAMMA, batch, key);
  double tot = 0.0;
  for (int j = 0; j < n_comp; ++j) {
    double w;
    if (wkind == W_DIRICHLET) w = gamma_draw(key, (uint64_t)j, wparam);
    else if (wkind == W_ZIPF) w = pow((double)(j + 1), -wparam);
    else w = 1.0;
    tot += w;
    cdf[j] = tot;
  }
  for (int j = 0; j < n_comp; ++j) cdf[j] /= tot;
  cdf[n_comp - 1] = 1.0;
}

static inline int pick_component(const double* cdf, int n, double u) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (u <= cdf[mid]) hi = mid; else lo = mid + 1;
  }
  return lo;
}

/*
 * Points of one batch: N x D row-major, written in `dtype` into out.
 *   n_comp == 0 : x ~ N(0, sigma^2 I)   (no cluster structure)
 *   n_comp  > 0 : Gaussian mixture, means ~ N(0, mean_std^2 I), isotropic
 *                 spread sigma, weights equal / Dirichlet(wparam) / Zipf(wparam)
 * labels (optional, may be NULL) receives each point's mixture component.
 * Returns 0, or -1 on a bad argument / allocation failure.
 */
int fkmgen_points(int64_t N, int D, int dtype, uint64_t seed, uint32_t batch, int n_comp,
                  int wkind, double wparam, double mean_std, double sigma, void* out,
                  int32_t* labels) {
  if (N < 0 || D <= 0 || !out || n_comp < 0 || dtype < 0 || dtype > 2) return -1;
  uint32_t knoise[2], klabel[2], kmean[2];
  make_key(seed, P_NOISE, batch, knoise);
  make_key(seed, P_LABEL, batch, klabel);
  make_key(seed, P_MEANS, batch, kmean);
  double* cdf = NULL;
  double* means = NULL;
  if (n_comp > 0) {
    cdf = (double*)malloc(sizeof(double) * (size_t)n_comp);
    means = (double*)malloc(sizeof(double) * (size_t)n_comp * (size_t)D);
    if (!cdf || !means) { free(cdf); free(means); return -1; }
    component_cdf(seed, batch, n_comp, wkind, wparam, cdf);
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < (int64_t)n_comp * D; ++e) means[e] = mean_std * normal_at(kmean, (uint64_t)e);
  }
  const uint64_t DD = (uint64_t)D;
#pragma omp parallel for schedule(static, 256)
  for (int64_t i = 0; i < N; ++i) {
    int comp = 0;
    if (n_comp > 0) {
      uint32_t r[4];
      draw(klabel, (uint64_t)i, 0u, r);
      comp = pick_component(cdf, n_comp, u53(r[0], r[1]));
    }
    if (labels) labels[i] = comp;
    const double* mu = n_comp > 0 ? means + (size_t)comp * DD : NULL;
    uint64_t base = (uint64_t)i * DD;
    for (int d = 0; d < D; d += 2) {
      uint32_t r[4];
      draw(knoise, (base + (uint64_t)d) >> 1, 0u, r);
      double z0, z1;
      normal_pair(r, &z0, &z1);
      if (D & 1) { /* odd D: fall back to the element-indexed form */
        z0 = normal_at(knoise, base + (uint64_t)d);
        z1 = (d + 1 < D) ? normal_at(knoise, base + (uint64_t)d + 1) : 0.0;
      }
      double v0 = sigma * z0 + (mu ? mu[d] : 0.0);
      store(out, dtype, base + (uint64_t)d, v0);
      if (d + 1 < D) {
        double v1 = sigma * z1 + (mu ? mu[d + 1] : 0.0);
        store(out, dtype, base + (uint64_t)d + 1, v1);
      }
    }
  }
  free(cdf);
  free(means);
  return 0;
}

/* ---- first K entries of a seeded Fisher-Yates permutation of [0, N) ---- */
typedef struct { int64_t* keys; int64_t* vals; uint64_t mask; } swapmap;

static int64_t sm_get(const swapmap* m, int64_t k) {
  uint64_t h = ((uint64_t)k * 0x9E3779B97F4A7C15ull) & m->mask;
  while (m->keys[h] != -1) {
    if (m->keys[h] == k) return m->vals[h];
    h = (h + 1) & m->mask;
  }
  return k;
}

static void sm_put(swapmap* m, int64_t k, int64_t v) {
  uint64_t h = ((uint64_t)k * 0x9E3779B97F4A7C15ull) & m->mask;
  while (m->keys[h] != -1 && m->keys[h] != k) h = (h + 1) & m->mask;
  m->keys[h] = k;
  m->vals[h] = v;
}

/* out[t] = perm[t], t < K, where perm is the Fisher-Yates shuffle of [0,N)
 * driven by uniforms from the (seed, batch) PERM stream.  Returns 0 / -1. */
int fkmgen_perm_prefix(int64_t N, int64_t K, uint64_t seed, uint32_t batch, int64_t* out) {
  if (N <= 0 || K < 0 || K > N || !out) return -1;
  uint64_t cap = 16;
  while (cap < (uint64_t)(4 * K + 16)) cap <<= 1;
  swapmap m;
  m.keys = (int64_t*)malloc(sizeof(int64_t) * cap);
  m.vals = (int64_t*)malloc(sizeof(int64_t) * cap);
  m.mask = cap - 1;
  if (!m.keys || !m.vals) { free(m.keys); free(m.vals); return -1; }
  for (uint64_t h = 0; h < cap; ++h) m.keys[h] = -1;
  uint32_t key[2];
  make_key(seed, P_PERM, batch, key);
  for (int64_t t = 0; t < K; ++t) {
    uint32_t r[4];
    draw(key, (uint64_t)t, 0u, r);
    int64_t span = N - t;
    int64_t off = (int64_t)(u53(r[0], r[1]) * (double)span);
    if (off >= span) off = span - 1;
    int64_t j = t + off;
    int64_t at = sm_get(&m, t), aj = sm_get(&m, j);
    sm_put(&m, t, aj);
    sm_put(&m, j, at);
    out[t] = aj;
  }
  free(m.keys);
  free(m.vals);
  return 0;
}
