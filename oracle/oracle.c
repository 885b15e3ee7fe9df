/*
 * fp64 CPU ORACLE for exact batched Lloyd k-means.  TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the package's smoke check and the benchmark's CPU
 * baseline may load this file's library.  It shares no code, header, table or
 * helper with the CUDA path, and the CUDA path never calls it.
 *
 * What it computes (one Lloyd iteration = assign then update), written out as
 * the plain definitions, with no blocking, fusion or reordering:
 *
 *   objective   min over (a, C) of  sum_i || x_i - c_{a_i} ||^2
 *               [Flash-KMeans paper summary at paper.rainbus.top, section
 *                "前置知识 / K-Means聚类算法" (prerequisites: the k-means algorithm)]
 *   assign      a_i = argmin_k || x_i - c_k ||^2, each point to its nearest centroid
 *               [same page, same section; and "Flash-KMeans: Fast and
 *                Memory-Efficient Exact K-Means" summary, section "Method"]
 *   update      c_k = s_k / n_k, s_k the sum and n_k the number of points
 *               assigned to k [rainbus page, section "方法步骤详情" (method
 *                step details), end of step (2)]
 *
 * Distances are the DIRECT squared difference sum_d (x_d - c_d)^2 in fp64, not
 * the expanded ||x||^2 + ||c||^2 - 2 x.c form the GPU kernels use (rainbus page,
 * "核心方法" (core method)); the expanded form is what is being checked.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - ties in the argmin go to the lowest centroid index;
 *   - an empty cluster keeps its previous centroid;
 *   - shift_b = sum_k ||c_k(t+1) - c_k(t)||^2; the loop stops after an update
 *     when max_b shift_b < tol (strict, so tol = 0 runs every iteration);
 *   - inertia is the objective of the LAST assignment, against the centroids
 *     that assignment used; ids are that assignment; centers come from the
 *     update that followed it;
 *   - "mirror" mode: the assign step measures distances to
 *         c_hat = m + q(fp32(fp32(c) - m)),
 *     with m the batch's mean centroid (the fp64 sum of the fp32 centroids
 *     in index order, divided by K, rounded to fp32) and q() round-to-nearest-
 *     even to the points' storage type (bf16 or fp16).  That is the precision
 *     contract "assignment operands are in the input dtype", applied to the
 *     centroids' offsets from their mean: k-means is translation invariant,
 *     so centring is exact ("Flash-KMeans" README, section "Centre your
 *     data"), and it keeps the rounding relative to the spread of the
 *     centroids rather than to their distance from the origin.  "Pure" mode
 *     uses c as is.
 *
 * Stable argsort: a counting sort, the textbook stable argsort of small
 * integer keys [rainbus page, "前置知识 / argsort与分段规约" (argsort and
 * segmented reduction), which works the example [3,1,2,1,3,2]].
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* storage dtype codes of the points */
enum { ORC_F32 = 0, ORC_F16 = 1, ORC_BF16 = 2 };
/* mirror argument: -1 = pure mode, otherwise the dtype centroids are rounded to */
#define ORC_PURE (-1)

/* ---------- reading stored points exactly into fp64 ---------- */
static inline double orc_read(const void* x, int dt, int64_t idx) {
  if (dt == ORC_F32) return (double)((const float*)x)[idx];
  if (dt == ORC_F16) {
    _Float16 h;
    memcpy(&h, (const uint16_t*)x + idx, 2);
    return (double)h;
  }
  uint32_t u = ((uint32_t)((const uint16_t*)x)[idx]) << 16; /* bf16 = top half of an fp32 */
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* ---------- the storage-type rounding of "mirror" mode ---------- */
/* fp32 -> bf16, round to nearest, ties to even: keep the top 16 bits after
 * adding half an ulp of bf16 (0x7FFF) plus the parity of the kept lsb. */
static double orc_round_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) != 0x7F800000u) {
    uint32_t keep_lsb = (u >> 16) & 1u;
    u = (u + 0x7FFFu + keep_lsb) & 0xFFFF0000u;
  } else {
    u &= 0xFFFF0000u;
  }
  float r;
  memcpy(&r, &u, 4);
  return (double)r;
}

static double orc_round_f16(float f) {
  _Float16 h = (_Float16)f; /* IEEE binary16, round to nearest even */
  return (double)h;
}

/* q(fp32(v)) elementwise in mirror mode, v in pure mode (n values) */
void orc_quantise(const double* c, int64_t n, int mirror, double* out) {
  for (int64_t j = 0; j < n; ++j) {
    if (mirror == ORC_PURE) { out[j] = c[j]; continue; }
    float f = (float)c[j];
    if (mirror == ORC_BF16) out[j] = orc_round_bf16(f);
    else if (mirror == ORC_F16) out[j] = orc_round_f16(f);
    else out[j] = (double)f;
  }
}

/* c_hat of B x K x D centroids: m + q(fp32(fp32(c) - m)) with m the batch's
 * mean fp32 centroid (mirror mode, bf16/fp16), fp32(c) for mirror = fp32, c
 * itself in pure mode. */
void orc_chat(const double* c, int64_t B, int64_t K, int64_t D, int mirror, double* out) {
  if (mirror == ORC_PURE || mirror == ORC_F32) {
    orc_quantise(c, B * K * D, mirror, out);
    return;
  }
  for (int64_t b = 0; b < B; ++b)
    for (int64_t d = 0; d < D; ++d) {
      /* the plain mean: fp64 sum over k = 0 .. K-1 in index order */
      double s = 0.0;
      for (int64_t k = 0; k < K; ++k) s += (double)(float)c[(b * K + k) * D + d];
      const float m = (float)(s / (double)K);
      for (int64_t k = 0; k < K; ++k) {
        const int64_t e = (b * K + k) * D + d;
        const float delta = (float)((double)(float)c[e] - (double)m); /* fp32 subtraction */
        double q;
        orc_quantise((const double[]){(double)delta}, 1, mirror, &q);
        out[e] = (double)m + q;
      }
    }
}

/* ---------- assign ---------- */
/* For every point: ids = argmin_k ||x_i - c_hat_k||^2 (lowest k on ties),
 * d1 = that distance, d2 = the second-smallest distance over the other
 * centroids (+inf when K == 1).  J[b] = sum_i d1.  Returns 0 or -1. */
int orc_assign(int64_t B, int64_t N, int64_t K, int64_t D, const void* x, int xdt,
               const double* c, int mirror, int32_t* ids, double* d1, double* d2, double* J) {
  if (B < 1 || N < 0 || K < 1 || D < 1 || !x || !c) return -1;
  double* ch = (double*)malloc(sizeof(double) * (size_t)(B * K * D));
  double* best_all = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
  if (!ch || !best_all) { free(ch); free(best_all); return -1; }
  orc_chat(c, B, K, D, mirror, ch);
  for (int64_t b = 0; b < B; ++b) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
      double xi[4096];
      double* xr = D <= 4096 ? xi : (double*)malloc(sizeof(double) * (size_t)D);
      for (int64_t d = 0; d < D; ++d) xr[d] = orc_read(x, xdt, (b * N + i) * D + d);
      double best = INFINITY, second = INFINITY;
      int64_t arg = 0;
      for (int64_t k = 0; k < K; ++k) {
        const double* ck = ch + (b * K + k) * D;
        double s = 0.0;
        for (int64_t d = 0; d < D; ++d) {
          double diff = xr[d] - ck[d];
          s += diff * diff;
        }
        if (s < best) { second = best; best = s; arg = k; }
        else if (s < second) { second = s; }
      }
      if (ids) ids[b * N + i] = (int32_t)arg;
      if (d1) d1[b * N + i] = best;
      if (d2) d2[b * N + i] = second;
      best_all[i] = best;
      if (xr != xi) free(xr);
    }
    /* the objective is summed in point order, so it does not depend on threads */
    double Jb = 0.0;
    for (int64_t i = 0; i < N; ++i) Jb += best_all[i];
    if (J) J[b] = Jb;
  }
  free(ch);
  free(best_all);
  return 0;
}

/* Objective of a given assignment: J[b] = sum_i ||x_i - c_hat_{ids_i}||^2. */
int orc_inertia(int64_t B, int64_t N, int64_t K, int64_t D, const void* x, int xdt,
                const int32_t* ids, const double* c, int mirror, double* J) {
  if (B < 1 || N < 0 || K < 1 || D < 1 || !x || !c || !ids || !J) return -1;
  double* ch = (double*)malloc(sizeof(double) * (size_t)(B * K * D));
  double* di = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
  if (!ch || !di) { free(ch); free(di); return -1; }
  orc_chat(c, B, K, D, mirror, ch);
  int bad = 0;
  for (int64_t b = 0; b < B; ++b) {
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t i = 0; i < N; ++i) {
      int64_t k = ids[b * N + i];
      di[i] = 0.0;
      if (k < 0 || k >= K) { bad |= 1; continue; }
      const double* ck = ch + (b * K + k) * D;
      double s = 0.0;
      for (int64_t d = 0; d < D; ++d) {
        double diff = orc_read(x, xdt, (b * N + i) * D + d) - ck[d];
        s += diff * diff;
      }
      di[i] = s;
    }
    double Jb = 0.0;
    for (int64_t i = 0; i < N; ++i) Jb += di[i];
    J[b] = Jb;
  }
  free(ch);
  free(di);
  return bad ? -1 : 0;
}

/* ---------- update ---------- */
/* counts[b,k] = #{i : ids = k}; c_new[b,k] = (sum of those x_i, in index
 * order, fp64) / counts, or c_prev[b,k] when counts == 0.
 * shift[b] = sum_k ||c_new - c_prev||^2.  Returns 0, or -1 on an id out of range. */
int orc_update(int64_t B, int64_t N, int64_t K, int64_t D, const void* x, int xdt,
               const int32_t* ids, const double* c_prev, double* c_new, int64_t* counts,
               double* shift) {
  if (B < 1 || N < 0 || K < 1 || D < 1 || !x || !ids || !c_prev || !c_new) return -1;
  int64_t* n = (int64_t*)calloc((size_t)(B * K), sizeof(int64_t));
  double* s = (double*)calloc((size_t)(B * K * D), sizeof(double));
  if (!n || !s) { free(n); free(s); return -1; }
  for (int64_t b = 0; b < B; ++b)
    for (int64_t i = 0; i < N; ++i) {
      int64_t k = ids[b * N + i];
      if (k < 0 || k >= K) { free(n); free(s); return -1; }
      n[b * K + k] += 1;
    }
  /* sums: every element summed over its cluster's points in index order.
   * Clusters are independent: thread t of T owns the clusters with
   * k % T == t and walks the points in index order adding only the rows of
   * its own clusters, so every row of x is read once, by one thread. */
#pragma omp parallel
  {
    const int64_t T = omp_get_num_threads(), t = omp_get_thread_num();
    for (int64_t b = 0; b < B; ++b)
      for (int64_t i = 0; i < N; ++i) {
        const int64_t k = ids[b * N + i];
        if (k % T != t) continue;
        double* sk = s + (b * K + k) * D;
        for (int64_t d = 0; d < D; ++d) sk[d] += orc_read(x, xdt, (b * N + i) * D + d);
      }
  }
  for (int64_t b = 0; b < B; ++b) {
    double sh = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      int64_t nk = n[b * K + k];
      for (int64_t d = 0; d < D; ++d) {
        int64_t e = (b * K + k) * D + d;
        double v = nk > 0 ? s[e] / (double)nk : c_prev[e];
        double diff = v - c_prev[e];
        sh += diff * diff;
        c_new[e] = v;
      }
      if (counts) counts[b * K + k] = nk;
    }
    if (shift) shift[b] = sh;
  }
  free(n);
  free(s);
  return 0;
}

/* ---------- centring ----------
 * k-means is translation invariant, so data with a large common offset can be
 * clustered after subtracting its mean and the centroids shifted back
 * ("Flash-KMeans" GitHub README, section "Centre your data").
 *   mu[b,d] = fp32( (sum over i of x[b,i,d], fp64, index order) / N )
 *   xc[b,i,d] = RNE_dtype( fp32(x[b,i,d]) - mu[b,d] ), the subtraction one IEEE
 *               fp32 operation; xc is written in the storage form of the dtype
 *               (fp32 values, fp16 values, bf16 bit patterns).
 * mu_in, when non-null, replaces the computed mean (to check the subtraction
 * for a given mean); mu_out (optional) receives the mean used. */
static void orc_store(void* out, int dt, int64_t idx, float v) {
  if (dt == ORC_F32) {
    ((float*)out)[idx] = v;
  } else if (dt == ORC_F16) {
    _Float16 h = (_Float16)v;
    memcpy((uint16_t*)out + idx, &h, 2);
  } else {
    const float r = (float)orc_round_bf16(v);
    uint32_t u;
    memcpy(&u, &r, 4);
    ((uint16_t*)out)[idx] = (uint16_t)(u >> 16);
  }
}

int orc_centre(int64_t B, int64_t N, int64_t D, const void* x, int xdt, const float* mu_in,
               float* mu_out, void* xc_out) {
  if (B < 1 || N < 1 || D < 1 || !x || !xc_out) return -1;
  float* mu = (float*)malloc(sizeof(float) * (size_t)(B * D));
  if (!mu) return -1;
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t b = 0; b < B; ++b)
    for (int64_t d = 0; d < D; ++d) {
      if (mu_in) {
        mu[b * D + d] = mu_in[b * D + d];
        continue;
      }
      double s = 0.0;
      for (int64_t i = 0; i < N; ++i) s += orc_read(x, xdt, (b * N + i) * D + d);
      mu[b * D + d] = (float)(s / (double)N);
    }
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t b = 0; b < B; ++b)
    for (int64_t i = 0; i < N; ++i)
      for (int64_t d = 0; d < D; ++d) {
        const int64_t e = (b * N + i) * D + d;
        const float v = (float)orc_read(x, xdt, e) - mu[b * D + d];
        orc_store(xc_out, xdt, e, v);
      }
  if (mu_out) memcpy(mu_out, mu, sizeof(float) * (size_t)(B * D));
  free(mu);
  return 0;
}

/* ---------- Lloyd loop ---------- */
/* centers starts as c0 and ends as the centroids after the last update.
 * J_hist / shift_hist (optional, [max_iters * B]) record every iteration. */
int orc_lloyd(int64_t B, int64_t N, int64_t K, int64_t D, const void* x, int xdt,
              const double* c0, int max_iters, double tol, int mirror, int32_t* ids,
              double* centers, int64_t* counts, double* inertia, int* n_iter, double* J_hist,
              double* shift_hist) {
  if (B < 1 || N < 0 || K < 1 || D < 1 || max_iters < 1 || !x || !c0 || !ids || !centers)
    return -1;
  int64_t nc = B * K * D;
  double* cur = (double*)malloc(sizeof(double) * (size_t)nc);
  double* nxt = (double*)malloc(sizeof(double) * (size_t)nc);
  double* J = (double*)malloc(sizeof(double) * (size_t)B);
  double* sh = (double*)malloc(sizeof(double) * (size_t)B);
  if (!cur || !nxt || !J || !sh) { free(cur); free(nxt); free(J); free(sh); return -1; }
  memcpy(cur, c0, sizeof(double) * (size_t)nc);
  int rc = 0, t = 0;
  for (t = 0; t < max_iters; ++t) {
    rc = orc_assign(B, N, K, D, x, xdt, cur, mirror, ids, NULL, NULL, J);
    if (rc) break;
    rc = orc_update(B, N, K, D, x, xdt, ids, cur, nxt, counts, sh);
    if (rc) break;
    double* tmp = cur; cur = nxt; nxt = tmp;
    double mx = 0.0;
    for (int64_t b = 0; b < B; ++b) {
      if (J_hist) J_hist[(int64_t)t * B + b] = J[b];
      if (shift_hist) shift_hist[(int64_t)t * B + b] = sh[b];
      if (sh[b] > mx) mx = sh[b];
    }
    if (mx < tol) { t += 1; break; }
  }
  if (!rc) {
    memcpy(centers, cur, sizeof(double) * (size_t)nc);
    if (inertia) memcpy(inertia, J, sizeof(double) * (size_t)B);
    if (n_iter) *n_iter = t;
  }
  free(cur); free(nxt); free(J); free(sh);
  return rc;
}

/* ---------- dot-product and cosine k-means ----------
 * The README lists cosine and dot-product k-means beside the Euclidean one
 * ("Flash-KMeans" GitHub README, section "Usage", the CuTe backend note) but
 * defines neither; the plainest readings are taken:
 *   dot      a_i = argmax_k x_i . c_k; c_k = mean of its points (as above);
 *            objective J = sum_i x_i . c_{a_i}
 *   cosine   a_i = argmax_k x_i . u_k with u_k = c_k / ||c_k|| (the point's
 *            own norm does not move its argmax); c_k = s_k / ||s_k||, the
 *            direction of its points' sum (spherical k-means; for unit-norm
 *            points the sum of directions); objective J = sum_i x_i . u_{a_i}
 * Ties go to the lowest index, an empty cluster (or one whose sum is the zero
 * vector) keeps its previous centroid, and shift is as above.  In mirror mode
 * the assignment measures against c_hat = m + q(fp32(v - m)) of v = c (dot)
 * or v = u (cosine), u = fp32(c_d / ||c||) with ||c|| in fp64 and m the mean
 * of the v rows, as orc_chat forms it; the objective uses the plain c or u. */
enum { ORC_EUCLID = 0, ORC_DOT = 1, ORC_COSINE = 2 };

/* u = fp32(c / ||c||) row by row (a zero row stays zero) */
static void orc_unit_rows(const double* c, int64_t rows, int64_t D, double* u) {
  for (int64_t r = 0; r < rows; ++r) {
    double nn = 0.0;
    for (int64_t d = 0; d < D; ++d) {
      const double v = (double)(float)c[r * D + d];
      nn += v * v;
    }
    const double n = sqrt(nn);
    for (int64_t d = 0; d < D; ++d)
      u[r * D + d] = n > 0.0 ? (double)(float)((double)(float)c[r * D + d] / n) : 0.0;
  }
}

/* the vectors a metric scores against, before any mirroring: c or u */
static int orc_metric_rows(const double* c, int64_t rows, int64_t D, int metric, double* out) {
  if (metric == ORC_COSINE) orc_unit_rows(c, rows, D, out);
  else if (metric == ORC_DOT) memcpy(out, c, sizeof(double) * (size_t)(rows * D));
  else return -1;
  return 0;
}

/* ids = argmax_k x_i . c_hat_k (lowest k on ties), s1 the best score, s2 the
 * second best over the other centroids (-inf when K == 1).  Returns 0 or -1. */
int orc_assign_sim(int64_t B, int64_t N, int64_t K, int64_t D, const void* x, int xdt,
                   const double* c, int metric, int mirror, int32_t* ids, double* s1,
                   double* s2) {
  if (B < 1 || N < 0 || K < 1 || D < 1 || !x || !c) return -1;
  double* v = (double*)malloc(sizeof(double) * (size_t)(B * K * D));
  double* ch = (double*)malloc(sizeof(double) * (size_t)(B * K * D));
  if (!v || !ch || orc_metric_rows(c, B * K, D, metric, v)) { free(v); free(ch); return -1; }
  orc_chat(v, B, K, D, mirror, ch);
  for (int64_t b = 0; b < B; ++b) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
      double best = -INFINITY, second = -INFINITY;
      int64_t arg = 0;
      for (int64_t k = 0; k < K; ++k) {
        const double* ck = ch + (b * K + k) * D;
        double sc = 0.0;
        for (int64_t d = 0; d < D; ++d) sc += orc_read(x, xdt, (b * N + i) * D + d) * ck[d];
        if (sc > best) { second = best; best = sc; arg = k; }
        else if (sc > second) { second = sc; }
      }
      if (ids) ids[b * N + i] = (int32_t)arg;
      if (s1) s1[b * N + i] = best;
      if (s2) s2[b * N + i] = second;
    }
  }
  free(v);
  free(ch);
  return 0;
}

/* J[b] = sum_i x_i . v_{ids_i} (point order), v = c (dot) or u (cosine). */
int orc_similarity(int64_t B, int64_t N, int64_t K, int64_t D, const void* x, int xdt,
                   const int32_t* ids, const double* c, int metric, double* J) {
  if (B < 1 || N < 0 || K < 1 || D < 1 || !x || !c || !ids || !J) return -1;
  double* v = (double*)malloc(sizeof(double) * (size_t)(B * K * D));
  if (!v || orc_metric_rows(c, B * K, D, metric, v)) { free(v); return -1; }
  int bad = 0;
  for (int64_t b = 0; b < B; ++b) {
    double Jb = 0.0;
    for (int64_t i = 0; i < N; ++i) {
      const int64_t k = ids[b * N + i];
      if (k < 0 || k >= K) { bad = 1; continue; }
      for (int64_t d = 0; d < D; ++d)
        Jb += orc_read(x, xdt, (b * N + i) * D + d) * v[(b * K + k) * D + d];
    }
    J[b] = Jb;
  }
  free(v);
  return bad ? -1 : 0;
}

/* The update of a metric: the mean for dot (orc_update); for cosine the mean
 * scaled to unit length, s_k / ||s_k||, unless the cluster is empty or its sum
 * is zero (then the previous centroid stays).  shift as in orc_update. */
int orc_update_sim(int64_t B, int64_t N, int64_t K, int64_t D, const void* x, int xdt,
                   const int32_t* ids, const double* c_prev, int metric, double* c_new,
                   int64_t* counts, double* shift) {
  if (metric != ORC_DOT && metric != ORC_COSINE) return -1;
  int64_t* n = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B * K));
  if (!n) return -1;
  int rc = orc_update(B, N, K, D, x, xdt, ids, c_prev, c_new, n, NULL);
  if (!rc) {
    for (int64_t b = 0; b < B; ++b) {
      double sh = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double* ck = c_new + (b * K + k) * D;
        if (metric == ORC_COSINE && n[b * K + k] > 0) {
          double nn = 0.0;
          for (int64_t d = 0; d < D; ++d) nn += ck[d] * ck[d];
          if (nn > 0.0) {
            const double r = sqrt(nn);
            for (int64_t d = 0; d < D; ++d) ck[d] /= r;
          } else {
            memcpy(ck, c_prev + (b * K + k) * D, sizeof(double) * (size_t)D);
          }
        }
        for (int64_t d = 0; d < D; ++d) {
          const double df = ck[d] - c_prev[(b * K + k) * D + d];
          sh += df * df;
        }
        if (counts) counts[b * K + k] = n[b * K + k];
      }
      if (shift) shift[b] = sh;
    }
  }
  free(n);
  return rc;
}

/* The Lloyd loop of a metric, as orc_lloyd: inertia is the objective J of the
 * last assignment against the centroids it used; J_hist / shift_hist record
 * every iteration. */
int orc_lloyd_sim(int64_t B, int64_t N, int64_t K, int64_t D, const void* x, int xdt,
                  const double* c0, int max_iters, double tol, int metric, int mirror,
                  int32_t* ids, double* centers, int64_t* counts, double* inertia, int* n_iter,
                  double* J_hist, double* shift_hist) {
  if (B < 1 || N < 0 || K < 1 || D < 1 || max_iters < 1 || !x || !c0 || !ids || !centers)
    return -1;
  const int64_t nc = B * K * D;
  double* cur = (double*)malloc(sizeof(double) * (size_t)nc);
  double* nxt = (double*)malloc(sizeof(double) * (size_t)nc);
  double* J = (double*)malloc(sizeof(double) * (size_t)B);
  double* sh = (double*)malloc(sizeof(double) * (size_t)B);
  if (!cur || !nxt || !J || !sh) { free(cur); free(nxt); free(J); free(sh); return -1; }
  memcpy(cur, c0, sizeof(double) * (size_t)nc);
  int rc = 0, t = 0;
  for (t = 0; t < max_iters; ++t) {
    rc = orc_assign_sim(B, N, K, D, x, xdt, cur, metric, mirror, ids, NULL, NULL);
    if (!rc) rc = orc_similarity(B, N, K, D, x, xdt, ids, cur, metric, J);
    if (!rc) rc = orc_update_sim(B, N, K, D, x, xdt, ids, cur, metric, nxt, counts, sh);
    if (rc) break;
    double* tmp = cur; cur = nxt; nxt = tmp;
    double mx = 0.0;
    for (int64_t b = 0; b < B; ++b) {
      if (J_hist) J_hist[(int64_t)t * B + b] = J[b];
      if (shift_hist) shift_hist[(int64_t)t * B + b] = sh[b];
      if (sh[b] > mx) mx = sh[b];
    }
    if (mx < tol) { t += 1; break; }
  }
  if (!rc) {
    memcpy(centers, cur, sizeof(double) * (size_t)nc);
    if (inertia) memcpy(inertia, J, sizeof(double) * (size_t)B);
    if (n_iter) *n_iter = t;
  }
  free(cur); free(nxt); free(J); free(sh);
  return rc;
}

/* ---------- stable argsort of small non-negative integer keys ---------- */
/* idx[r] = the index of the r-th smallest key; equal keys keep index order. */
int orc_argsort_stable(const int64_t* keys, int64_t n, int64_t n_keys, int64_t* idx) {
  if (n < 0 || n_keys < 1 || (n > 0 && (!keys || !idx))) return -1;
  int64_t* start = (int64_t*)calloc((size_t)n_keys + 1, sizeof(int64_t));
  if (!start) return -1;
  for (int64_t i = 0; i < n; ++i) {
    if (keys[i] < 0 || keys[i] >= n_keys) { free(start); return -1; }
    start[keys[i] + 1] += 1;
  }
  for (int64_t k = 0; k < n_keys; ++k) start[k + 1] += start[k];
  for (int64_t i = 0; i < n; ++i) idx[start[keys[i]]++] = i;
  free(start);
  return 0;
}
