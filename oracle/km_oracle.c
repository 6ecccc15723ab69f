/*
 * km_oracle.c -- plain float64 Lloyd K-Means on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this library.  It shares no code, header, table
 * or helper with the CUDA library; it is written to be checked by eye.
 *
 * What it follows: "Flash-KMeans: Fast and Memory-Efficient Exact K-Means",
 * §2 (Methodology) states that the method keeps the mathematics of standard
 * Lloyd K-Means unchanged and introduces no approximation, and §3 (Key
 * Contributions, "数学精确性") repeats that the result is exact.  So this file
 * is the textbook definition of one Lloyd iteration:
 *
 *   assignment  a_i = argmin_k ||x_i - c_k||^2     (lowest k on exact ties)
 *   update      c_k = mean{ x_i : a_i = k }        (keep c_k if no member)
 *   objective   J   = sum_i min_k ||x_i - c_k||^2  (under the centroids used
 *                                                   for that assignment)
 *
 * Readings where the pages are silent (tie rule, empty clusters, objective
 * timing) are the plainest ones and are listed in the design notes.
 * Distances use the direct form sum_j (x_ij - c_kj)^2, never the expanded
 * ||x||^2 - 2 x.c + ||c||^2 form the GPU uses.  OpenMP splits only loops
 * over points (the assignment, and the objective of a given assignment in
 * fixed blocks); every per-cluster sum runs in point order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Number of threads the OpenMP loops use (1 without OpenMP). */
int kmo_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void kmo_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Squared Euclidean distance, direct form. */
static double sqdist(const double* x, const double* c, int D) {
  double s = 0.0;
  for (int j = 0; j < D; ++j) {
    double t = x[j] - c[j];
    s += t * t;
  }
  return s;
}

/*
 * Assignment step (Flash-KMeans §2.1 FlashAssign computes exactly this
 * argmin; the oracle simply evaluates every distance).
 *   X: N x D row-major, C: K x D row-major.
 *   idx[i]  = smallest k with ||x_i - c_k||^2 minimal.
 *   d1[i]   = that minimal distance.
 *   d2[i]   = smallest distance over k != idx[i] (+inf when K == 1); may be
 *             NULL.  Used for the near-tie rule of the parity tests.
 */
void kmo_assign(const double* X, const double* C, int64_t N, int D, int K,
                int32_t* idx, double* d1, double* d2) {
  int64_t i;
#pragma omp parallel for schedule(static)
  for (i = 0; i < N; ++i) {
    const double* x = X + i * (int64_t)D;
    double best = INFINITY, second = INFINITY;
    int32_t bk = 0;
    for (int k = 0; k < K; ++k) {
      double d = sqdist(x, C + (int64_t)k * D, D);
      if (d < best) {
        second = best;
        best = d;
        bk = k;
      } else if (d < second) {
        second = d;
      }
    }
    idx[i] = bk;
    if (d1) d1[i] = best;
    if (d2) d2[i] = second;
  }
}

/*
 * Update step: the mean of each cluster's members (Flash-KMeans §2.2
 * Sort-Inverse Update reorganises how these sums are formed; the values are
 * the plain means).  Sums run sequentially in point order.
 *   C:      in = previous centroids, out = new centroids (K x D).
 *   counts: out, members per cluster.  A cluster with no member keeps its
 *           previous centroid.
 */
void kmo_update(const double* X, const int32_t* idx, int64_t N, int D, int K,
                double* C, int64_t* counts) {
  double* sums = (double*)calloc((size_t)K * (size_t)D, sizeof(double));
  for (int k = 0; k < K; ++k) counts[k] = 0;
  for (int64_t i = 0; i < N; ++i) {
    int32_t k = idx[i];
    const double* x = X + i * (int64_t)D;
    double* s = sums + (int64_t)k * D;
    for (int j = 0; j < D; ++j) s[j] += x[j];
    counts[k] += 1;
  }
  for (int k = 0; k < K; ++k) {
    if (counts[k] == 0) continue;
    for (int j = 0; j < D; ++j)
      C[(int64_t)k * D + j] = sums[(int64_t)k * D + j] / (double)counts[k];
  }
  free(sums);
}

/* Objective: sequential float64 sum of the per-point minimal distances. */
double kmo_objective(const double* d1, int64_t N) {
  double s = 0.0;
  for (int64_t i = 0; i < N; ++i) s += d1[i];
  return s;
}

/*
 * Objective of a given assignment, for point sets too large to convert to
 * float64 at once: J = sum_i ||x_i - c_{idx[i]}||^2 (direct form), with X
 * given as raw bfloat16 bit patterns.  A bfloat16 value is the upper 16 bits
 * of a float32, so it widens exactly: place the bits in the top half of a
 * 32-bit word, read it as a float, widen to double.  Points are summed in
 * blocks of 4096, each block sequentially, and the block sums sequentially
 * in block order (the order does not depend on the thread count).
 *   Xbits: N x D uint16, C: K x D float64, idx: N entries in [0, K).
 */
static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

double kmo_objective_assigned_bf16(const uint16_t* Xbits, const double* C, const int32_t* idx,
                                   int64_t N, int D) {
  const int64_t blk = 4096;
  const int64_t nb = (N + blk - 1) / blk;
  double* part = (double*)calloc((size_t)(nb > 0 ? nb : 1), sizeof(double));
  int64_t b;
#pragma omp parallel for schedule(static)
  for (b = 0; b < nb; ++b) {
    double s = 0.0;
    const int64_t i1 = (b + 1) * blk < N ? (b + 1) * blk : N;
    for (int64_t i = b * blk; i < i1; ++i) {
      const uint16_t* x = Xbits + i * (int64_t)D;
      const double* c = C + (int64_t)idx[i] * D;
      for (int j = 0; j < D; ++j) {
        double t = bf16_bits_to_double(x[j]) - c[j];
        s += t * t;
      }
    }
    part[b] = s;
  }
  double J = 0.0;
  for (b = 0; b < nb; ++b) J += part[b];
  free(part);
  return J;
}

/*
 * Round a double to the nearest bfloat16 value (8 exponent bits, 7 stored
 * mantissa bits), ties to even, written from the format's definition: a
 * normal bf16 number is m * 2^(e-7) with 128 <= |m| < 256 an integer.
 */
double kmo_round_bf16_one(double v) {
  if (!isfinite(v) || v == 0.0) return v;
  int e;
  double m = frexp(v, &e); /* v = m * 2^e, 0.5 <= |m| < 1 */
  int scale_exp = 8;       /* |m| * 2^8 in [128, 256) */
  /* Below the smallest normal (2^-126) the spacing stays 2^-133. */
  if (e - 1 < -126) scale_exp = 8 - (-126 - (e - 1));
  double t = ldexp(m, scale_exp);
  double r = floor(t);
  double frac = t - r;
  if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
  double out = ldexp(r, e - scale_exp);
  /* Largest finite bf16 is (2 - 2^-7) * 2^127. */
  if (fabs(out) > ldexp(255.0, 120)) out = v > 0 ? INFINITY : -INFINITY;
  return out;
}

void kmo_round_bf16(const double* in, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = kmo_round_bf16_one(in[i]);
}

void kmo_round_f32(const double* in, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = (double)(float)in[i];
}

/*
 * Stable argsort of the assignment vector by counting (the "explicit inverse
 * map" of Flash-KMeans §2.2: indices ordered by cluster id, ties in point
 * order).  perm: N entries.  start: K+1 entries, start[k] = first position of
 * cluster k in perm, start[K] = N.
 */
void kmo_argsort(const int32_t* idx, int64_t N, int K, int32_t* perm, int64_t* start) {
  int64_t* cursor = (int64_t*)calloc((size_t)K + 1, sizeof(int64_t));
  for (int64_t i = 0; i < N; ++i) cursor[idx[i] + 1] += 1;
  for (int k = 0; k < K; ++k) cursor[k + 1] += cursor[k];
  for (int k = 0; k <= K; ++k) start[k] = cursor[k];
  for (int64_t i = 0; i < N; ++i) perm[cursor[idx[i]]++] = (int32_t)i;
  free(cursor);
}

/*
 * T Lloyd iterations from C0 (Flash-KMeans §2: the iteration is standard
 * Lloyd).  Iteration t assigns under C_{t-1}, records J_t, then updates.
 *   mirror: 0 = the centroids used for assignment are the float64 means;
 *           1 = they are rounded to bfloat16 (as a bf16 device pipeline
 *               stores its operand copy); 2 = rounded to float32.
 *   C: in = C0 (K x D), out = C_T (float64 master values).
 *   idx: out, assignment of the last iteration.  counts: out, last counts.
 *   J: out, T objective values.
 */
void kmo_fit(const double* X, int64_t N, int D, int K, int T, int mirror,
             double* C, int32_t* idx, int64_t* counts, double* J) {
  size_t kd = (size_t)K * (size_t)D;
  double* Cuse = (double*)malloc(kd * sizeof(double));
  double* d1 = (double*)malloc((size_t)N * sizeof(double));
  for (int t = 0; t < T; ++t) {
    if (mirror == 1)
      kmo_round_bf16(C, Cuse, (int64_t)kd);
    else if (mirror == 2)
      kmo_round_f32(C, Cuse, (int64_t)kd);
    else
      memcpy(Cuse, C, kd * sizeof(double));
    kmo_assign(X, Cuse, N, D, K, idx, d1, NULL);
    J[t] = kmo_objective(d1, N);
    kmo_update(X, idx, N, D, K, C, counts);
  }
  free(d1);
  free(Cuse);
}
