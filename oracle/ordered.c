/*
 * ordered.c -- the oracle's fixed-order float32 (and sequential float64) view
 * of the batch-invariant operations. TEST INFRASTRUCTURE ONLY: nothing on the
 * product path links or loads this file. Plain C99, no CUDA, no shared code
 * with the GPU library.
 *
 * Every reduction here is written out as one left-to-right loop, so the order
 * of additions is visible in the source:
 *   - sums: acc = acc + v[i], i = 0, 1, ..., n-1
 *   - dot products: acc = fmaf(a[k], b[k], acc), k = 0, 1, ..., K-1
 *
 * "Defeating Nondeterminism in LLM Inference":
 *   section "The original sin: floating-point non-associativity" -- sums
 *     in different orders give different results;
 *   section "Batch-invariant RMSNorm" -- x * rsqrt(mean(x^2)) * weight;
 *   section "Batch-invariant matmul" -- pointwise products reduced over K;
 *   section "Batch-invariant attention" -- causal softmax attention.
 *
 * Build: gcc -O2 -std=c99 -fPIC -shared -ffp-contract=off -fopenmp
 * (-ffp-contract=off: the compiler may not fuse a*b+c on its own, so only the
 * explicit fmaf calls fuse).
 */
#include <math.h>
#include <stdint.h>

/* ---- sums ---------------------------------------------------------------- */

double seq_sum_f64(const double* v, int64_t n) {
  double acc = 0.0;
  for (int64_t i = 0; i < n; ++i) acc = acc + v[i];
  return acc;
}

/* out[r] = seq_sum_f64(v + r*n, n) for each row r. */
void seq_sum_rows_f64(const double* v, int64_t rows, int64_t n, double* out) {
  for (int64_t r = 0; r < rows; ++r) out[r] = seq_sum_f64(v + r * n, n);
}

/* The summation CPython's built-in sum() performs (version 3.12 and later) on
 * a list that mixes Python ints and floats, as in the shuffled-sum experiment
 * of "Defeating Nondeterminism in LLM Inference" (section "The original sin:
 * floating-point non-associativity"), whose list holds the ints 1 and -1 next
 * to float powers of ten:
 *   - leading int terms are added exactly (as integers);
 *   - the first float term is added to that integer sum in plain float64;
 *   - later float terms use Neumaier's compensated addition (Neumaier,
 *     "Rundungsfehleranalyse einiger Verfahren zur Summation endlicher
 *     Summen", ZAMM 1974): s = s + x, and the rounding error of that addition,
 *     (s_old - s) + x or (x - s) + s_old depending on which operand is larger
 *     in magnitude, accumulates in c;
 *   - later int terms are added to s in plain float64 (c unchanged);
 *   - the result is s + c (c added only when it is non-zero and finite).
 * is_int[i] != 0 marks v[i] as an int term (its value must be integral). */
double mixed_sum_f64(const double* v, const int8_t* is_int, int64_t n) {
  int64_t i = 0;
  double isum = 0.0; /* exact for the small integers this is used with */
  while (i < n && is_int[i]) isum = isum + v[i++];
  if (i == n) return isum;
  double s = isum + v[i++], c = 0.0;
  for (; i < n; ++i) {
    if (is_int[i]) {
      s = s + v[i];
      continue;
    }
    double t = s + v[i];
    if (fabs(s) >= fabs(v[i]))
      c = c + ((s - t) + v[i]);
    else
      c = c + ((v[i] - t) + s);
    s = t;
  }
  if (c != 0.0 && isfinite(c)) s = s + c;
  return s;
}

void mixed_sum_rows_f64(const double* v, const int8_t* is_int, int64_t rows,
                        int64_t n, double* out) {
  for (int64_t r = 0; r < rows; ++r)
    out[r] = mixed_sum_f64(v + r * n, is_int + r * n, n);
}

float seq_sum_f32(const float* v, int64_t n) {
  float acc = 0.0f;
  for (int64_t i = 0; i < n; ++i) acc = acc + v[i];
  return acc;
}

/* n values cut into consecutive groups of `group`; each group summed left to
 * right, then the group sums summed left to right. group == n is seq_sum_f32. */
float grouped_sum_f32(const float* v, int64_t n, int64_t group) {
  float total = 0.0f;
  for (int64_t g0 = 0; g0 < n; g0 += group) {
    float part = 0.0f;
    int64_t g1 = g0 + group < n ? g0 + group : n;
    for (int64_t i = g0; i < g1; ++i) part = part + v[i];
    total = total + part;
  }
  return total;
}

/* ---- RMSNorm --------------------------------------------------------------- */

/* y[i, j] = (x[i, j] * r_i) * gamma[j], r_i = 1 / sqrtf(ss_i / D + eps),
 * ss_i = sum_j x_ij^2 accumulated left to right with fmaf, all float32. */
void rmsnorm_f32(const float* x, const float* gamma, float* y, int64_t M,
                 int64_t D, float eps) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < M; ++i) {
    const float* xi = x + i * D;
    float ss = 0.0f;
    for (int64_t j = 0; j < D; ++j) ss = fmaf(xi[j], xi[j], ss);
    float r = 1.0f / sqrtf(ss / (float)D + eps);
    for (int64_t j = 0; j < D; ++j) y[i * D + j] = (xi[j] * r) * gamma[j];
  }
}

/* ---- GEMM ------------------------------------------------------------------ */

/* C[m, n] = sum_k A[m, k] W[n, k], fmaf left to right over k, float32. */
void gemm_f32(const float* A, const float* W, float* C, int64_t M, int64_t N,
              int64_t K) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      const float* a = A + m * K;
      const float* w = W + n * K;
      float acc = 0.0f;
      for (int64_t k = 0; k < K; ++k) acc = fmaf(a[k], w[k], acc);
      C[m * N + n] = acc;
    }
  }
}

/* ---- attention ------------------------------------------------------------- */

/* Causal grouped-query attention for the queries of one sequence, float32,
 * two passes per (query, head): scores and their max, then exp / sum / weighted
 * values, then one division.
 *   q [n, Hq, d], k and v [L, Hkv, d], q_pos [n], out [n, Hq, d].
 * Query i attends keys 0..q_pos[i]; head h reads kv head h / (Hq / Hkv).
 * scratch: at least L floats per thread (caller-owned, [threads, L]). */
void attention_f32(const float* q, const float* k, const float* v,
                   const int32_t* q_pos, int64_t n, int64_t L, int64_t Hq,
                   int64_t Hkv, int64_t d, float scale, float* out,
                   float* scratch, int64_t scratch_rows) {
  int64_t group = Hq / Hkv;
#pragma omp parallel for schedule(static) num_threads(scratch_rows)
  for (int64_t ih = 0; ih < n * Hq; ++ih) {
    int tid = 0;
#ifdef _OPENMP
    extern int omp_get_thread_num(void);
    tid = omp_get_thread_num();
#endif
    float* s = scratch + (int64_t)tid * L;
    int64_t i = ih / Hq, h = ih % Hq, g = h / group;
    int64_t last = q_pos[i];
    const float* qi = q + (i * Hq + h) * d;
    float m = -INFINITY;
    for (int64_t j = 0; j <= last; ++j) {
      const float* kj = k + (j * Hkv + g) * d;
      float acc = 0.0f;
      for (int64_t e = 0; e < d; ++e) acc = fmaf(qi[e], kj[e], acc);
      s[j] = acc * scale;
      if (s[j] > m) m = s[j];
    }
    float l = 0.0f;
    float* o = out + (i * Hq + h) * d;
    for (int64_t e = 0; e < d; ++e) o[e] = 0.0f;
    for (int64_t j = 0; j <= last; ++j) {
      float p = expf(s[j] - m);
      l = l + p;
      const float* vj = v + (j * Hkv + g) * d;
      for (int64_t e = 0; e < d; ++e) o[e] = fmaf(p, vj[e], o[e]);
    }
    for (int64_t e = 0; e < d; ++e) o[e] = o[e] / l;
  }
}

/* ---- threads ------------------------------------------------------------- */

/* OpenMP threads the parallel loops above use (timing only: every output
 * element is computed by one thread in the order written, so the results do
 * not depend on it). */
#ifdef _OPENMP
extern void omp_set_num_threads(int);
extern int omp_get_max_threads(void);
#endif
void ordered_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int ordered_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

int ordered_abi_version(void) { return 1; }
