/*
 * kda_oracle.c -- fp64 CPU oracle for the bounded-decay gated delta rule
 * (the Kimi Delta Attention scan with a lower-bounded per-channel decay).
 *
 * TEST INFRASTRUCTURE. This file is the parity oracle: only the test suite,
 * the smoke check and the benchmark's CPU-baseline leg load it. The CUDA
 * library never links it, includes it or calls it, and it shares no header,
 * helper or constant with the CUDA path.
 *
 * What it computes, and where the pages define it:
 *
 *   Gate ("Kimi K3: Bounded Decay and Delta Memory", Formula and conventions,
 *   eq. 5; "KDA cheat sheet", Lower-bounded decay):
 *       g = g_min * sigmoid(exp(A_h) * z),   alpha = exp(g),   g_min < 0.
 *
 *   Scan ("Kimi K3: Bounded Decay and Delta Memory", eq. 1; "KDARecurrent",
 *   The state recurrence in source order). Per sequence and head, token by
 *   token, with the state S stored key-by-value (K rows, V columns):
 *       fade:    Sbar = Diag(alpha_t) S            (alpha scales key rows)
 *       correct: delta = v_t - Sbar^T k_t
 *                S = Sbar + beta_t k_t delta^T
 *       read:    o_t = S^T q_t                     (after the write)
 *   No query scaling inside the scan (the PaperLeet contract states that the
 *   scan performs no query scaling or key normalisation).
 *
 * Arithmetic is plain double precision in the order written above; there is
 * no blocking, chunking or reordering. Independent (sequence, head) pairs run
 * on separate OpenMP threads; each pair's arithmetic is sequential.
 *
 * Layouts (all contiguous, row-major, fp64):
 *   q, k, alpha : [B, T, H, K]      v, o : [B, T, H, V]      beta : [B, T, H]
 *   s0, s_final : [N, H, K, V]  with N = B, or N = n_seq when cu_seqlens is
 *   given (then B must be 1 and sequence n spans tokens
 *   cu_seqlens[n] .. cu_seqlens[n+1]-1 of the packed time axis).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Logistic function, evaluated without overflow for either sign. */
static double oracle_sigmoid(double x) {
  if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
  double e = exp(x);
  return e / (1.0 + e);
}

/* Bounded decay gate, elementwise over [B,T,H,K]. Writes alpha and, when
 * g_out is not NULL, the log-decay g as well. */
void kda_oracle_bounded_decay(const double* z, const double* A_log, double g_min,
                              int64_t B, int64_t T, int64_t H, int64_t K,
                              double* alpha_out, double* g_out) {
  for (int64_t b = 0; b < B; ++b)
    for (int64_t t = 0; t < T; ++t)
      for (int64_t h = 0; h < H; ++h) {
        double scale = exp(A_log[h]);
        for (int64_t c = 0; c < K; ++c) {
          int64_t idx = ((b * T + t) * H + h) * K + c;
          double g = g_min * oracle_sigmoid(scale * z[idx]);
          if (g_out) g_out[idx] = g;
          alpha_out[idx] = exp(g);
        }
      }
}

/* Returns 0 on success, -1 on an invalid argument. */
int kda_oracle_scan(const double* q, const double* k, const double* v,
                    const double* alpha, const double* beta, const double* s0,
                    const int64_t* cu_seqlens, int64_t n_seq,
                    int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                    double* o, double* s_final, int n_threads) {
  if (B < 0 || T < 0 || H <= 0 || K <= 0 || V <= 0) return -1;
  int64_t N = B;
  if (cu_seqlens) {
    if (B != 1 || n_seq < 0) return -1;
    N = n_seq;
    if (cu_seqlens[0] != 0 || cu_seqlens[N] != T) return -1;
    for (int64_t n = 0; n < N; ++n)
      if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
  }
  int64_t pairs = N * H;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
  int failed = 0;
#pragma omp parallel
  {
    double* S = (double*)malloc(sizeof(double) * (size_t)(K * V));
    double* delta = (double*)malloc(sizeof(double) * (size_t)V);
    if (!S || !delta) {
#pragma omp atomic write
      failed = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t p = 0; p < pairs; ++p) {
      if (!S || !delta) continue;
      int64_t n = p / H, h = p % H;
      /* Token range of this sequence on the [B,T] grid: (batch row, t0, t1). */
      int64_t brow = cu_seqlens ? 0 : n;
      int64_t t0 = cu_seqlens ? cu_seqlens[n] : 0;
      int64_t t1 = cu_seqlens ? cu_seqlens[n + 1] : T;
      if (s0) memcpy(S, s0 + (n * H + h) * K * V, sizeof(double) * (size_t)(K * V));
      else memset(S, 0, sizeof(double) * (size_t)(K * V));
      for (int64_t t = t0; t < t1; ++t) {
        int64_t row = brow * T + t;
        const double* kt = k + (row * H + h) * K;
        const double* qt = q + (row * H + h) * K;
        const double* at = alpha + (row * H + h) * K;
        const double* vt = v + (row * H + h) * V;
        double bt = beta[row * H + h];
        /* fade: scale key row i by alpha_t[i] */
        for (int64_t i = 0; i < K; ++i)
          for (int64_t j = 0; j < V; ++j) S[i * V + j] *= at[i];
        /* correct: delta = v_t - Sbar^T k_t */
        for (int64_t j = 0; j < V; ++j) delta[j] = 0.0;
        for (int64_t i = 0; i < K; ++i)
          for (int64_t j = 0; j < V; ++j) delta[j] += S[i * V + j] * kt[i];
        for (int64_t j = 0; j < V; ++j) delta[j] = vt[j] - delta[j];
        /* S = Sbar + beta_t k_t delta^T */
        for (int64_t i = 0; i < K; ++i)
          for (int64_t j = 0; j < V; ++j) S[i * V + j] += bt * kt[i] * delta[j];
        /* read after the write: o_t = S^T q_t */
        double* ot = o + (row * H + h) * V;
        for (int64_t j = 0; j < V; ++j) ot[j] = 0.0;
        for (int64_t i = 0; i < K; ++i)
          for (int64_t j = 0; j < V; ++j) ot[j] += S[i * V + j] * qt[i];
      }
      if (s_final) memcpy(s_final + (n * H + h) * K * V, S, sizeof(double) * (size_t)(K * V));
    }
    free(S);
    free(delta);
  }
  return failed ? -1 : 0;
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
int kda_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
