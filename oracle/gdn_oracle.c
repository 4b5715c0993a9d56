/*
 * gdn_oracle.c -- fp64 CPU oracle for the Gated DeltaNet recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path (the CUDA library
 * and its Python binding) may link, load or call this file; only the test
 * suite, the smoke check and the benchmark's CPU-baseline leg do.  It shares
 * no code, headers or constants with the CUDA implementation.
 *
 * What it computes (plain definition, no chunking, no blocking):
 *   "NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI Training
 *   Runs", section "Solving the linear-attention headache": Gated DeltaNet
 *   has a recurrent form and a chunkwise-parallel form that are
 *   mathematically identical; CPR evaluates the recurrence.  The recurrence
 *   itself, in the notation used throughout this repository, is
 *
 *       S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *       o_t = scale * S_t q_t
 *
 *   with S a d_v x d_k matrix (row index = value channel, column index =
 *   key channel), alpha_t = exp(g_t), one state per (sequence, head),
 *   sequences packed back to back and delimited by cu_seqlens.
 *
 * Each token is applied exactly as written: first the product
 * S_{t-1}(I - beta k k^T) = S - beta (S k) k^T, then the scaling by alpha,
 * then the rank-one write beta v k^T.  Everything is double precision; the
 * inputs are whatever values the caller passes (bf16 or fp32 inputs widen
 * exactly to double).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG (-1)
#define ORACLE_NO_MEMORY (-2)

/* One (sequence, head) unit: tokens [t0, t1) of head h. */
static void run_unit(const double* q, const double* k, const double* v,
                     const double* beta, const double* gate, int gate_is_log,
                     int64_t t0, int64_t t1, int H, int h, int dk, int dv,
                     double scale, const double* s0, double* o, double* s_out,
                     double* S, double* p) {
  if (s0) memcpy(S, s0, sizeof(double) * (size_t)dv * dk);
  else memset(S, 0, sizeof(double) * (size_t)dv * dk);
  for (int64_t t = t0; t < t1; t++) {
    const double* kt = k + ((size_t)t * H + h) * dk;
    const double* vt = v + ((size_t)t * H + h) * dv;
    const double* qt = q + ((size_t)t * H + h) * dk;
    double b = beta[(size_t)t * H + h];
    double gt = gate[(size_t)t * H + h];
    double a = gate_is_log ? exp(gt) : gt;
    /* p = S_{t-1} k_t */
    for (int r = 0; r < dv; r++) {
      double acc = 0.0;
      for (int j = 0; j < dk; j++) acc += S[(size_t)r * dk + j] * kt[j];
      p[r] = acc;
    }
    /* S_t = a * (S_{t-1} - b p k^T) + b v k^T */
    for (int r = 0; r < dv; r++) {
      for (int j = 0; j < dk; j++) {
        double s = S[(size_t)r * dk + j];
        S[(size_t)r * dk + j] = a * (s - b * p[r] * kt[j]) + b * vt[r] * kt[j];
      }
    }
    /* o_t = scale * S_t q_t */
    double* ot = o + ((size_t)t * H + h) * dv;
    for (int r = 0; r < dv; r++) {
      double acc = 0.0;
      for (int j = 0; j < dk; j++) acc += S[(size_t)r * dk + j] * qt[j];
      ot[r] = scale * acc;
    }
  }
  if (s_out) memcpy(s_out, S, sizeof(double) * (size_t)dv * dk);
}

static int run_all(const double* q, const double* k, const double* v,
                   const double* beta, const double* gate, int gate_is_log,
                   const int32_t* cu_seqlens, int n_seqs, int H, int dk, int dv,
                   double scale, const double* h0, double* o, double* s_final,
                   int n_threads) {
  if (!q || !k || !v || !beta || !gate || !cu_seqlens || !o) return ORACLE_BAD_ARG;
  if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0) return ORACLE_BAD_ARG;
  if (cu_seqlens[0] != 0) return ORACLE_BAD_ARG;
  for (int n = 0; n < n_seqs; n++)
    if (cu_seqlens[n + 1] < cu_seqlens[n]) return ORACLE_BAD_ARG;
  int64_t units = (int64_t)n_seqs * H;
  int failed = 0;
#ifdef _OPENMP
  if (n_threads <= 0) n_threads = omp_get_max_threads();
#pragma omp parallel num_threads(n_threads)
#endif
  {
    double* S = (double*)malloc(sizeof(double) * (size_t)dv * dk);
    double* p = (double*)malloc(sizeof(double) * (size_t)dv);
    if (!S || !p) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
      failed = 1;
    } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
      for (int64_t u = 0; u < units; u++) {
        int n = (int)(u / H), h = (int)(u % H);
        const double* s0 = h0 ? h0 + (size_t)u * dv * dk : NULL;
        double* s_out = s_final ? s_final + (size_t)u * dv * dk : NULL;
        run_unit(q, k, v, beta, gate, gate_is_log, cu_seqlens[n], cu_seqlens[n + 1], H, h,
                 dk, dv, scale, s0, o, s_out, S, p);
      }
    }
    free(S);
    free(p);
  }
  return failed ? ORACLE_NO_MEMORY : ORACLE_OK;
}

/* Gate given as log-decay g (alpha = exp(g), computed here in double). */
int gdn_oracle_forward(const double* q, const double* k, const double* v, const double* beta,
                       const double* g, const int32_t* cu_seqlens, int n_seqs, int H, int dk,
                       int dv, double scale, const double* h0, double* o, double* s_final,
                       int n_threads) {
  return run_all(q, k, v, beta, g, 1, cu_seqlens, n_seqs, H, dk, dv, scale, h0, o, s_final,
                 n_threads);
}

/* Gate given directly as alpha (used for exact-rational and alpha = 0 checks). */
int gdn_oracle_forward_alpha(const double* q, const double* k, const double* v,
                             const double* beta, const double* alpha, const int32_t* cu_seqlens,
                             int n_seqs, int H, int dk, int dv, double scale, const double* h0,
                             double* o, double* s_final, int n_threads) {
  return run_all(q, k, v, beta, alpha, 0, cu_seqlens, n_seqs, H, dk, dv, scale, h0, o, s_final,
                 n_threads);
}

/* Number of threads an OpenMP region started with n_threads<=0 would use. */
int gdn_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
