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

/*
 * Reverse mode of the same recurrence (the gradient of a loss through the
 * token loop above, plain definition, fp64).  Given dO = dL/do_t and dS_end =
 * dL/dS_final, it returns dL/dq, dL/dk, dL/dv, dL/dbeta, dL/dg and dL/dh0.
 * Per token, with p = S_{t-1} k_t, a = exp(g_t), b = beta_t and
 * S_t = a (S_{t-1} - b p k^T) + b v k^T, o_t = scale S_t q_t, walking t
 * downwards with dS = dL/dS_t:
 *   dS   += scale do_t q_t^T           dq_t  = scale S_t^T do_t
 *   w     = dS k_t                     da    = <dS, S_{t-1}> - b w.p
 *   dbeta = w.(v_t - a p)              dv_t  = b w
 *   dk_t  = dS^T (b (v_t - a p)) + S_{t-1}^T dp,   dp = -a b w
 *   dg_t  = a da                       dS_{t-1} = a dS + dp k_t^T
 * and finally dh0 = dS.  States are kept at every ORACLE_CKPT-th token and the
 * ones in between recomputed by the forward loop (the same operations in the
 * same order, so the same values).
 */
#define ORACLE_CKPT 64

static void fwd_token(double* S, double* p, const double* kt, const double* vt, double a,
                      double b, int dk, int dv) {
  for (int r = 0; r < dv; r++) {
    double acc = 0.0;
    for (int j = 0; j < dk; j++) acc += S[(size_t)r * dk + j] * kt[j];
    p[r] = acc;
  }
  for (int r = 0; r < dv; r++)
    for (int j = 0; j < dk; j++) {
      double s = S[(size_t)r * dk + j];
      S[(size_t)r * dk + j] = a * (s - b * p[r] * kt[j]) + b * vt[r] * kt[j];
    }
}

static void bwd_unit(const double* q, const double* k, const double* v, const double* beta,
                     const double* g, int64_t t0, int64_t t1, int H, int h, int dk, int dv,
                     double scale, const double* s0, const double* dO, const double* dS_end,
                     double* dq, double* dkk, double* dvv, double* dbeta, double* dg,
                     double* dh0, double* ck, double* st, double* dS, double* p, double* w) {
  const size_t DD = (size_t)dv * dk;
  const int64_t L = t1 - t0;
  const int64_t nck = (L + ORACLE_CKPT - 1) / ORACLE_CKPT;
  /* checkpoints: state before token t0 + c * ORACLE_CKPT */
  if (s0) memcpy(ck, s0, sizeof(double) * DD);
  else memset(ck, 0, sizeof(double) * DD);
  for (int64_t c = 1; c < nck; c++) {
    memcpy(ck + (size_t)c * DD, ck + (size_t)(c - 1) * DD, sizeof(double) * DD);
    for (int64_t t = t0 + (c - 1) * ORACLE_CKPT; t < t0 + c * ORACLE_CKPT; t++) {
      const size_t u = (size_t)t * H + h;
      fwd_token(ck + (size_t)c * DD, p, k + u * dk, v + u * dv, exp(g[u]), beta[u], dk, dv);
    }
  }
  if (dS_end) memcpy(dS, dS_end, sizeof(double) * DD);
  else memset(dS, 0, sizeof(double) * DD);
  for (int64_t c = nck - 1; c >= 0; c--) {
    const int64_t a0 = t0 + c * ORACLE_CKPT;
    const int64_t a1 = (a0 + ORACLE_CKPT < t1) ? a0 + ORACLE_CKPT : t1;
    /* st[i] = state before token a0 + i, i = 0 .. a1 - a0 (last = after a1 - 1) */
    memcpy(st, ck + (size_t)c * DD, sizeof(double) * DD);
    for (int64_t t = a0; t < a1; t++) {
      const size_t u = (size_t)t * H + h;
      double* nx = st + (size_t)(t - a0 + 1) * DD;
      memcpy(nx, st + (size_t)(t - a0) * DD, sizeof(double) * DD);
      fwd_token(nx, p, k + u * dk, v + u * dv, exp(g[u]), beta[u], dk, dv);
    }
    for (int64_t t = a1 - 1; t >= a0; t--) {
      const size_t u = (size_t)t * H + h;
      const double* Sp = st + (size_t)(t - a0) * DD;      /* S_{t-1} */
      const double* Sc = st + (size_t)(t - a0 + 1) * DD;  /* S_t */
      const double *kt = k + u * dk, *vt = v + u * dv, *qt = q + u * dk, *dot = dO + u * dv;
      const double a = exp(g[u]), b = beta[u];
      for (int r = 0; r < dv; r++)
        for (int j = 0; j < dk; j++) dS[(size_t)r * dk + j] += scale * dot[r] * qt[j];
      for (int j = 0; j < dk; j++) {
        double acc = 0.0;
        for (int r = 0; r < dv; r++) acc += Sc[(size_t)r * dk + j] * dot[r];
        dq[u * dk + j] = scale * acc;
      }
      for (int r = 0; r < dv; r++) {
        double acc = 0.0, pr = 0.0;
        for (int j = 0; j < dk; j++) {
          acc += dS[(size_t)r * dk + j] * kt[j];
          pr += Sp[(size_t)r * dk + j] * kt[j];
        }
        w[r] = acc;
        p[r] = pr;
      }
      double da = 0.0, db = 0.0;
      for (size_t e = 0; e < DD; e++) da += dS[e] * Sp[e];
      for (int r = 0; r < dv; r++) {
        da -= b * w[r] * p[r];
        db += w[r] * (vt[r] - a * p[r]);
        dvv[u * dv + r] = b * w[r];
      }
      for (int j = 0; j < dk; j++) {
        double acc = 0.0;
        for (int r = 0; r < dv; r++) {
          const double dpr = -a * b * w[r];
          acc += dS[(size_t)r * dk + j] * (b * (vt[r] - a * p[r])) + Sp[(size_t)r * dk + j] * dpr;
        }
        dkk[u * dk + j] = acc;
      }
      dbeta[u] = db;
      dg[u] = a * da;
      for (int r = 0; r < dv; r++) {
        const double dpr = -a * b * w[r];
        for (int j = 0; j < dk; j++)
          dS[(size_t)r * dk + j] = a * dS[(size_t)r * dk + j] + dpr * kt[j];
      }
    }
  }
  if (dh0) memcpy(dh0, dS, sizeof(double) * DD);
}

int gdn_oracle_backward(const double* q, const double* k, const double* v, const double* beta,
                        const double* g, const int32_t* cu_seqlens, int n_seqs, int H, int dk,
                        int dv, double scale, const double* h0, const double* dO,
                        const double* dS_end, double* dq, double* dkk, double* dvv,
                        double* dbeta, double* dg, double* dh0, int n_threads) {
  if (!q || !k || !v || !beta || !g || !cu_seqlens || !dO || !dq || !dkk || !dvv || !dbeta ||
      !dg)
    return ORACLE_BAD_ARG;
  if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || cu_seqlens[0] != 0) return ORACLE_BAD_ARG;
  int64_t maxlen = 0;
  for (int n = 0; n < n_seqs; n++) {
    if (cu_seqlens[n + 1] < cu_seqlens[n]) return ORACLE_BAD_ARG;
    if (cu_seqlens[n + 1] - cu_seqlens[n] > maxlen) maxlen = cu_seqlens[n + 1] - cu_seqlens[n];
  }
  const size_t DD = (size_t)dv * dk;
  const int64_t nck = (maxlen + ORACLE_CKPT - 1) / ORACLE_CKPT + 1;
  const int64_t units = (int64_t)n_seqs * H;
  int failed = 0;
#ifdef _OPENMP
  if (n_threads <= 0) n_threads = omp_get_max_threads();
#pragma omp parallel num_threads(n_threads)
#endif
  {
    double* ck = (double*)malloc(sizeof(double) * DD * (size_t)nck);
    double* st = (double*)malloc(sizeof(double) * DD * (ORACLE_CKPT + 1));
    double* dS = (double*)malloc(sizeof(double) * DD);
    double* p = (double*)malloc(sizeof(double) * (size_t)dv);
    double* w = (double*)malloc(sizeof(double) * (size_t)dv);
    if (!ck || !st || !dS || !p || !w) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
      failed = 1;
    } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
      for (int64_t u = 0; u < units; u++) {
        const int n = (int)(u / H), h = (int)(u % H);
        bwd_unit(q, k, v, beta, g, cu_seqlens[n], cu_seqlens[n + 1], H, h, dk, dv, scale,
                 h0 ? h0 + (size_t)u * DD : NULL, dO, dS_end ? dS_end + (size_t)u * DD : NULL,
                 dq, dkk, dvv, dbeta, dg, dh0 ? dh0 + (size_t)u * DD : NULL, ck, st, dS, p, w);
      }
    }
    free(ck);
    free(st);
    free(dS);
    free(p);
    free(w);
  }
  return failed ? ORACLE_NO_MEMORY : ORACLE_OK;
}
