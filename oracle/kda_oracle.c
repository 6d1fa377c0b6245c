/*
 * kda_oracle.c -- the plain, slow, obviously-correct fp64 CPU oracle for the
 * Kimi Delta Attention (KDA) recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  The test-suite, the smoke check and the
 * benchmark's CPU-baseline leg call it; the product (the CUDA library under
 * kimi_delta_attention_31_b200/) never does, and the two share no code,
 * header, table or helper.
 *
 * Sources (web pages, cited by title and section):
 *   [notes]  "Kimi K3 notes 1: KDA" (jaimeyzzz.com), section 4 (KDA state
 *            update, the projection form) and section 5 (boxed summary:
 *            decay with Diag(alpha_t), then the delta correction).
 *   [deriv]  "Deriving Kimi Delta Attention from scratch" (HN summary),
 *            sections 3-5: predict v^ from the (decayed) state with the key,
 *            error e = beta (v - v^), write e along the key, read with q;
 *            section 6: the chunked mode is a schedule of the same formula.
 *   [tutor]  "Linear / sparse attention" tutorial (mathieu0905), section 6.2
 *            (chunk = inter term through the carried state + intra term
 *            inside the chunk + state hand-off) and appendix A (the
 *            schedule-equivalence invariants).
 *
 * Conventions (the same layouts the CUDA library uses, written out here
 * independently):
 *   q, k, g : [B, T, H, dk]    v, o : [B, T, H, dv]    beta : [B, T, H]
 *   S0, S_out : [N, H, dk, dv] (row c = key channel, column j = value channel)
 *   g is log(alpha) per key channel.  With cu_seqlens (length num_seqs+1) the
 *   token axis is one packed stream (B = 1, T = total) and sequence n owns
 *   tokens [cu_seqlens[n], cu_seqlens[n+1]); without it, N = B sequences of
 *   length T.
 *
 * Per token (decay first, then predict / correct / read, [notes] section 5):
 *   S~   = Diag(alpha_t) S_{t-1}          (row c scaled by alpha_{t,c})
 *   v^   = S~^T k_t
 *   e_t  = beta_t (v_t - v^)
 *   S_t  = S~ + k_t e_t^T
 *   o_t  = S_t^T q_t                     (the post-update state)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Test knob: force the prediction v^ to zero (the "erase term dropped" case
 * of [tutor] appendix A item 4).  Not a mutation: a documented variant. */
#define KDA_ORACLE_NO_ERASE 1
/* Deliberate mistakes, planted only by the mutation tests to show that the
 * pins catch each plausible error.  Never set outside those tests. */
#define KDA_ORACLE_MUT_GATE_ON_VALUE_AXIS 0x100 /* scale columns, not rows   */
#define KDA_ORACLE_MUT_PREDICT_UNDECAYED 0x200  /* v^ from S_{t-1}, not S~   */
#define KDA_ORACLE_MUT_OUTPUT_PRE_WRITE 0x400   /* o from S~, not S_t        */
#define KDA_ORACLE_MUT_NO_DECAY 0x800           /* alpha ignored             */
#define KDA_ORACLE_MUT_READ_TRANSPOSED 0x1000   /* o_j = sum_c S[j][c] q_c   */
#define KDA_ORACLE_MUT_ERROR_SIGN 0x2000        /* e = beta (v^ - v)         */

static int kda_oracle_num_units(const int64_t *cu_seqlens, int num_seqs, int B) {
  return cu_seqlens ? num_seqs : B;
}

static void kda_oracle_seq_range(const int64_t *cu_seqlens, int n, int T,
                                 int64_t *start, int64_t *end) {
  if (cu_seqlens) {
    *start = cu_seqlens[n];
    *end = cu_seqlens[n + 1];
  } else {
    *start = (int64_t)n * T;
    *end = (int64_t)(n + 1) * T;
  }
}

static int kda_oracle_check(const int64_t *cu_seqlens, int num_seqs, int B,
                            int T, int H, int dk, int dv) {
  if (H <= 0 || dk <= 0 || dv <= 0 || B < 0 || T < 0) return 1;
  if (cu_seqlens) {
    if (num_seqs < 0 || B != 1) return 1;
    if (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T) return 1;
    for (int n = 0; n < num_seqs; ++n)
      if (cu_seqlens[n + 1] < cu_seqlens[n]) return 1;
  }
  return 0;
}

/*
 * Token-by-token recurrence: the definition.  S_hist (optional, may be NULL)
 * receives S_t after every token, laid out like o but with dk*dv entries per
 * (token, head); only for small cases.
 * Returns 0 on success, 1 on inconsistent sizes, 2 on allocation failure.
 */
int kda_oracle_recurrent(const double *q, const double *k, const double *v,
                         const double *g, const double *beta, const double *S0,
                         double *o, double *S_out, const int64_t *cu_seqlens,
                         int num_seqs, int B, int T, int H, int dk, int dv,
                         int flags, double *S_hist, int num_threads) {
  if (kda_oracle_check(cu_seqlens, num_seqs, B, T, H, dk, dv)) return 1;
  if ((flags & (KDA_ORACLE_MUT_GATE_ON_VALUE_AXIS | KDA_ORACLE_MUT_READ_TRANSPOSED)) &&
      dk != dv)
    return 1;
  const int N = kda_oracle_num_units(cu_seqlens, num_seqs, B);
  const int64_t units = (int64_t)N * H;
  int failed = 0;
#ifdef _OPENMP
  if (num_threads <= 0) num_threads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads) reduction(| : failed)
#endif
  for (int64_t u = 0; u < units; ++u) {
    const int n = (int)(u / H), h = (int)(u % H);
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *vhat = (double *)malloc(sizeof(double) * (size_t)dv);
    double *e = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!S || !vhat || !e) {
      free(S); free(vhat); free(e);
      failed |= 1;
      continue;
    }
    if (S0)
      memcpy(S, S0 + (size_t)u * dk * dv, sizeof(double) * (size_t)dk * dv);
    else
      memset(S, 0, sizeof(double) * (size_t)dk * dv);

    int64_t t0, t1;
    kda_oracle_seq_range(cu_seqlens, n, T, &t0, &t1);
    for (int64_t t = t0; t < t1; ++t) {
      const size_t rk = ((size_t)t * H + h) * dk;
      const size_t rv = ((size_t)t * H + h) * dv;
      const double *qt = q + rk, *kt = k + rk, *gt = g + rk, *vt = v + rv;
      const double bt = beta[(size_t)t * H + h];

      /* prediction from the undecayed state: only under the mutation */
      if (flags & KDA_ORACLE_MUT_PREDICT_UNDECAYED) {
        for (int j = 0; j < dv; ++j) {
          double acc = 0.0;
          for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * kt[c];
          vhat[j] = acc;
        }
      }
      /* S~ = Diag(alpha_t) S_{t-1}: the gate acts on the key channel (row) */
      if (!(flags & KDA_ORACLE_MUT_NO_DECAY)) {
        for (int c = 0; c < dk; ++c) {
          const double a = exp(gt[c]);
          if (flags & KDA_ORACLE_MUT_GATE_ON_VALUE_AXIS) {
            for (int r = 0; r < dk; ++r) S[(size_t)r * dv + c] *= a;
          } else {
            for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= a;
          }
        }
      }
      /* v^ = S~^T k_t */
      if (!(flags & KDA_ORACLE_MUT_PREDICT_UNDECAYED)) {
        for (int j = 0; j < dv; ++j) {
          double acc = 0.0;
          for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * kt[c];
          vhat[j] = acc;
        }
      }
      if (flags & KDA_ORACLE_NO_ERASE)
        for (int j = 0; j < dv; ++j) vhat[j] = 0.0;
      /* e_t = beta_t (v_t - v^) */
      for (int j = 0; j < dv; ++j)
        e[j] = (flags & KDA_ORACLE_MUT_ERROR_SIGN) ? bt * (vhat[j] - vt[j])
                                                   : bt * (vt[j] - vhat[j]);
      /* o from S~ (pre-write) only under the mutation */
      double *ot = o + rv;
      if (flags & KDA_ORACLE_MUT_OUTPUT_PRE_WRITE) {
        for (int j = 0; j < dv; ++j) {
          double acc = 0.0;
          for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * qt[c];
          ot[j] = acc;
        }
      }
      /* S_t = S~ + k_t e_t^T */
      for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] += kt[c] * e[j];
      /* o_t = S_t^T q_t */
      if (!(flags & KDA_ORACLE_MUT_OUTPUT_PRE_WRITE)) {
        for (int j = 0; j < dv; ++j) {
          double acc = 0.0;
          if (flags & KDA_ORACLE_MUT_READ_TRANSPOSED) {
            for (int c = 0; c < dk; ++c) acc += S[(size_t)j * dv + c] * qt[c];
          } else {
            for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * qt[c];
          }
          ot[j] = acc;
        }
      }
      if (S_hist)
        memcpy(S_hist + ((size_t)t * H + h) * dk * dv, S,
               sizeof(double) * (size_t)dk * dv);
    }
    if (S_out) memcpy(S_out + (size_t)u * dk * dv, S, sizeof(double) * (size_t)dk * dv);
    free(S); free(vhat); free(e);
  }
  return failed ? 2 : 0;
}

/*
 * Chunkwise schedule in fp64, written from the algebra, not from any kernel:
 * within a chunk of C tokens starting from the carried state S_c, with
 * G_r = sum_{i<=r} g_i (cumulative log-decay, chunk-relative),
 *   (I + A) E = diag(beta) (V - (K o e^G) S_c),
 *       A_rj = beta_r sum_c k_rc k_jc e^{G_rc - G_jc}     (j < r)
 *   O   = (Q o e^G) S_c + P E,  P_rj = sum_c q_rc k_jc e^{G_rc - G_jc} (j <= r)
 *   S_{c+1} = Diag(e^{G_last}) S_c + (K o e^{G_last - G})^T E
 * ([deriv] section 6: lower-triangular system that corrects each token's
 * provisional error; [tutor] section 6.2: inter + intra split and the state
 * hand-off, with the decays folded in).  The pairwise exponentials are taken
 * directly (every exponent is <= 0) and the triangular system is solved by
 * plain forward substitution.  Chunks restart at every sequence start; the
 * last chunk of a sequence may be short.
 */
int kda_oracle_chunk(const double *q, const double *k, const double *v,
                     const double *g, const double *beta, const double *S0,
                     double *o, double *S_out, const int64_t *cu_seqlens,
                     int num_seqs, int B, int T, int H, int dk, int dv,
                     int chunk_size, int num_threads) {
  if (kda_oracle_check(cu_seqlens, num_seqs, B, T, H, dk, dv)) return 1;
  if (chunk_size <= 0) return 1;
  const int N = kda_oracle_num_units(cu_seqlens, num_seqs, B);
  const int64_t units = (int64_t)N * H;
  const int C = chunk_size;
  int failed = 0;
#ifdef _OPENMP
  if (num_threads <= 0) num_threads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads) reduction(| : failed)
#endif
  for (int64_t u = 0; u < units; ++u) {
    const int n = (int)(u / H), h = (int)(u % H);
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *Sn = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *G = (double *)malloc(sizeof(double) * (size_t)C * dk);
    double *A = (double *)malloc(sizeof(double) * (size_t)C * C);
    double *P = (double *)malloc(sizeof(double) * (size_t)C * C);
    double *E = (double *)malloc(sizeof(double) * (size_t)C * dv);
    if (!S || !Sn || !G || !A || !P || !E) {
      free(S); free(Sn); free(G); free(A); free(P); free(E);
      failed |= 1;
      continue;
    }
    if (S0)
      memcpy(S, S0 + (size_t)u * dk * dv, sizeof(double) * (size_t)dk * dv);
    else
      memset(S, 0, sizeof(double) * (size_t)dk * dv);

    int64_t t0, t1;
    kda_oracle_seq_range(cu_seqlens, n, T, &t0, &t1);
    for (int64_t s = t0; s < t1; s += C) {
      const int Cn = (int)((t1 - s) < C ? (t1 - s) : C);
#define ROWK(r) (((size_t)(s + (r)) * H + h) * dk)
#define ROWV(r) (((size_t)(s + (r)) * H + h) * dv)
#define BETA(r) (beta[(size_t)(s + (r)) * H + h])
      /* cumulative log-decay inside the chunk */
      for (int c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int r = 0; r < Cn; ++r) {
          acc += g[ROWK(r) + c];
          G[(size_t)r * dk + c] = acc;
        }
      }
      /* A (strictly lower) and P (lower, with diagonal), pairwise ratios */
      for (int r = 0; r < Cn; ++r) {
        for (int j = 0; j < Cn; ++j) {
          double a = 0.0, p = 0.0;
          if (j <= r) {
            for (int c = 0; c < dk; ++c) {
              const double w = exp(G[(size_t)r * dk + c] - G[(size_t)j * dk + c]);
              a += k[ROWK(r) + c] * k[ROWK(j) + c] * w;
              p += q[ROWK(r) + c] * k[ROWK(j) + c] * w;
            }
          }
          A[(size_t)r * C + j] = (j < r) ? BETA(r) * a : 0.0;
          P[(size_t)r * C + j] = (j <= r) ? p : 0.0;
        }
      }
      /* right-hand side, then forward substitution: (I + A) E = rhs */
      for (int r = 0; r < Cn; ++r) {
        for (int jv = 0; jv < dv; ++jv) {
          double pred = 0.0;
          for (int c = 0; c < dk; ++c)
            pred += k[ROWK(r) + c] * exp(G[(size_t)r * dk + c]) * S[(size_t)c * dv + jv];
          double rhs = BETA(r) * (v[ROWV(r) + jv] - pred);
          for (int j = 0; j < r; ++j) rhs -= A[(size_t)r * C + j] * E[(size_t)j * dv + jv];
          E[(size_t)r * dv + jv] = rhs;
        }
      }
      /* outputs: inter term through S_c plus intra term P E */
      for (int r = 0; r < Cn; ++r) {
        for (int jv = 0; jv < dv; ++jv) {
          double acc = 0.0;
          for (int c = 0; c < dk; ++c)
            acc += q[ROWK(r) + c] * exp(G[(size_t)r * dk + c]) * S[(size_t)c * dv + jv];
          for (int j = 0; j <= r; ++j) acc += P[(size_t)r * C + j] * E[(size_t)j * dv + jv];
          o[ROWV(r) + jv] = acc;
        }
      }
      /* state hand-off */
      for (int c = 0; c < dk; ++c) {
        const double Gl = G[(size_t)(Cn - 1) * dk + c];
        for (int jv = 0; jv < dv; ++jv) {
          double acc = exp(Gl) * S[(size_t)c * dv + jv];
          for (int r = 0; r < Cn; ++r)
            acc += k[ROWK(r) + c] * exp(Gl - G[(size_t)r * dk + c]) * E[(size_t)r * dv + jv];
          Sn[(size_t)c * dv + jv] = acc;
        }
      }
      memcpy(S, Sn, sizeof(double) * (size_t)dk * dv);
#undef ROWK
#undef ROWV
#undef BETA
    }
    if (S_out) memcpy(S_out + (size_t)u * dk * dv, S, sizeof(double) * (size_t)dk * dv);
    free(S); free(Sn); free(G); free(A); free(P); free(E);
  }
  return failed ? 2 : 0;
}

/* Thread count the oracle uses when given num_threads <= 0. */
int kda_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
