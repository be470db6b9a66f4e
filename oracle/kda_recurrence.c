/*
 * fp64 CPU oracle of the Kimi Delta Attention (KDA) forward recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this file's library.  The CUDA path shares no code
 * with it; it is built separately by oracle/build_oracle.py.
 *
 * What it computes (plain definition, one (sequence, head) at a time, every
 * number in double precision, token by token in the order the tokens arrive):
 *
 *   S  <- S_init            (or zero)                  S is d_k x d_v
 *   for each token t:
 *     S'  = Diag(exp(l_t)) S                            decay, per key channel
 *     e   = S'^T k_t                                    what the memory returns
 *     S   = S' + beta_t k_t (v_t - e)^T                 delta-rule write
 *     o_t = S^T q_t                                     read with the query
 *   final_state = S
 *
 * Sources, stated in this file's own words:
 *  - Delta rule: read the stored value S^T k for key k, form the error v - S^T k
 *    and write the error back along k, scaled by beta_t.
 *    ("Kimi Delta Attention", akshathtiwari.co.in, the delta-rule passage;
 *     "Attention? More like notation warfare", Key Points, last item;
 *     "The fourth layer remembers", section "What each kind of layer keeps".)
 *  - Per-channel forget vector alpha_t applied as Diag(alpha_t) to the previous
 *    state before the write; each key channel (a row of S) decays at its own
 *    rate.  ("Kimi Delta Attention", akshathtiwari.co.in, channel-wise gating
 *    passage; "Teacher guide - Kimi Delta Attention", Misconceptions table,
 *    row 2, S' = diag(a) S; "The fourth layer remembers", the paragraph on the
 *    g_t forget gate.)
 *  - Readings where the pages are silent: the error is read from the decayed
 *    state S' (the (I - beta k k^T) Diag(alpha) transition form); S is
 *    d_k x d_v with the decay on rows; the output reads the updated state S_t;
 *    the gate arrives as log(alpha) = l_t <= 0 and is exponentiated here.
 *
 * Layout (all row-major, double, host memory owned by the caller):
 *   q, k, log_alpha : [T_total, H, d_k]
 *   v, out          : [T_total, H, d_v]
 *   beta            : [T_total, H]
 *   state_in/out    : [n_seqs, H, d_k, d_v]    (state_in may be NULL = zeros)
 *   seq_offsets     : [n_seqs + 1] token offsets; sequence s owns tokens
 *                     seq_offsets[s] .. seq_offsets[s+1]-1.
 * Returns 0, or -1 on an argument error.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static void one_sequence_head(int64_t t0, int64_t t1, int64_t h, int64_t H,
                              int64_t dk, int64_t dv, const double* q,
                              const double* k, const double* v,
                              const double* log_alpha, const double* beta,
                              const double* s_in, double* out, double* s_out,
                              double* e /* scratch, d_v */) {
  /* The running state lives in s_out: start it from s_in or from zero. */
  if (s_in)
    memcpy(s_out, s_in, (size_t)(dk * dv) * sizeof(double));
  else
    memset(s_out, 0, (size_t)(dk * dv) * sizeof(double));
  double* S = s_out;

  for (int64_t t = t0; t < t1; ++t) {
    const double* kt = k + (t * H + h) * dk;
    const double* qt = q + (t * H + h) * dk;
    const double* lt = log_alpha + (t * H + h) * dk;
    const double* vt = v + (t * H + h) * dv;
    const double bt = beta[t * H + h];
    double* ot = out + (t * H + h) * dv;

    /* S' = Diag(alpha_t) S : row c (key channel c) scaled by exp(l_t[c]). */
    for (int64_t c = 0; c < dk; ++c) {
      const double a = exp(lt[c]);
      for (int64_t j = 0; j < dv; ++j) S[c * dv + j] *= a;
    }
    /* e = S'^T k_t */
    for (int64_t j = 0; j < dv; ++j) e[j] = 0.0;
    for (int64_t c = 0; c < dk; ++c)
      for (int64_t j = 0; j < dv; ++j) e[j] += S[c * dv + j] * kt[c];
    /* S = S' + beta_t k_t (v_t - e)^T */
    for (int64_t c = 0; c < dk; ++c)
      for (int64_t j = 0; j < dv; ++j)
        S[c * dv + j] += bt * kt[c] * (vt[j] - e[j]);
    /* o_t = S_t^T q_t */
    for (int64_t j = 0; j < dv; ++j) ot[j] = 0.0;
    for (int64_t c = 0; c < dk; ++c)
      for (int64_t j = 0; j < dv; ++j) ot[j] += S[c * dv + j] * qt[c];
  }
}

int kda_oracle_recurrent(int64_t n_seqs, const int64_t* seq_offsets, int64_t H,
                         int64_t dk, int64_t dv, const double* q,
                         const double* k, const double* v,
                         const double* log_alpha, const double* beta,
                         const double* state_in, double* out,
                         double* state_out) {
  if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !seq_offsets || !q || !k ||
      !v || !log_alpha || !beta || !out || !state_out)
    return -1;
  for (int64_t s = 0; s < n_seqs; ++s)
    if (seq_offsets[s + 1] < seq_offsets[s]) return -1;

  const int64_t units = n_seqs * H;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t u = 0; u < units; ++u) {
    const int64_t s = u / H, h = u % H;
    double* e = (double*)malloc((size_t)dv * sizeof(double));
    if (!e) {
      bad |= 1;
      continue;
    }
    one_sequence_head(seq_offsets[s], seq_offsets[s + 1], h, H, dk, dv, q, k,
                      v, log_alpha, beta,
                      state_in ? state_in + (s * H + h) * dk * dv : NULL, out,
                      state_out + (s * H + h) * dk * dv, e);
    free(e);
  }
  return bad ? -1 : 0;
}

/* The number of threads an OpenMP parallel region of this library uses. */
int kda_oracle_num_threads(void) {
  int n = 1;
#ifdef _OPENMP
#pragma omp parallel
  {
#pragma omp single
    n = omp_get_num_threads();
  }
#endif
  return n;
}
