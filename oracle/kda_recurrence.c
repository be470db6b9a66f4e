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

/*
 * Gradients of the same recurrence, reverse mode, fp64 (the backward pass).
 *
 * For the scalar  L = sum_t <dO_t, o_t> + <dS_T, S_T>  (dS_T may be NULL =
 * zero) it returns dL/dq, dL/dk, dL/dv, dL/dlog_alpha, dL/dbeta and dL/dS_0,
 * in the forward's layouts (d_state_in may be NULL when not wanted).
 *
 * With D = dL/dS_t carried backwards and, for token t, S' = Diag(a_t) S_{t-1},
 * e = S'^T k_t, d = beta_t (v_t - e), S_t = S' + k_t d^T, o_t = S_t^T q_t:
 *   D    += q_t dO_t^T              dq_t   = S_t dO_t
 *   dd    = D^T k_t                 dk_t   = D d
 *   dv_t  = beta_t dd               dbeta_t = <dd, v_t - e>      de = -beta_t dd
 *   D'    = D + k_t de^T            dk_t  += S' de
 *   dlog_alpha_t = rowsum(D' .* S') (d/dl of exp(l) S_{t-1} is exp(l) S_{t-1})
 *   D    <- Diag(a_t) D'            (the gradient of S_{t-1})
 * Each line is the chain rule applied to one line of the forward step.  The
 * forward states are recomputed: S is saved at the start of every block of 64
 * tokens, and the reverse pass over a block first re-runs the block's forward
 * steps into a buffer.
 */
static void forward_step(int64_t dk, int64_t dv, const double* kt,
                         const double* lt, const double* vt, double bt,
                         const double* S_prev, double* S_next, double* Sp,
                         double* e) {
  for (int64_t c = 0; c < dk; ++c) {
    const double a = exp(lt[c]);
    for (int64_t j = 0; j < dv; ++j) Sp[c * dv + j] = a * S_prev[c * dv + j];
  }
  for (int64_t j = 0; j < dv; ++j) e[j] = 0.0;
  for (int64_t c = 0; c < dk; ++c)
    for (int64_t j = 0; j < dv; ++j) e[j] += Sp[c * dv + j] * kt[c];
  for (int64_t c = 0; c < dk; ++c)
    for (int64_t j = 0; j < dv; ++j)
      S_next[c * dv + j] = Sp[c * dv + j] + bt * kt[c] * (vt[j] - e[j]);
}

static int one_sequence_head_bwd(int64_t t0, int64_t t1, int64_t h, int64_t H,
                                 int64_t dk, int64_t dv, const double* q,
                                 const double* k, const double* v,
                                 const double* log_alpha, const double* beta,
                                 const double* s_in, const double* d_out,
                                 const double* ds_out, double* dq, double* dk_g,
                                 double* dv_g, double* dla, double* dbeta,
                                 double* ds_in) {
  const int64_t BLK = 64, T = t1 - t0, nblk = (T + BLK - 1) / BLK;
  const size_t SZ = (size_t)(dk * dv);
  double* ck = (double*)malloc((size_t)(nblk + 1) * SZ * sizeof(double));
  double* st = (double*)malloc((size_t)(BLK + 1) * SZ * sizeof(double));
  double* D = (double*)malloc(SZ * sizeof(double));
  double* Sp = (double*)malloc(SZ * sizeof(double));
  double* e = (double*)malloc((size_t)dv * sizeof(double));
  double* dd = (double*)malloc((size_t)dv * sizeof(double));
  double* de = (double*)malloc((size_t)dv * sizeof(double));
  if (!ck || !st || !D || !Sp || !e || !dd || !de) {
    free(ck); free(st); free(D); free(Sp); free(e); free(dd); free(de);
    return -1;
  }
  /* forward sweep: the state at the start of every block */
  if (s_in) memcpy(ck, s_in, SZ * sizeof(double));
  else memset(ck, 0, SZ * sizeof(double));
  for (int64_t b = 0; b < nblk; ++b) {
    memcpy(st, ck + (size_t)b * SZ, SZ * sizeof(double));
    const int64_t tb = t0 + b * BLK, te = tb + BLK < t1 ? tb + BLK : t1;
    for (int64_t t = tb; t < te; ++t) {
      forward_step(dk, dv, k + (t * H + h) * dk, log_alpha + (t * H + h) * dk,
                   v + (t * H + h) * dv, beta[t * H + h], st, st + SZ, Sp, e);
      memcpy(st, st + SZ, SZ * sizeof(double));
    }
    memcpy(ck + (size_t)(b + 1) * SZ, st, SZ * sizeof(double));
  }
  /* reverse sweep */
  if (ds_out) memcpy(D, ds_out, SZ * sizeof(double));
  else memset(D, 0, SZ * sizeof(double));
  for (int64_t b = nblk - 1; b >= 0; --b) {
    const int64_t tb = t0 + b * BLK, te = tb + BLK < t1 ? tb + BLK : t1;
    memcpy(st, ck + (size_t)b * SZ, SZ * sizeof(double));
    for (int64_t t = tb; t < te; ++t)  /* st[i] = state after i tokens */
      forward_step(dk, dv, k + (t * H + h) * dk, log_alpha + (t * H + h) * dk,
                   v + (t * H + h) * dv, beta[t * H + h],
                   st + (size_t)(t - tb) * SZ, st + (size_t)(t - tb + 1) * SZ,
                   Sp, e);
    for (int64_t t = te - 1; t >= tb; --t) {
      const double* kt = k + (t * H + h) * dk;
      const double* qt = q + (t * H + h) * dk;
      const double* lt = log_alpha + (t * H + h) * dk;
      const double* vt = v + (t * H + h) * dv;
      const double* dot = d_out + (t * H + h) * dv;
      const double bt = beta[t * H + h];
      const double* S_prev = st + (size_t)(t - tb) * SZ;
      const double* S_t = st + (size_t)(t - tb + 1) * SZ;
      double* dqt = dq + (t * H + h) * dk;
      double* dkt = dk_g + (t * H + h) * dk;
      double* dvt = dv_g + (t * H + h) * dv;
      double* dlt = dla + (t * H + h) * dk;
      /* S' and e again (the forward step's intermediates) */
      for (int64_t c = 0; c < dk; ++c) {
        const double a = exp(lt[c]);
        for (int64_t j = 0; j < dv; ++j) Sp[c * dv + j] = a * S_prev[c * dv + j];
      }
      for (int64_t j = 0; j < dv; ++j) e[j] = 0.0;
      for (int64_t c = 0; c < dk; ++c)
        for (int64_t j = 0; j < dv; ++j) e[j] += Sp[c * dv + j] * kt[c];
      /* o_t = S_t^T q_t */
      for (int64_t c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int64_t j = 0; j < dv; ++j) {
          acc += S_t[c * dv + j] * dot[j];
          D[c * dv + j] += qt[c] * dot[j];
        }
        dqt[c] = acc;
      }
      /* S_t = S' + k d^T */
      for (int64_t j = 0; j < dv; ++j) dd[j] = 0.0;
      for (int64_t c = 0; c < dk; ++c)
        for (int64_t j = 0; j < dv; ++j) dd[j] += D[c * dv + j] * kt[c];
      for (int64_t c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int64_t j = 0; j < dv; ++j) acc += D[c * dv + j] * bt * (vt[j] - e[j]);
        dkt[c] = acc;
      }
      /* d = beta (v - e) */
      double db = 0.0;
      for (int64_t j = 0; j < dv; ++j) {
        dvt[j] = bt * dd[j];
        db += dd[j] * (vt[j] - e[j]);
        de[j] = -bt * dd[j];
      }
      dbeta[t * H + h] = db;
      /* e = S'^T k: D' = D + k de^T, dk += S' de */
      for (int64_t c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int64_t j = 0; j < dv; ++j) {
          acc += Sp[c * dv + j] * de[j];
          D[c * dv + j] += kt[c] * de[j];
        }
        dkt[c] += acc;
      }
      /* S' = Diag(exp(l)) S_{t-1} */
      for (int64_t c = 0; c < dk; ++c) {
        double acc = 0.0;
        const double a = exp(lt[c]);
        for (int64_t j = 0; j < dv; ++j) {
          acc += D[c * dv + j] * Sp[c * dv + j];
          D[c * dv + j] *= a;
        }
        dlt[c] = acc;
      }
    }
  }
  if (ds_in) memcpy(ds_in, D, SZ * sizeof(double));
  free(ck); free(st); free(D); free(Sp); free(e); free(dd); free(de);
  return 0;
}

int kda_oracle_recurrent_bwd(int64_t n_seqs, const int64_t* seq_offsets,
                             int64_t H, int64_t dk, int64_t dv, const double* q,
                             const double* k, const double* v,
                             const double* log_alpha, const double* beta,
                             const double* state_in, const double* d_out,
                             const double* d_state_out, double* dq, double* dk_g,
                             double* dv_g, double* dlog_alpha, double* dbeta,
                             double* d_state_in) {
  if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !seq_offsets || !q || !k ||
      !v || !log_alpha || !beta || !d_out || !dq || !dk_g || !dv_g ||
      !dlog_alpha || !dbeta)
    return -1;
  for (int64_t s = 0; s < n_seqs; ++s)
    if (seq_offsets[s + 1] < seq_offsets[s]) return -1;
  const int64_t units = n_seqs * H;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t u = 0; u < units; ++u) {
    const int64_t s = u / H, h = u % H;
    const size_t off = (size_t)(s * H + h) * (size_t)(dk * dv);
    bad |= one_sequence_head_bwd(
               seq_offsets[s], seq_offsets[s + 1], h, H, dk, dv, q, k, v,
               log_alpha, beta, state_in ? state_in + off : NULL, d_out,
               d_state_out ? d_state_out + off : NULL, dq, dk_g, dv_g,
               dlog_alpha, dbeta, d_state_in ? d_state_in + off : NULL) != 0;
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
