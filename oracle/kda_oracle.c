/*
 * kda_oracle.c -- fp64 CPU oracle for Kimi Delta Attention (KDA) prefill and the
 * context-parallel segment summary / exclusive scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark may load this library.  It shares no code, header or constant with the
 * CUDA library and must never be used as a fallback for it.
 *
 * Everything here is the plain definition, one token at a time, in double precision:
 *
 *   gate       g_i   = -exp(a_log[h]) * softplus(raw_gate[t,h,i] + dt_bias[h,i])
 *              ("max.nn.state_space.kda_chunk", Parameters: raw_gate is the forget-gate
 *              pre-activation before dt_bias is added; a_log and dt_bias per value head).
 *              "safe" gate mode: g_i = max(g_i, lower_bound)  (the docs name a lower bound,
 *              KDA_GATE_LOWER_BOUND, without giving its form; a clamp is the reading taken).
 *   beta       beta  = sigmoid(beta_logits[t,h])  or taken as given in "probability" mode
 *              (kda_chunk, Parameters: beta_mode).
 *   step       S <- Diag(exp(g)) S                      (per-channel decay of key rows)
 *              pred  = k^T S                            (prediction from the DECAYED state)
 *              S <- S + k (beta (v - pred))^T           (delta-rule write: overwrites along k)
 *              o     = q^T S                            (readout AFTER the write)
 *              ("nx_nofloat_kda.nx source": header comments of the file, kda_gate, kda_write,
 *              kda_forward -- gate, then delta write, then read, per token).
 *   heads      key head of value head h is h / (Hv/Hk)   (contiguous groups; reading).
 *   pool       state of sequence b lives in state_pool[state_indices[b], h], read as the
 *              initial state and written back as the final state (kda_chunk: state_pool is a
 *              mutable pool, state_indices gives the slot per sequence).  K_FIRST stores
 *              S as [dk][dv]; V_FIRST stores S^T as [dv][dk] (kda_chunk: state_layout).
 *
 * Segment summary ("KDA Context Parallelism", Theory):
 *   M_i = the segment's transition: the recurrence run from S = I (dk x dk) with all v = 0.
 *   U_i = the segment's local contribution: the recurrence run from S = 0 with the real v.
 *   Both are obtained by replaying the segment's tokens, by definition, not from any algebra.
 * Exclusive scan ("KDA Context Parallelism", Incoming and outgoing states / Implementation
 * order): in_0 = S_initial; out_i = M_i in_i + U_i; in_{i+1} = out_i; final = out_{N-1}.
 * Composition ("KDA Context Parallelism", Compose segments in sequence order):
 *   (M2,U2) o (M1,U1) = (M2 M1, M2 U1 + U2).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_GATE_SAFE 1u
#define ORACLE_BETA_PROB 2u
#define ORACLE_V_FIRST 4u

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_BAD_SLOT 2
#define ORACLE_BAD_SEQLENS 3

static double oracle_softplus(double x) {
  /* log(1 + e^x), written so neither branch overflows */
  return fmax(x, 0.0) + log1p(exp(-fabs(x)));
}

static double oracle_sigmoid(double x) {
  if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
  double e = exp(x);
  return e / (1.0 + e);
}

double kda_oracle_gate(double raw, double a_log, double dt_bias, uint32_t flags, double lower_bound) {
  double g = -exp(a_log) * oracle_softplus(raw + dt_bias);
  if ((flags & ORACLE_GATE_SAFE) && g < lower_bound) g = lower_bound;
  return g;
}

double kda_oracle_beta(double logit, uint32_t flags) {
  return (flags & ORACLE_BETA_PROB) ? logit : oracle_sigmoid(logit);
}

/*
 * One token on a dk x dw state S (row-major [dk][dw]).  v may be NULL (all-zero values,
 * used for the transition M).  o may be NULL (no readout).  pred is dw doubles of scratch.
 */
static void oracle_token_step(double *S, int dk, int dw, const double *q, const double *k,
                              const double *v, const double *g, double beta, double *o,
                              double *pred) {
  for (int i = 0; i < dk; ++i) {
    double a = exp(g[i]);
    for (int j = 0; j < dw; ++j) S[(size_t)i * dw + j] *= a;
  }
  for (int j = 0; j < dw; ++j) {
    double acc = 0.0;
    for (int i = 0; i < dk; ++i) acc += k[i] * S[(size_t)i * dw + j];
    pred[j] = acc;
  }
  for (int i = 0; i < dk; ++i) {
    for (int j = 0; j < dw; ++j) {
      double vj = v ? v[j] : 0.0;
      S[(size_t)i * dw + j] += k[i] * (beta * (vj - pred[j]));
    }
  }
  if (o) {
    for (int j = 0; j < dw; ++j) {
      double acc = 0.0;
      for (int i = 0; i < dk; ++i) acc += q[i] * S[(size_t)i * dw + j];
      o[j] = acc;
    }
  }
}

/* load / store one pool block into a row-major [dk][dv] working state */
static void oracle_load_state(double *S, const double *blk, int dk, int dv, int v_first) {
  for (int i = 0; i < dk; ++i)
    for (int j = 0; j < dv; ++j)
      S[(size_t)i * dv + j] = v_first ? blk[(size_t)j * dk + i] : blk[(size_t)i * dv + j];
}

static void oracle_store_state(double *blk, const double *S, int dk, int dv, int v_first) {
  for (int i = 0; i < dk; ++i)
    for (int j = 0; j < dv; ++j) {
      if (v_first) blk[(size_t)j * dk + i] = S[(size_t)i * dv + j];
      else blk[(size_t)i * dv + j] = S[(size_t)i * dv + j];
    }
}

/*
 * Full prefill over a varlen batch.
 *   q,k [T,Hk,dk]; v [T,Hv,dv]; raw_gate [T,Hv,dk]; beta_in [T,Hv]; a_log [Hv];
 *   dt_bias [Hv,dk]; cu_seqlens [batch+1]; state_pool [max_slots,Hv,dk,dv] (or V_FIRST);
 *   state_indices [batch]; out [T,Hv,dv] (may be NULL).
 * Returns ORACLE_OK, or an error code (nothing is written for a bad slot / bad offsets of
 * that sequence; other sequences still run).
 */
int kda_oracle_forward(const double *q, const double *k, const double *v, const double *raw_gate,
                       const double *beta_in, const double *a_log, const double *dt_bias,
                       const int32_t *cu_seqlens, int32_t batch, int64_t total_tokens, int32_t Hk,
                       int32_t Hv, int32_t dk, int32_t dv, double *state_pool, int32_t max_slots,
                       const int32_t *state_indices, double *out, uint32_t flags,
                       double lower_bound) {
  if (batch < 0 || Hk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0 || Hv % Hk != 0) return ORACLE_BAD_ARG;
  const int group = Hv / Hk;
  const int v_first = (flags & ORACLE_V_FIRST) ? 1 : 0;
  int status = ORACLE_OK;
  const int64_t pairs = (int64_t)batch * Hv;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t p = 0; p < pairs; ++p) {
    const int b = (int)(p / Hv), h = (int)(p % Hv), kh = h / group;
    const int64_t t0 = cu_seqlens[b], t1 = cu_seqlens[b + 1];
    const int32_t slot = state_indices ? state_indices[b] : b;
    if (slot < 0 || slot >= max_slots) {
#pragma omp critical
      status = ORACLE_BAD_SLOT;
      continue;
    }
    if (t0 < 0 || t1 < t0 || t1 > total_tokens) {
#pragma omp critical
      status = ORACLE_BAD_SEQLENS;
      continue;
    }
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *pred = (double *)malloc(sizeof(double) * (size_t)dv);
    double *g = (double *)malloc(sizeof(double) * (size_t)dk);
    double *blk = state_pool + ((size_t)slot * Hv + h) * (size_t)dk * dv;
    oracle_load_state(S, blk, dk, dv, v_first);
    for (int64_t t = t0; t < t1; ++t) {
      const double *qt = q + ((size_t)t * Hk + kh) * dk;
      const double *kt = k + ((size_t)t * Hk + kh) * dk;
      const double *vt = v + ((size_t)t * Hv + h) * dv;
      const double *rt = raw_gate + ((size_t)t * Hv + h) * dk;
      for (int i = 0; i < dk; ++i)
        g[i] = kda_oracle_gate(rt[i], a_log[h], dt_bias[(size_t)h * dk + i], flags, lower_bound);
      double beta = kda_oracle_beta(beta_in[(size_t)t * Hv + h], flags);
      double *ot = out ? out + ((size_t)t * Hv + h) * dv : NULL;
      oracle_token_step(S, dk, dv, qt, kt, vt, g, beta, ot, pred);
    }
    oracle_store_state(blk, S, dk, dv, v_first);
    free(S);
    free(pred);
    free(g);
  }
  return status;
}

/*
 * Segment summaries of one sequence split at seg_offsets [N+1]:
 *   M [N,Hv,dk,dk]  (row-major, M_i left-multiplies the state: F_i(S) = M_i S + U_i)
 *   U [N,Hv,dk,dv]  (K_FIRST) or [N,Hv,dv,dk] (V_FIRST, stored transposed like a pool slot)
 * M_i: recurrence from S = I with zero values.  U_i: recurrence from S = 0 with real values.
 */
int kda_oracle_segment_summary(const double *k, const double *v, const double *raw_gate,
                               const double *beta_in, const double *a_log, const double *dt_bias,
                               int64_t total_tokens, int32_t Hk, int32_t Hv, int32_t dk,
                               int32_t dv, const int32_t *seg_offsets, int32_t num_segments,
                               double *M, double *U, uint32_t flags, double lower_bound) {
  if (num_segments < 1 || Hk <= 0 || Hv <= 0 || Hv % Hk != 0 || dk <= 0 || dv <= 0) return ORACLE_BAD_ARG;
  for (int i = 0; i < num_segments; ++i)
    if (seg_offsets[i] < 0 || seg_offsets[i + 1] < seg_offsets[i] || seg_offsets[i + 1] > total_tokens)
      return ORACLE_BAD_SEQLENS;
  const int group = Hv / Hk;
  const int v_first = (flags & ORACLE_V_FIRST) ? 1 : 0;
  const int64_t pairs = (int64_t)num_segments * Hv;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t p = 0; p < pairs; ++p) {
    const int s = (int)(p / Hv), h = (int)(p % Hv), kh = h / group;
    double *Sm = (double *)malloc(sizeof(double) * (size_t)dk * dk);
    double *Su = (double *)calloc((size_t)dk * dv, sizeof(double));
    double *pred = (double *)malloc(sizeof(double) * (size_t)(dk > dv ? dk : dv));
    double *g = (double *)malloc(sizeof(double) * (size_t)dk);
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < dk; ++j) Sm[(size_t)i * dk + j] = (i == j) ? 1.0 : 0.0;
    for (int64_t t = seg_offsets[s]; t < seg_offsets[s + 1]; ++t) {
      const double *kt = k + ((size_t)t * Hk + kh) * dk;
      const double *vt = v + ((size_t)t * Hv + h) * dv;
      const double *rt = raw_gate + ((size_t)t * Hv + h) * dk;
      for (int i = 0; i < dk; ++i)
        g[i] = kda_oracle_gate(rt[i], a_log[h], dt_bias[(size_t)h * dk + i], flags, lower_bound);
      double beta = kda_oracle_beta(beta_in[(size_t)t * Hv + h], flags);
      oracle_token_step(Sm, dk, dk, NULL, kt, NULL, g, beta, NULL, pred);
      oracle_token_step(Su, dk, dv, NULL, kt, vt, g, beta, NULL, pred);
    }
    memcpy(M + ((size_t)s * Hv + h) * (size_t)dk * dk, Sm, sizeof(double) * (size_t)dk * dk);
    oracle_store_state(U + ((size_t)s * Hv + h) * (size_t)dk * dv, Su, dk, dv, v_first);
    free(Sm);
    free(Su);
    free(pred);
    free(g);
  }
  return ORACLE_OK;
}

/* C = A (n x m) * B (m x p), all row-major */
static void oracle_matmul(const double *A, const double *B, double *C, int n, int m, int p) {
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < p; ++j) {
      double acc = 0.0;
      for (int l = 0; l < m; ++l) acc += A[(size_t)i * m + l] * B[(size_t)l * p + j];
      C[(size_t)i * p + j] = acc;
    }
}

/*
 * Ordered composition of two affine maps, later map first in the argument list:
 *   (M2,U2) o (M1,U1) = (M2 M1, M2 U1 + U2).   Mo is dk x dk, Uo is dk x dv (row-major).
 */
void kda_oracle_compose(const double *M2, const double *U2, const double *M1, const double *U1,
                        int32_t dk, int32_t dv, double *Mo, double *Uo) {
  oracle_matmul(M2, M1, Mo, dk, dk, dk);
  oracle_matmul(M2, U1, Uo, dk, dk, dv);
  for (size_t e = 0; e < (size_t)dk * dv; ++e) Uo[e] += U2[e];
}

/*
 * Exclusive scan over N segments for every head.
 *   M [N,H,dk,dk]; U, incoming, outgoing [N,H,<state>]; initial, final [H,<state>], where
 *   <state> is [dk][dv] (K_FIRST) or [dv][dk] (V_FIRST).  incoming/outgoing/final may be
 *   NULL.  Inputs are never written.
 */
int kda_oracle_affine_scan(const double *M, const double *U, const double *initial,
                           int32_t num_segments, int32_t H, int32_t dk, int32_t dv, uint32_t flags,
                           double *incoming, double *outgoing, double *final_state) {
  if (num_segments < 1 || H <= 0 || dk <= 0 || dv <= 0) return ORACLE_BAD_ARG;
  const int v_first = (flags & ORACLE_V_FIRST) ? 1 : 0;
  const size_t st = (size_t)dk * dv;
#pragma omp parallel for schedule(dynamic, 1)
  for (int h = 0; h < H; ++h) {
    double *cur = (double *)malloc(sizeof(double) * st);
    double *nxt = (double *)malloc(sizeof(double) * st);
    double *u = (double *)malloc(sizeof(double) * st);
    oracle_load_state(cur, initial + (size_t)h * st, dk, dv, v_first);
    for (int i = 0; i < num_segments; ++i) {
      if (incoming) oracle_store_state(incoming + ((size_t)i * H + h) * st, cur, dk, dv, v_first);
      const double *Mi = M + ((size_t)i * H + h) * (size_t)dk * dk;
      oracle_load_state(u, U + ((size_t)i * H + h) * st, dk, dv, v_first);
      oracle_matmul(Mi, cur, nxt, dk, dk, dv);
      for (size_t e = 0; e < st; ++e) nxt[e] += u[e];
      if (outgoing) oracle_store_state(outgoing + ((size_t)i * H + h) * st, nxt, dk, dv, v_first);
      double *tmp = cur;
      cur = nxt;
      nxt = tmp;
    }
    if (final_state) oracle_store_state(final_state + (size_t)h * st, cur, dk, dv, v_first);
    free(cur);
    free(nxt);
    free(u);
  }
  return ORACLE_OK;
}

int kda_oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
