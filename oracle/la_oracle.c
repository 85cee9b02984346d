/*
 * la_oracle.c -- fp64 CPU oracle for causal Lightning Attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the test suite, the package smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code with the CUDA library.
 *
 * What it computes (plain definitions, fp64 throughout).  Sources are cited
 * by page title and section:
 *   [MX01] "MiniMax-01与Lightning Attention" (metaphor-xennon notes);
 *   [VGX]  "如何理解MiniMax股价创历史新高？拆解国产大模型技术底座" (vergex),
 *          section "Lightning Attention：长上下文为什么突然变得便宜了",
 *          the chunkwise PyTorch sketch.
 *
 *   Quadratic (masked) form.  [MX01] section 2.2 rewrites attention as
 *   phi(Q) (phi(K)^T V) by associativity; the [VGX] sketch keeps an inclusive
 *   lower-triangular mask inside a block (torch's tril(), diagonal included)
 *   and carries every earlier block through the running state.  Summed over
 *   the whole sequence the two terms are
 *
 *       O[b,h,t,:] = sum_{s <= t} (q[b,h,t] . k[b,g(h),s]) v[b,g(h),s,:]
 *
 *   with phi = identity, no normalisation, no decay and no scaling (the [VGX]
 *   sketch leaves normalisation out; the 1/sqrt(d) factor lives in the input
 *   data).  g(h) = floor(h / (Hq/Hkv)) maps a query head to the kv head whose
 *   state it shares (grouped-query attention: [MX01] section 1.1 lists 128
 *   attention heads and 32 kv heads).
 *
 *   Recurrent form.  [MX01] section 4.1 (the "Streaming" row) and the state
 *   update of the [VGX] sketch carry the kv state forward incrementally with
 *   no history kept.  Token by token, for every kv head g: S_g += k_t^T v_t,
 *   then o_{t,h} = q_{t,h} S_g for each query head h of the group (update
 *   first, then read, so the diagonal term s = t is included as in the
 *   masked form).
 *
 *   State.  S[b,g] = K^T V = sum_s k_s^T v_s ([MX01] section 2.2, the kv_sum
 *   einsum over the sequence axis).
 *
 *   Decode step.  One recurrent step applied to a given state: S += k^T v,
 *   then o_h = q_h S.
 *
 * Element storage: every input array is either IEEE fp32 or bfloat16 (the
 * upper 16 bits of an fp32); each element is widened exactly to double before
 * use.  Layouts are contiguous: q,o [B,Hq,N,d]; k,v [B,Hkv,N,d]; S [B,Hkv,d,d]
 * with S[i][j] = sum_s k_s[i] v_s[j].
 *
 * Threads: independent (b, kv head) units are split over POSIX threads; each
 * unit runs sequentially, so results do not depend on the thread count.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_BF16 = 1 };

static double elem(const void *p, int64_t i, int dtype) {
  if (dtype == OR_BF16) {
    uint32_t bits = ((uint32_t)((const uint16_t *)p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return (double)((const float *)p)[i];
}

/* ---- tiny thread pool over an index range ------------------------------ */

typedef void (*unit_fn)(void *ctx, int64_t unit);
typedef struct {
  unit_fn fn;
  void *ctx;
  int64_t begin, end, stride;
} span_arg;

static void *run_span(void *a_) {
  span_arg *a = (span_arg *)a_;
  for (int64_t u = a->begin; u < a->end; u += a->stride) a->fn(a->ctx, u);
  return NULL;
}

static void parallel_units(unit_fn fn, void *ctx, int64_t nunits, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nunits) nthreads = (int)(nunits > 0 ? nunits : 1);
  if (nthreads == 1) {
    for (int64_t u = 0; u < nunits; ++u) fn(ctx, u);
    return;
  }
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
  span_arg *args = (span_arg *)malloc(sizeof(span_arg) * nthreads);
  for (int i = 0; i < nthreads; ++i) {
    args[i].fn = fn;
    args[i].ctx = ctx;
    args[i].begin = i;
    args[i].end = nunits;
    args[i].stride = nthreads;
    pthread_create(&th[i], NULL, run_span, &args[i]);
  }
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  free(th);
  free(args);
}

typedef struct {
  const void *q, *k, *v;
  int dtype, B, Hq, Hkv, d;
  int64_t N;
  const double *S0;
  double *o;
  float *o32;
  double *S;
  const int64_t *rows;
} job;

/* ---- quadratic masked form: one unit = one (b, query head) ------------- */

static void quadratic_unit(void *ctx, int64_t unit) {
  job *J = (job *)ctx;
  const int G = J->Hq / J->Hkv;
  const int64_t b = unit / J->Hq, h = unit % J->Hq, g = h / G;
  const int64_t N = J->N, d = J->d;
  const int64_t qbase = (b * J->Hq + h) * N * d;
  const int64_t kbase = (b * J->Hkv + g) * N * d;
  for (int64_t t = 0; t < N; ++t) {
    double *out = J->o + qbase + t * d;
    for (int64_t j = 0; j < d; ++j) out[j] = 0.0;
    for (int64_t s = 0; s <= t; ++s) { /* causal: s <= t, diagonal included */
      double a = 0.0;
      for (int64_t i = 0; i < d; ++i)
        a += elem(J->q, qbase + t * d + i, J->dtype) * elem(J->k, kbase + s * d + i, J->dtype);
      for (int64_t j = 0; j < d; ++j) out[j] += a * elem(J->v, kbase + s * d + j, J->dtype);
    }
  }
}

int la_oracle_quadratic(const void *q, const void *k, const void *v, int dtype, int B, int Hq,
                        int Hkv, int64_t N, int d, double *o, int nthreads) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0 || Hq % Hkv) return 1;
  job J = {q, k, v, dtype, B, Hq, Hkv, d, N, NULL, o, NULL, NULL, NULL};
  parallel_units(quadratic_unit, &J, (int64_t)B * Hq, nthreads);
  return 0;
}

/* ---- the masked form at selected rows: one unit = one requested row ----- */
/* rows holds triples (b, h, t); out[r*d + j] = O[b,h,t,j].                   */

static void rows_unit(void *ctx, int64_t r) {
  job *J = (job *)ctx;
  const int G = J->Hq / J->Hkv;
  const int64_t b = J->rows[3 * r], h = J->rows[3 * r + 1], t = J->rows[3 * r + 2];
  const int64_t g = h / G, N = J->N, d = J->d;
  const int64_t qbase = (b * J->Hq + h) * N * d;
  const int64_t kbase = (b * J->Hkv + g) * N * d;
  double *out = J->o + r * d;
  for (int64_t j = 0; j < d; ++j) out[j] = 0.0;
  for (int64_t s = 0; s <= t; ++s) {
    double a = 0.0;
    for (int64_t i = 0; i < d; ++i)
      a += elem(J->q, qbase + t * d + i, J->dtype) * elem(J->k, kbase + s * d + i, J->dtype);
    for (int64_t j = 0; j < d; ++j) out[j] += a * elem(J->v, kbase + s * d + j, J->dtype);
  }
}

int la_oracle_rows(const void *q, const void *k, const void *v, int dtype, int B, int Hq, int Hkv,
                   int64_t N, int d, const int64_t *rows, int64_t nrows, double *out,
                   int nthreads) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0 || Hq % Hkv) return 1;
  for (int64_t r = 0; r < nrows; ++r)
    if (rows[3 * r] < 0 || rows[3 * r] >= B || rows[3 * r + 1] < 0 || rows[3 * r + 1] >= Hq ||
        rows[3 * r + 2] < 0 || rows[3 * r + 2] >= N)
      return 2;
  job J = {q, k, v, dtype, B, Hq, Hkv, d, N, NULL, out, NULL, NULL, rows};
  parallel_units(rows_unit, &J, nrows, nthreads);
  return 0;
}

/* ---- recurrent form: one unit = one (b, kv head) with its G query heads - */
/* S0 (nullable) is the initial state, zero when NULL; S receives the final  */
/* state.  Outputs go to o (double) or o32 (float, rounded once from double) */
/* when either is non-NULL.                                                  */

static void recurrent_unit(void *ctx, int64_t unit) {
  job *J = (job *)ctx;
  const int G = J->Hq / J->Hkv;
  const int64_t b = unit / J->Hkv, g = unit % J->Hkv;
  const int64_t N = J->N, d = J->d;
  double *S = J->S + unit * d * d;
  if (J->S0)
    memcpy(S, J->S0 + unit * d * d, sizeof(double) * d * d);
  else
    memset(S, 0, sizeof(double) * d * d);
  const int64_t kbase = (b * J->Hkv + g) * N * d;
  double *kt = (double *)malloc(sizeof(double) * d);
  double *vt = (double *)malloc(sizeof(double) * d);
  double *ot = (double *)malloc(sizeof(double) * d);
  for (int64_t t = 0; t < N; ++t) {
    for (int64_t i = 0; i < d; ++i) {
      kt[i] = elem(J->k, kbase + t * d + i, J->dtype);
      vt[i] = elem(J->v, kbase + t * d + i, J->dtype);
    }
    for (int64_t i = 0; i < d; ++i) /* S += k_t^T v_t */
      for (int64_t j = 0; j < d; ++j) S[i * d + j] += kt[i] * vt[j];
    if (!J->o && !J->o32) continue;
    for (int hh = 0; hh < G; ++hh) { /* o_{t,h} = q_{t,h} S */
      const int64_t h = g * G + hh;
      const int64_t qoff = ((b * J->Hq + h) * N + t) * d;
      for (int64_t j = 0; j < d; ++j) ot[j] = 0.0;
      for (int64_t i = 0; i < d; ++i) {
        const double qi = elem(J->q, qoff + i, J->dtype);
        for (int64_t j = 0; j < d; ++j) ot[j] += qi * S[i * d + j];
      }
      if (J->o)
        for (int64_t j = 0; j < d; ++j) J->o[qoff + j] = ot[j];
      if (J->o32)
        for (int64_t j = 0; j < d; ++j) J->o32[qoff + j] = (float)ot[j];
    }
  }
  free(kt);
  free(vt);
  free(ot);
}

int la_oracle_recurrent(const void *q, const void *k, const void *v, int dtype, int B, int Hq,
                        int Hkv, int64_t N, int d, const double *S0, double *o, float *o32,
                        double *S, int nthreads) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0 || Hq % Hkv || !S) return 1;
  job J = {q, k, v, dtype, B, Hq, Hkv, d, N, S0, o, o32, S, NULL};
  parallel_units(recurrent_unit, &J, (int64_t)B * Hkv, nthreads);
  return 0;
}

/* ---- state only: S[b,g] = K^T V, one unit = one (b, kv head) ----------- */

static void state_unit(void *ctx, int64_t unit) {
  job *J = (job *)ctx;
  const int64_t N = J->N, d = J->d;
  const int64_t kbase = unit * N * d;
  double *S = J->S + unit * d * d;
  memset(S, 0, sizeof(double) * d * d);
  for (int64_t s = 0; s < N; ++s)
    for (int64_t i = 0; i < d; ++i) {
      const double ki = elem(J->k, kbase + s * d + i, J->dtype);
      for (int64_t j = 0; j < d; ++j) S[i * d + j] += ki * elem(J->v, kbase + s * d + j, J->dtype);
    }
}

int la_oracle_state(const void *k, const void *v, int dtype, int B, int Hkv, int64_t N, int d,
                    double *S, int nthreads) {
  if (B <= 0 || Hkv <= 0 || N < 0 || d <= 0 || !S) return 1;
  job J = {NULL, k, v, dtype, B, Hkv, Hkv, d, N, NULL, NULL, NULL, S, NULL};
  parallel_units(state_unit, &J, (int64_t)B * Hkv, nthreads);
  return 0;
}

/* ---- decode step: S (in/out, [B,Hkv,d,d]) += k^T v; o_h = q_h S -------- */
/* q,o [B,Hq,d]; k,v [B,Hkv,d].  One unit = one (b, kv head).                */

typedef struct {
  double *S;
  const void *q, *k, *v;
  int dtype, Hq, Hkv, d;
  double *o;
} decode_job;

static void decode_unit(void *ctx, int64_t unit) {
  decode_job *J = (decode_job *)ctx;
  const int G = J->Hq / J->Hkv;
  const int64_t b = unit / J->Hkv, g = unit % J->Hkv, d = J->d;
  double *Sg = J->S + unit * d * d;
  const int64_t kv = unit * d;
  for (int64_t i = 0; i < d; ++i) { /* S += k^T v */
    const double ki = elem(J->k, kv + i, J->dtype);
    for (int64_t j = 0; j < d; ++j) Sg[i * d + j] += ki * elem(J->v, kv + j, J->dtype);
  }
  for (int hh = 0; hh < G; ++hh) { /* o_h = q_h S */
    const int64_t qo = (b * J->Hq + g * G + hh) * d;
    for (int64_t j = 0; j < d; ++j) J->o[qo + j] = 0.0;
    for (int64_t i = 0; i < d; ++i) {
      const double qi = elem(J->q, qo + i, J->dtype);
      for (int64_t j = 0; j < d; ++j) J->o[qo + j] += qi * Sg[i * d + j];
    }
  }
}

int la_oracle_decode(double *S, const void *q, const void *k, const void *v, int dtype, int B,
                     int Hq, int Hkv, int d, double *o, int nthreads) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv || !S || !o) return 1;
  decode_job J = {S, q, k, v, dtype, Hq, Hkv, d, o};
  parallel_units(decode_unit, &J, (int64_t)B * Hkv, nthreads);
  return 0;
}

/* ---- backward ----------------------------------------------------------
 * Gradients of the prefill (fp64) for a loss whose gradient with respect to
 * O is dO and with respect to the final state is dSf (nullable = 0).  From
 * o_t = q_t S_t and S_t = S0 + sum_{s<=t} k_s^T v_s:
 *   dq_t  = do_t S0^T + sum_{s<=t} (do_t . v_s) k_s
 *   dk_s  = sum_{h in g} sum_{t>=s} (v_s . do_{t,h}) q_{t,h} + v_s dSf^T
 *   dv_s  = sum_{h in g} sum_{t>=s} (k_s . q_{t,h}) do_{t,h} + k_s dSf
 *   dS0   = dSf + sum_{h in g} sum_t q_{t,h}^T do_{t,h}
 * Quadratic form: these sums written out.  Recurrent form: a forward sweep for
 * dq (S_t as in the forward recurrence) and a reverse sweep for dk, dv with
 * G_s = dSf + sum_{h} sum_{t>=s} q_{t,h}^T do_{t,h} (update, then read).
 * Layouts as the forward; do, dq [B,Hq,N,d]; dk, dv [B,Hkv,N,d]; S0, dSf,
 * dS0 [B,Hkv,d,d].  Outputs are double.  One unit = one (b, kv head). */

typedef struct {
  const void *q, *k, *v, *dO;
  int dtype, B, Hq, Hkv, d;
  int64_t N;
  const double *S0, *dSf;
  double *dq, *dk, *dv, *dS0;
} bwd_job;

static void backward_quadratic_unit(void *ctx, int64_t unit) {
  bwd_job *J = (bwd_job *)ctx;
  const int G = J->Hq / J->Hkv;
  const int64_t b = unit / J->Hkv, g = unit % J->Hkv, N = J->N, d = J->d;
  const int64_t kb = (b * J->Hkv + g) * N * d;
  const double *S0 = J->S0 ? J->S0 + unit * d * d : NULL;
  const double *dSf = J->dSf ? J->dSf + unit * d * d : NULL;
  for (int hh = 0; hh < G; ++hh) { /* dq of every query head of the group */
    const int64_t qb = (b * J->Hq + g * G + hh) * N * d;
    for (int64_t t = 0; t < N; ++t) {
      double *out = J->dq + qb + t * d;
      for (int64_t i = 0; i < d; ++i) {
        double a = 0.0;
        if (S0)
          for (int64_t j = 0; j < d; ++j) a += elem(J->dO, qb + t * d + j, J->dtype) * S0[i * d + j];
        out[i] = a;
      }
      for (int64_t s = 0; s <= t; ++s) {
        double a = 0.0;
        for (int64_t j = 0; j < d; ++j)
          a += elem(J->dO, qb + t * d + j, J->dtype) * elem(J->v, kb + s * d + j, J->dtype);
        for (int64_t i = 0; i < d; ++i) out[i] += a * elem(J->k, kb + s * d + i, J->dtype);
      }
    }
  }
  for (int64_t s = 0; s < N; ++s) { /* dk, dv */
    double *dk = J->dk + kb + s * d, *dv = J->dv + kb + s * d;
    for (int64_t i = 0; i < d; ++i) {
      double a = 0.0, c = 0.0;
      if (dSf)
        for (int64_t j = 0; j < d; ++j) {
          a += elem(J->v, kb + s * d + j, J->dtype) * dSf[i * d + j]; /* (v dSf^T)_i */
          c += elem(J->k, kb + s * d + j, J->dtype) * dSf[j * d + i]; /* (k dSf)_i */
        }
      dk[i] = a;
      dv[i] = c;
    }
    for (int hh = 0; hh < G; ++hh) {
      const int64_t qb = (b * J->Hq + g * G + hh) * N * d;
      for (int64_t t = s; t < N; ++t) {
        double vd = 0.0, kq = 0.0;
        for (int64_t j = 0; j < d; ++j) {
          vd += elem(J->v, kb + s * d + j, J->dtype) * elem(J->dO, qb + t * d + j, J->dtype);
          kq += elem(J->k, kb + s * d + j, J->dtype) * elem(J->q, qb + t * d + j, J->dtype);
        }
        for (int64_t i = 0; i < d; ++i) {
          dk[i] += vd * elem(J->q, qb + t * d + i, J->dtype);
          dv[i] += kq * elem(J->dO, qb + t * d + i, J->dtype);
        }
      }
    }
  }
  if (J->dS0) {
    double *o = J->dS0 + unit * d * d;
    for (int64_t e = 0; e < d * d; ++e) o[e] = dSf ? dSf[e] : 0.0;
    for (int hh = 0; hh < G; ++hh) {
      const int64_t qb = (b * J->Hq + g * G + hh) * N * d;
      for (int64_t t = 0; t < N; ++t)
        for (int64_t i = 0; i < d; ++i) {
          const double qi = elem(J->q, qb + t * d + i, J->dtype);
          for (int64_t j = 0; j < d; ++j) o[i * d + j] += qi * elem(J->dO, qb + t * d + j, J->dtype);
        }
    }
  }
}

static void backward_recurrent_unit(void *ctx, int64_t unit) {
  bwd_job *J = (bwd_job *)ctx;
  const int G = J->Hq / J->Hkv;
  const int64_t b = unit / J->Hkv, g = unit % J->Hkv, N = J->N, d = J->d;
  const int64_t kb = (b * J->Hkv + g) * N * d;
  double *St = (double *)malloc(sizeof(double) * d * d);
  double *kt = (double *)malloc(sizeof(double) * d);
  double *vt = (double *)malloc(sizeof(double) * d);
  /* forward sweep: S_t, dq_t = do_t S_t^T */
  if (J->S0)
    memcpy(St, J->S0 + unit * d * d, sizeof(double) * d * d);
  else
    memset(St, 0, sizeof(double) * d * d);
  for (int64_t t = 0; t < N; ++t) {
    for (int64_t i = 0; i < d; ++i) {
      kt[i] = elem(J->k, kb + t * d + i, J->dtype);
      vt[i] = elem(J->v, kb + t * d + i, J->dtype);
    }
    for (int64_t i = 0; i < d; ++i)
      for (int64_t j = 0; j < d; ++j) St[i * d + j] += kt[i] * vt[j];
    for (int hh = 0; hh < G; ++hh) {
      const int64_t qo = (b * J->Hq + g * G + hh) * N * d + t * d;
      for (int64_t i = 0; i < d; ++i) {
        double a = 0.0;
        for (int64_t j = 0; j < d; ++j) a += elem(J->dO, qo + j, J->dtype) * St[i * d + j];
        J->dq[qo + i] = a;
      }
    }
  }
  /* reverse sweep: G_s += sum_h q_{s,h}^T do_{s,h}; dk_s = v_s G_s^T; dv_s = k_s G_s */
  if (J->dSf)
    memcpy(St, J->dSf + unit * d * d, sizeof(double) * d * d);
  else
    memset(St, 0, sizeof(double) * d * d);
  for (int64_t s = N - 1; s >= 0; --s) {
    for (int hh = 0; hh < G; ++hh) {
      const int64_t qo = (b * J->Hq + g * G + hh) * N * d + s * d;
      for (int64_t i = 0; i < d; ++i) {
        const double qi = elem(J->q, qo + i, J->dtype);
        for (int64_t j = 0; j < d; ++j) St[i * d + j] += qi * elem(J->dO, qo + j, J->dtype);
      }
    }
    for (int64_t i = 0; i < d; ++i) {
      kt[i] = elem(J->k, kb + s * d + i, J->dtype);
      vt[i] = elem(J->v, kb + s * d + i, J->dtype);
    }
    for (int64_t i = 0; i < d; ++i) {
      double a = 0.0, c = 0.0;
      for (int64_t j = 0; j < d; ++j) {
        a += vt[j] * St[i * d + j]; /* (v G^T)_i */
        c += kt[j] * St[j * d + i]; /* (k G)_i */
      }
      J->dk[kb + s * d + i] = a;
      J->dv[kb + s * d + i] = c;
    }
  }
  if (J->dS0) memcpy(J->dS0 + unit * d * d, St, sizeof(double) * d * d);
  free(St);
  free(kt);
  free(vt);
}

static int backward(unit_fn fn, const void *q, const void *k, const void *v, const void *dO,
                    int dtype, int B, int Hq, int Hkv, int64_t N, int d, const double *S0,
                    const double *dSf, double *dq, double *dk, double *dv, double *dS0,
                    int nthreads) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0 || Hq % Hkv || !dq || !dk || !dv) return 1;
  bwd_job J = {q, k, v, dO, dtype, B, Hq, Hkv, d, N, S0, dSf, dq, dk, dv, dS0};
  parallel_units(fn, &J, (int64_t)B * Hkv, nthreads);
  return 0;
}

int la_oracle_backward_quadratic(const void *q, const void *k, const void *v, const void *dO,
                                 int dtype, int B, int Hq, int Hkv, int64_t N, int d,
                                 const double *S0, const double *dSf, double *dq, double *dk,
                                 double *dv, double *dS0, int nthreads) {
  return backward(backward_quadratic_unit, q, k, v, dO, dtype, B, Hq, Hkv, N, d, S0, dSf, dq, dk,
                  dv, dS0, nthreads);
}

int la_oracle_backward_recurrent(const void *q, const void *k, const void *v, const void *dO,
                                 int dtype, int B, int Hq, int Hkv, int64_t N, int d,
                                 const double *S0, const double *dSf, double *dq, double *dk,
                                 double *dv, double *dS0, int nthreads) {
  return backward(backward_recurrent_unit, q, k, v, dO, dtype, B, Hq, Hkv, N, d, S0, dSf, dq, dk,
                  dv, dS0, nthreads);
}
