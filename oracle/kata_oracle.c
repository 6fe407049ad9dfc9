/*
 * kata_oracle.c -- plain, slow, fp64 CPU oracle for the KATA forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the CPU-baseline leg of the benchmark may load this library.  It shares no
 * code, header, table or helper with the CUDA path, and it never calls it.
 *
 * What it computes (one (batch b, head h) pair at a time, q_t,k_t in R^p,
 * v_t in R^dv, t = 1..T):
 *
 *   psi(u) = vec(u u^T)                       rank-one PSD feature map
 *       -- gist.science technical summary of arXiv:2607.17419, sec. 2.2
 *          ("PSD Kegel (Rank-One)"): the map squares the raw inner product;
 *          ai.info summary, Main Findings ("Squaring the inner product
 *          changes the geometry").
 *   w_{t,s} = <psi(q_t), psi(k_s)> = (q_t . k_s)^2 >= 0
 *   N_t = sum_{s<=t} w_{t,s} v_s,   D_t = sum_{s<=t} w_{t,s},   o_t = N_t / D_t
 *       -- normalized linear attention whose denominator is the
 *          parameter-free convex output gate (gist.science sec. 2.1, "Output
 *          Gating"; ai.info Main Findings, "The readout gate is free").
 *
 * Two independent evaluations are provided, so that each can be checked
 * against the other:
 *   kata_oracle_direct     -- the defining double sum, O(T^2 (p + dv)).
 *   kata_oracle_recurrent  -- the explicit state recurrence on the fixed-size
 *                             state (ai.info, Methodology in Plain English: the
 *                             feature inner product turns token mixing into a
 *                             recurrence on a fixed-size state):
 *                               S_t = S_{t-1} + psi(k_t) v_t^T   (p^2 x dv)
 *                               z_t = z_{t-1} + psi(k_t)         (p^2)
 *                               o_t = psi(q_t)^T S_t / psi(q_t)^T z_t
 *                             with psi materialised as an explicit p^2 vector.
 *
 * Readings of points the pages leave open:
 *   - the causal sum includes s = t (the gate weight beta_t = c_t / D_t uses
 *     the current token's own score, ai.info Main Findings);
 *   - D_t = 0 gives o_t = 0 (the pages print no epsilon anywhere);
 *   - no 1/sqrt(d) or temperature scaling of q.k (none is printed);
 *   - q and k are used as given (no normalisation inside the operation).
 *
 * Layouts: row-major contiguous q,k [B,H,T,p], v,o [B,H,T,dv],
 * S [B,H,p*p,dv] with psi index r = i*p + j, z [B,H,p*p].  All doubles.
 *
 * Threads: work is split over (b,h) pairs with pthreads; nthreads <= 0 means
 * one thread per online CPU.  Every (b,h) pair is computed by exactly one
 * thread with a fixed summation order, so results do not depend on nthreads.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define KATA_ORACLE_OK 0
#define KATA_ORACLE_EINVAL 1
#define KATA_ORACLE_ENOMEM 2

/* ------------------------------------------------------------------------ */
/* thread pool over (b,h) pairs                                              */
/* ------------------------------------------------------------------------ */

typedef void (*pair_fn)(void *ctx, int64_t bh);

typedef struct {
  pair_fn fn;
  void *ctx;
  int64_t n;
  int64_t next;
  pthread_mutex_t lock;
} pair_pool;

static void *pair_worker(void *arg) {
  pair_pool *pool = (pair_pool *)arg;
  for (;;) {
    pthread_mutex_lock(&pool->lock);
    int64_t bh = pool->next++;
    pthread_mutex_unlock(&pool->lock);
    if (bh >= pool->n) break;
    pool->fn(pool->ctx, bh);
  }
  return NULL;
}

static int run_pairs(pair_fn fn, void *ctx, int64_t n, int nthreads) {
  if (nthreads <= 0) {
    long c = sysconf(_SC_NPROCESSORS_ONLN);
    nthreads = c > 0 ? (int)c : 1;
  }
  if (nthreads > n) nthreads = (int)(n > 0 ? n : 1);
  pair_pool pool;
  pool.fn = fn;
  pool.ctx = ctx;
  pool.n = n;
  pool.next = 0;
  pthread_mutex_init(&pool.lock, NULL);
  if (nthreads == 1) {
    pair_worker(&pool);
  } else {
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) {
      pthread_mutex_destroy(&pool.lock);
      return KATA_ORACLE_ENOMEM;
    }
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, pair_worker, &pool);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
  }
  pthread_mutex_destroy(&pool.lock);
  return KATA_ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* direct form: the defining double sum                                      */
/* ------------------------------------------------------------------------ */

typedef struct {
  const double *q, *k, *v;
  double *o;
  int64_t T;
  int p, dv;
} direct_ctx;

/* o_t for one query row: accumulate N and D over s = 0..t in increasing s. */
static void direct_row(const double *q_t, const double *k, const double *v,
                       int64_t t, int p, int dv, double *N, double *o_t) {
  double D = 0.0;
  for (int e = 0; e < dv; ++e) N[e] = 0.0;
  for (int64_t s = 0; s <= t; ++s) {
    const double *k_s = k + s * p;
    double dot = 0.0;
    for (int i = 0; i < p; ++i) dot += q_t[i] * k_s[i];
    double w = dot * dot; /* (q_t . k_s)^2 */
    D += w;
    const double *v_s = v + s * dv;
    for (int e = 0; e < dv; ++e) N[e] += w * v_s[e];
  }
  for (int e = 0; e < dv; ++e) o_t[e] = (D > 0.0) ? N[e] / D : 0.0;
}

static void direct_pair(void *vctx, int64_t bh) {
  direct_ctx *c = (direct_ctx *)vctx;
  const double *q = c->q + bh * c->T * c->p;
  const double *k = c->k + bh * c->T * c->p;
  const double *v = c->v + bh * c->T * c->dv;
  double *o = c->o + bh * c->T * c->dv;
  double *N = (double *)malloc(sizeof(double) * (size_t)c->dv);
  if (!N) return;
  for (int64_t t = 0; t < c->T; ++t) direct_row(q + t * c->p, k, v, t, c->p, c->dv, N, o + t * c->dv);
  free(N);
}

int kata_oracle_direct(const double *q, const double *k, const double *v, double *o,
                       int64_t B, int64_t H, int64_t T, int p, int dv, int nthreads) {
  if (!q || !k || !v || !o || B < 0 || H < 0 || T < 0 || p <= 0 || dv <= 0) return KATA_ORACLE_EINVAL;
  direct_ctx c = {q, k, v, o, T, p, dv};
  return run_pairs(direct_pair, &c, B * H, nthreads);
}

/* Direct form on selected rows only: row r is (bh_idx[r], t_idx[r]) and its
 * output goes to o_rows[r*dv ..].  D_t for the row is written to d_rows[r]
 * when d_rows is non-NULL.  Cost O(t (p + dv)) per row, for sampling outputs
 * of long sequences. */
int kata_oracle_direct_rows(const double *q, const double *k, const double *v,
                            int64_t BH, int64_t T, int p, int dv,
                            const int64_t *bh_idx, const int64_t *t_idx, int64_t nrows,
                            double *o_rows, double *d_rows) {
  if (!q || !k || !v || !bh_idx || !t_idx || !o_rows || p <= 0 || dv <= 0) return KATA_ORACLE_EINVAL;
  double *N = (double *)malloc(sizeof(double) * (size_t)dv);
  if (!N) return KATA_ORACLE_ENOMEM;
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t bh = bh_idx[r], t = t_idx[r];
    if (bh < 0 || bh >= BH || t < 0 || t >= T) {
      free(N);
      return KATA_ORACLE_EINVAL;
    }
    const double *qb = q + bh * T * p, *kb = k + bh * T * p, *vb = v + bh * T * dv;
    direct_row(qb + t * p, kb, vb, t, p, dv, N, o_rows + r * dv);
    if (d_rows) {
      double D = 0.0;
      for (int64_t s = 0; s <= t; ++s) {
        double dot = 0.0;
        for (int i = 0; i < p; ++i) dot += qb[t * p + i] * kb[s * p + i];
        D += dot * dot;
      }
      d_rows[r] = D;
    }
  }
  free(N);
  return KATA_ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* recurrent form: explicit psi and state                                    */
/* ------------------------------------------------------------------------ */

typedef struct {
  const double *q, *k, *v;
  double *o;
  int64_t T;
  int p, dv;
  const double *S0, *z0; /* may be NULL: zero initial state */
  double *S_out, *z_out; /* may be NULL */
} recur_ctx;

/* psi(u) = vec(u u^T), index r = i*p + j. */
static void psi(const double *u, int p, double *out) {
  for (int i = 0; i < p; ++i)
    for (int j = 0; j < p; ++j) out[i * p + j] = u[i] * u[j];
}

static void recur_pair(void *vctx, int64_t bh) {
  recur_ctx *c = (recur_ctx *)vctx;
  const int p = c->p, dv = c->dv;
  const int64_t P = (int64_t)p * p, T = c->T;
  double *S = (double *)malloc(sizeof(double) * (size_t)(P * dv));
  double *z = (double *)malloc(sizeof(double) * (size_t)P);
  double *pk = (double *)malloc(sizeof(double) * (size_t)P);
  double *pq = (double *)malloc(sizeof(double) * (size_t)P);
  double *num = (double *)malloc(sizeof(double) * (size_t)dv);
  if (!S || !z || !pk || !pq || !num) goto done;
  if (c->S0) memcpy(S, c->S0 + bh * P * dv, sizeof(double) * (size_t)(P * dv));
  else memset(S, 0, sizeof(double) * (size_t)(P * dv));
  if (c->z0) memcpy(z, c->z0 + bh * P, sizeof(double) * (size_t)P);
  else memset(z, 0, sizeof(double) * (size_t)P);

  const double *q = c->q + bh * T * p, *k = c->k + bh * T * p, *v = c->v + bh * T * dv;
  double *o = c->o ? c->o + bh * T * dv : NULL;
  for (int64_t t = 0; t < T; ++t) {
    /* state update with the current token first (inclusive causal sum) */
    psi(k + t * p, p, pk);
    const double *v_t = v + t * dv;
    for (int64_t r = 0; r < P; ++r) {
      z[r] += pk[r];
      double *Sr = S + r * dv;
      for (int e = 0; e < dv; ++e) Sr[e] += pk[r] * v_t[e];
    }
    /* readout o_t = psi(q_t)^T S_t / psi(q_t)^T z_t */
    if (o) {
      psi(q + t * p, p, pq);
      double den = 0.0;
      for (int e = 0; e < dv; ++e) num[e] = 0.0;
      for (int64_t r = 0; r < P; ++r) {
        den += pq[r] * z[r];
        const double *Sr = S + r * dv;
        for (int e = 0; e < dv; ++e) num[e] += pq[r] * Sr[e];
      }
      for (int e = 0; e < dv; ++e) o[t * dv + e] = (den > 0.0) ? num[e] / den : 0.0;
    }
  }
  if (c->S_out) memcpy(c->S_out + bh * P * dv, S, sizeof(double) * (size_t)(P * dv));
  if (c->z_out) memcpy(c->z_out + bh * P, z, sizeof(double) * (size_t)P);
done:
  free(S);
  free(z);
  free(pk);
  free(pq);
  free(num);
}

/* o may be NULL (state only).  S0/z0 give the state before token 1 (NULL:
 * zero); S_out/z_out receive the state after token T (NULL: not returned). */
int kata_oracle_recurrent(const double *q, const double *k, const double *v, double *o,
                          int64_t B, int64_t H, int64_t T, int p, int dv,
                          const double *S0, const double *z0, double *S_out, double *z_out,
                          int nthreads) {
  if (!q || !k || !v || B < 0 || H < 0 || T < 0 || p <= 0 || dv <= 0) return KATA_ORACLE_EINVAL;
  if ((S0 == NULL) != (z0 == NULL)) return KATA_ORACLE_EINVAL;
  recur_ctx c = {q, k, v, o, T, p, dv, S0, z0, S_out, z_out};
  return run_pairs(recur_pair, &c, B * H, nthreads);
}

/* ------------------------------------------------------------------------ */
/* KATA-Mg: g PSD factors over a head of width d                             */
/* ------------------------------------------------------------------------ */
/*
 * The head's d coordinates are split into g consecutive groups of width
 * p = d / g, u = [u^1 | ... | u^g], and the feature is the concatenation of
 * the rank-one maps of the groups:
 *
 *   psi_Mg(u) = [psi(u^1) | ... | psi(u^g)],   psi(u^j) = vec(u^j u^j^T)
 *   w_{t,s}   = <psi_Mg(q_t), psi_Mg(k_s)> = sum_j (q_t^j . k_s^j)^2
 *
 * with one shared value vector and one shared denominator (arXiv abstract
 * and gist.science sec. 2.3 "Varianten": KATA-Mg, several PSD factors; the
 * ai.info summary, Main Findings, gives its state as d(d/g+1)/2 * dv packed,
 * i.e. g blocks of (d/g)(d/g+1)/2 * dv, and g = 1 is the full map).  The
 * state of the recurrent form is [g*p*p, dv] with row r = j*p*p + a*p + b
 * holding psi(u^j)_{a*p+b} = u^j_a u^j_b.
 */

typedef struct {
  const double *q, *k, *v;
  double *o;
  int64_t T;
  int d, g, dv;
} direct_mg_ctx;

/* w_{t,s} = sum over groups of the squared group dot product. */
static double weight_mg(const double *q_t, const double *k_s, int d, int g) {
  const int p = d / g;
  double w = 0.0;
  for (int j = 0; j < g; ++j) {
    double dot = 0.0;
    for (int i = 0; i < p; ++i) dot += q_t[j * p + i] * k_s[j * p + i];
    w += dot * dot;
  }
  return w;
}

static void direct_mg_row(const double *q_t, const double *k, const double *v, int64_t t, int d, int g,
                          int dv, double *N, double *o_t, double *D_out) {
  double D = 0.0;
  for (int e = 0; e < dv; ++e) N[e] = 0.0;
  for (int64_t s = 0; s <= t; ++s) {
    const double w = weight_mg(q_t, k + s * d, d, g);
    D += w;
    const double *v_s = v + s * dv;
    for (int e = 0; e < dv; ++e) N[e] += w * v_s[e];
  }
  for (int e = 0; e < dv; ++e) o_t[e] = (D > 0.0) ? N[e] / D : 0.0;
  if (D_out) *D_out = D;
}

static void direct_mg_pair(void *vctx, int64_t bh) {
  direct_mg_ctx *c = (direct_mg_ctx *)vctx;
  const double *q = c->q + bh * c->T * c->d;
  const double *k = c->k + bh * c->T * c->d;
  const double *v = c->v + bh * c->T * c->dv;
  double *o = c->o + bh * c->T * c->dv;
  double *N = (double *)malloc(sizeof(double) * (size_t)c->dv);
  if (!N) return;
  for (int64_t t = 0; t < c->T; ++t)
    direct_mg_row(q + t * c->d, k, v, t, c->d, c->g, c->dv, N, o + t * c->dv, NULL);
  free(N);
}

static int mg_shape_ok(int d, int g, int dv) { return d > 0 && g > 0 && dv > 0 && d % g == 0; }

/* q,k [B,H,T,d], v,o [B,H,T,dv]. */
int kata_oracle_direct_mg(const double *q, const double *k, const double *v, double *o,
                          int64_t B, int64_t H, int64_t T, int d, int g, int dv, int nthreads) {
  if (!q || !k || !v || !o || B < 0 || H < 0 || T < 0 || !mg_shape_ok(d, g, dv)) return KATA_ORACLE_EINVAL;
  direct_mg_ctx c = {q, k, v, o, T, d, g, dv};
  return run_pairs(direct_mg_pair, &c, B * H, nthreads);
}

/* The direct Mg sum on rows (bh_idx[r], t_idx[r]); D_t to d_rows when non-NULL. */
int kata_oracle_direct_mg_rows(const double *q, const double *k, const double *v,
                               int64_t BH, int64_t T, int d, int g, int dv,
                               const int64_t *bh_idx, const int64_t *t_idx, int64_t nrows,
                               double *o_rows, double *d_rows) {
  if (!q || !k || !v || !bh_idx || !t_idx || !o_rows || !mg_shape_ok(d, g, dv)) return KATA_ORACLE_EINVAL;
  double *N = (double *)malloc(sizeof(double) * (size_t)dv);
  if (!N) return KATA_ORACLE_ENOMEM;
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t bh = bh_idx[r], t = t_idx[r];
    if (bh < 0 || bh >= BH || t < 0 || t >= T) {
      free(N);
      return KATA_ORACLE_EINVAL;
    }
    const double *qb = q + bh * T * d, *kb = k + bh * T * d, *vb = v + bh * T * dv;
    direct_mg_row(qb + t * d, kb, vb, t, d, g, dv, N, o_rows + r * dv, d_rows ? d_rows + r : NULL);
  }
  free(N);
  return KATA_ORACLE_OK;
}

typedef struct {
  const double *q, *k, *v;
  double *o;
  int64_t T;
  int d, g, dv;
  const double *S0, *z0;
  double *S_out, *z_out;
} recur_mg_ctx;

/* psi_Mg(u): the g group maps one after another, row r = j*p*p + a*p + b. */
static void psi_mg(const double *u, int d, int g, double *out) {
  const int p = d / g;
  for (int j = 0; j < g; ++j) psi(u + j * p, p, out + (int64_t)j * p * p);
}

static void recur_mg_pair(void *vctx, int64_t bh) {
  recur_mg_ctx *c = (recur_mg_ctx *)vctx;
  const int d = c->d, g = c->g, dv = c->dv, p = d / g;
  const int64_t P = (int64_t)g * p * p, T = c->T;
  double *S = (double *)malloc(sizeof(double) * (size_t)(P * dv));
  double *z = (double *)malloc(sizeof(double) * (size_t)P);
  double *pk = (double *)malloc(sizeof(double) * (size_t)P);
  double *pq = (double *)malloc(sizeof(double) * (size_t)P);
  double *num = (double *)malloc(sizeof(double) * (size_t)dv);
  if (!S || !z || !pk || !pq || !num) goto done;
  if (c->S0) memcpy(S, c->S0 + bh * P * dv, sizeof(double) * (size_t)(P * dv));
  else memset(S, 0, sizeof(double) * (size_t)(P * dv));
  if (c->z0) memcpy(z, c->z0 + bh * P, sizeof(double) * (size_t)P);
  else memset(z, 0, sizeof(double) * (size_t)P);

  const double *q = c->q + bh * T * d, *k = c->k + bh * T * d, *v = c->v + bh * T * dv;
  double *o = c->o ? c->o + bh * T * dv : NULL;
  for (int64_t t = 0; t < T; ++t) {
    psi_mg(k + t * d, d, g, pk);
    const double *v_t = v + t * dv;
    for (int64_t r = 0; r < P; ++r) {
      z[r] += pk[r];
      double *Sr = S + r * dv;
      for (int e = 0; e < dv; ++e) Sr[e] += pk[r] * v_t[e];
    }
    if (o) {
      psi_mg(q + t * d, d, g, pq);
      double den = 0.0;
      for (int e = 0; e < dv; ++e) num[e] = 0.0;
      for (int64_t r = 0; r < P; ++r) {
        den += pq[r] * z[r];
        const double *Sr = S + r * dv;
        for (int e = 0; e < dv; ++e) num[e] += pq[r] * Sr[e];
      }
      for (int e = 0; e < dv; ++e) o[t * dv + e] = (den > 0.0) ? num[e] / den : 0.0;
    }
  }
  if (c->S_out) memcpy(c->S_out + bh * P * dv, S, sizeof(double) * (size_t)(P * dv));
  if (c->z_out) memcpy(c->z_out + bh * P, z, sizeof(double) * (size_t)P);
done:
  free(S);
  free(z);
  free(pk);
  free(pq);
  free(num);
}

/* The Mg state recurrence: state [B,H,g*p*p,dv] and [B,H,g*p*p]; the
 * arguments are as for kata_oracle_recurrent with p replaced by (d, g). */
int kata_oracle_recurrent_mg(const double *q, const double *k, const double *v, double *o,
                             int64_t B, int64_t H, int64_t T, int d, int g, int dv,
                             const double *S0, const double *z0, double *S_out, double *z_out,
                             int nthreads) {
  if (!q || !k || !v || B < 0 || H < 0 || T < 0 || !mg_shape_ok(d, g, dv)) return KATA_ORACLE_EINVAL;
  if ((S0 == NULL) != (z0 == NULL)) return KATA_ORACLE_EINVAL;
  recur_mg_ctx c = {q, k, v, o, T, d, g, dv, S0, z0, S_out, z_out};
  return run_pairs(recur_mg_pair, &c, B * H, nthreads);
}

/* Number of threads run_pairs uses for nthreads <= 0. */
int kata_oracle_default_threads(void) {
  long c = sysconf(_SC_NPROCESSORS_ONLN);
  return c > 0 ? (int)c : 1;
}
