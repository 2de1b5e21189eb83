/*
 * ace_oracle.c -- plain, slow, fp64 CPU oracle for ACE per-token expert
 * skipping in a routed SwiGLU MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header, table or constant with the
 * CUDA path.
 *
 * Source of every formula: "ACE: Adaptive Calibration-Free Expert Skipping
 * for MoE-based LLMs" (picx.dev whiteboard summary of arXiv 2609.05228),
 * cited below as [ACE] plus its section; the news article "ACE Skips
 * Low-Contribution MoE Experts Per Token" (ainews.surl.tw) is cited as [NEWS].
 *
 * Conventions
 *   - every computation is in double precision; weights arrive as float
 *     arrays (exact copies of the stored bf16 / fp32 values) and are widened
 *     element by element;
 *   - storage layouts (row-major):
 *       gamma [d]                       RMSNorm scale, diag of Gamma_l
 *       wr    [E][d]                    router; row e is w_{l,e}
 *       wg,wu [E][m][d]                 wg[e][j][i] = W^gate_{l,e}[i][j]
 *                                       (the page's W^gate is d x m)
 *       wd    [E][d][m]                 wd[e][i][j] = W^down_{l,e}[j][i]
 *                                       (the page's W^down is m x d)
 *   - no blocking, fusion or reordering beyond the definitions: each loop is
 *     the sum the formula writes.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------------ */
/* a tiny parallel-for over independent items (tokens or experts)            */
/* ------------------------------------------------------------------------ */
static int g_threads = 0;

void ora_set_threads(int n) { g_threads = n; }

int ora_get_threads(void) {
  if (g_threads > 0) return g_threads;
  long n = sysconf(_SC_NPROCESSORS_ONLN);
  return n > 0 ? (int)n : 1;
}

typedef void (*ora_body)(void *ctx, long item);
typedef struct { ora_body fn; void *ctx; long n; long next; } par_job;

static void *par_worker(void *p) {
  par_job *job = (par_job *)p;
  for (;;) {
    long i = __atomic_fetch_add(&job->next, 1, __ATOMIC_RELAXED);
    if (i >= job->n) break;
    job->fn(job->ctx, i);
  }
  return NULL;
}

static void par_for(long n, ora_body fn, void *ctx) {
  par_job job = {fn, ctx, n, 0};
  int nt = ora_get_threads();
  if (nt > n) nt = (int)n;
  if (nt <= 1) { par_worker(&job); return; }
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
  int started = 0;
  for (int i = 0; i < nt; ++i)
    if (pthread_create(&th[i], NULL, par_worker, &job) == 0) ++started;
  if (started == 0) par_worker(&job);
  for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  free(th);
}

/* ------------------------------------------------------------------------ */
/* RMSNorm input map: x = xbar Gamma_l                                       */
/* [ACE] "Theoretical Foundation": xbar is the RMS-normalised input           */
/* direction and Gamma_l the diagonal RMSNorm scale.                          */
/* ------------------------------------------------------------------------ */
void ora_rmsnorm(int T, int d, const double *u, const double *gamma,
                 double eps_rms, double *xbar, double *x) {
  for (int t = 0; t < T; ++t) {
    double ss = 0.0;
    for (int i = 0; i < d; ++i) ss += u[(long)t * d + i] * u[(long)t * d + i];
    double r = 1.0 / sqrt(ss / d + eps_rms);
    for (int i = 0; i < d; ++i) {
      double xb = u[(long)t * d + i] * r;
      if (xbar) xbar[(long)t * d + i] = xb;
      x[(long)t * d + i] = xb * gamma[i];
    }
  }
}

/* ------------------------------------------------------------------------ */
/* SwiGLU expert, [ACE] "Theoretical Foundation", the equation for f_{l,e}:  */
/*   f(x) = ( SiLU(xbar Gamma W^gate) (.) xbar Gamma W^up ) W^down            */
/* z is the already-scaled row xbar Gamma (length d).  h (length m) receives  */
/* the gated intermediate, out (length d) the expert output.                  */
/* ------------------------------------------------------------------------ */
static double silu(double a) { return a / (1.0 + exp(-a)); }

void ora_swiglu(int d, int m, const double *z, const float *wg, const float *wu,
                const float *wd, double *h, double *out) {
  for (int j = 0; j < m; ++j) {
    double a = 0.0, b = 0.0;           /* (z W^gate)_j and (z W^up)_j */
    for (int i = 0; i < d; ++i) {
      a += z[i] * (double)wg[(long)j * d + i];
      b += z[i] * (double)wu[(long)j * d + i];
    }
    h[j] = silu(a) * b;
  }
  for (int i = 0; i < d; ++i) {        /* (h W^down)_i */
    double s = 0.0;
    for (int j = 0; j < m; ++j) s += h[j] * (double)wd[(long)i * m + j];
    out[i] = s;
  }
}

/* ------------------------------------------------------------------------ */
/* Router, top-k and gate.  logits l_{t,e} = x_t . w_e (+ b_e);              */
/* p = softmax(l) over all E experts; the k largest logits are selected,     */
/* ties broken by the smaller expert index; rank 0 is the top-1 expert       */
/* ([ACE] "Conservative Fusion": the top-1 expert is the one with the        */
/* highest original router gate).  With renorm the gate of slot i is          */
/* p_{e_i} / sum_{j<k} p_{e_j}; without it, p_{e_i}.                          */
/* ------------------------------------------------------------------------ */
typedef struct {
  int T, d, E, k, renorm;
  const double *x; const float *wr; const float *bias;
  double *logits; int *idx; double *gate;
} router_ctx;

static void router_token(void *vctx, long t) {
  router_ctx *c = (router_ctx *)vctx;
  int d = c->d, E = c->E, k = c->k;
  double *l = c->logits + t * E;
  for (int e = 0; e < E; ++e) {
    double s = 0.0;
    for (int i = 0; i < d; ++i) s += c->x[t * d + i] * (double)c->wr[(long)e * d + i];
    if (c->bias) s += (double)c->bias[e];
    l[e] = s;
  }
  /* selection of the k best (logit desc, index asc) */
  int *sel = c->idx + t * k;
  for (int r = 0; r < k; ++r) {
    int best = -1;
    for (int e = 0; e < E; ++e) {
      int taken = 0;
      for (int q = 0; q < r; ++q) if (sel[q] == e) { taken = 1; break; }
      if (taken) continue;
      if (best < 0 || l[e] > l[best]) best = e;   /* strict: keeps lower index on ties */
    }
    sel[r] = best;
  }
  double lmax = l[0];
  for (int e = 1; e < E; ++e) if (l[e] > lmax) lmax = l[e];
  double Z = 0.0;
  for (int e = 0; e < E; ++e) Z += exp(l[e] - lmax);
  double ztop = 0.0;
  for (int r = 0; r < k; ++r) ztop += exp(l[sel[r]] - lmax) / Z;
  for (int r = 0; r < k; ++r) {
    double p = exp(l[sel[r]] - lmax) / Z;
    c->gate[t * k + r] = c->renorm ? p / ztop : p;
  }
}

void ora_router(int T, int d, int E, int k, const double *x, const float *wr,
                const float *bias, int renorm, double *logits, int *idx,
                double *gate) {
  router_ctx c = {T, d, E, k, renorm, x, wr, bias, logits, idx, gate};
  par_for(T, router_token, &c);
}

/* ------------------------------------------------------------------------ */
/* Norms used by GSP                                                          */
/* ------------------------------------------------------------------------ */
/* ||Gamma W||_F for W stored [m][d] (page orientation d x m). */
static double fro_gamma_w(int d, int m, const double *gamma, const float *w) {
  double s = 0.0;
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < m; ++j) {
      double v = gamma[i] * (double)w[(long)j * d + i];
      s += v * v;
    }
  return sqrt(s);
}

/* ||Gamma W W^down||_F, formed as the explicit d x d product
 * P[i][i'] = gamma_i sum_j W[i][j] W^down[j][i'].                            */
static double fro_gamma_w_wdown(int d, int m, const double *gamma,
                                const float *w, const float *wd) {
  double s = 0.0;
  for (int i = 0; i < d; ++i)
    for (int i2 = 0; i2 < d; ++i2) {
      double p = 0.0;
      for (int j = 0; j < m; ++j)
        p += (double)w[(long)j * d + i] * (double)wd[(long)i2 * m + j];
      p *= gamma[i];
      s += p * p;
    }
  return sqrt(s);
}

/* Matrix-free operators on R^m used by the power iteration.
 *   op_factor: v -> A^T A v for A in {Gamma W^gate, Gamma W^up, (W^down)^T},
 *              each a d x m matrix (sigma_1(W^down) = sigma_1((W^down)^T)).
 *   op_product: v -> (A_w^T A_w)(W^down (W^down)^T) v, whose dominant
 *              eigenvalue is sigma_1(Gamma W W^down)^2 (the non-zero
 *              spectrum of XY equals that of YX).                            */
enum { MAT_GATE_OR_UP = 0, MAT_DOWN_T = 1 };

/* y = A v (length d), A is d x m. */
static void a_times(int d, int m, const double *gamma, const float *w, int kind,
                    const double *v, double *y) {
  for (int i = 0; i < d; ++i) {
    double s = 0.0;
    if (kind == MAT_GATE_OR_UP) {
      for (int j = 0; j < m; ++j) s += (double)w[(long)j * d + i] * v[j];
      s *= gamma[i];
    } else {                       /* (W^down)^T [i][j] = wd[i][j] */
      for (int j = 0; j < m; ++j) s += (double)w[(long)i * m + j] * v[j];
    }
    y[i] = s;
  }
}

/* v = A^T y (length m). */
static void at_times(int d, int m, const double *gamma, const float *w, int kind,
                     const double *y, double *v) {
  for (int j = 0; j < m; ++j) {
    double s = 0.0;
    if (kind == MAT_GATE_OR_UP) {
      for (int i = 0; i < d; ++i) s += gamma[i] * (double)w[(long)j * d + i] * y[i];
    } else {
      for (int i = 0; i < d; ++i) s += (double)w[(long)i * m + j] * y[i];
    }
    v[j] = s;
  }
}

static double norm2(int n, const double *v) {
  double s = 0.0;
  for (int i = 0; i < n; ++i) s += v[i] * v[i];
  return sqrt(s);
}

/* Power iteration: v_0 = (1,...,1)/sqrt(m); iters times v <- A^T A v /
 * ||A^T A v||; returns ||A v_K||.  If a step hits the zero vector the
 * matrix annihilates v and 0 is returned. */
static double power_factor(int d, int m, const double *gamma, const float *w,
                           int kind, int iters) {
  double *v = (double *)malloc(sizeof(double) * m);
  double *y = (double *)malloc(sizeof(double) * d);
  double *t = (double *)malloc(sizeof(double) * m);
  for (int j = 0; j < m; ++j) v[j] = 1.0 / sqrt((double)m);
  double sigma = 0.0;
  int dead = 0;
  for (int it = 0; it < iters && !dead; ++it) {
    a_times(d, m, gamma, w, kind, v, y);
    at_times(d, m, gamma, w, kind, y, t);
    double n = norm2(m, t);
    if (n == 0.0) { dead = 1; break; }
    for (int j = 0; j < m; ++j) v[j] = t[j] / n;
  }
  if (!dead) { a_times(d, m, gamma, w, kind, v, y); sigma = norm2(d, y); }
  free(v); free(y); free(t);
  return sigma;
}

/* Power iteration for sigma_1(Gamma W W^down): v_0 = 1/sqrt(m); iters
 * times v <- M v / ||M v|| with M = (A_w^T A_w)(A_d^T A_d) where
 * A_d = (W^down)^T; returns sqrt(||M v_K||). */
static double power_product(int d, int m, const double *gamma, const float *w,
                            const float *wd, int iters) {
  double *v = (double *)malloc(sizeof(double) * m);
  double *y = (double *)malloc(sizeof(double) * d);
  double *t = (double *)malloc(sizeof(double) * m);
  for (int j = 0; j < m; ++j) v[j] = 1.0 / sqrt((double)m);
  for (int it = 0; it <= iters; ++it) {
    a_times(d, m, gamma, wd, MAT_DOWN_T, v, y);   /* D v */
    at_times(d, m, gamma, wd, MAT_DOWN_T, y, t);
    a_times(d, m, gamma, w, MAT_GATE_OR_UP, t, y); /* G (D v) */
    at_times(d, m, gamma, w, MAT_GATE_OR_UP, y, t);
    double n = norm2(m, t);
    if (it == iters || n == 0.0) { free(v); free(y); free(t); return sqrt(n); }
    for (int j = 0; j < m; ++j) v[j] = t[j] / n;
  }
  free(v); free(y); free(t);
  return 0.0;
}

/* ------------------------------------------------------------------------ */
/* Spectral bound constants: sigma_1 of Gamma W^gate, Gamma W^up, W^down.    */
/* [ACE] "Theoretical Foundation", the upper bound on ||f(x)||_2.            */
/* out[e*3 + {0,1,2}].                                                        */
/* ------------------------------------------------------------------------ */
typedef struct {
  int d, m, iters; const double *gamma; const float *wg, *wu, *wd; double *out;
} sigma_ctx;

static void sigma_expert(void *vctx, long e) {
  sigma_ctx *c = (sigma_ctx *)vctx;
  long off = e * (long)c->m * c->d;
  c->out[e * 3 + 0] = power_factor(c->d, c->m, c->gamma, c->wg + off, MAT_GATE_OR_UP, c->iters);
  c->out[e * 3 + 1] = power_factor(c->d, c->m, c->gamma, c->wu + off, MAT_GATE_OR_UP, c->iters);
  c->out[e * 3 + 2] = power_factor(c->d, c->m, c->gamma, c->wd + off, MAT_DOWN_T, c->iters);
}

void ora_sigma_factors(int E, int d, int m, const double *gamma, const float *wg,
                       const float *wu, const float *wd, int iters, double *out) {
  sigma_ctx c = {d, m, iters, gamma, wg, wu, wd, out};
  par_for(E, sigma_expert, &c);
}

/* ------------------------------------------------------------------------ */
/* Global Spectral Proxy, [ACE] "Methodology 1. Global Spectral Proxy":      */
/*   a^up   = ||Gamma W^up||   * ||Gamma W^gate W^down||                      */
/*   a^gate = ||Gamma W^gate|| * ||Gamma W^up W^down||                        */
/*   atilde = sqrt(a^up a^gate)                                               */
/*   A(e)   = atilde_e / (mean_j atilde_j + eps)                              */
/* spectral = 0: Frobenius norms as printed; spectral = 1: every norm is the  */
/* largest singular value from the power iteration above.                     */
/* norms[e*4 + {0,1,2,3}] = ||GWu||, ||GWgWd||, ||GWg||, ||GWuWd||.           */
/* ------------------------------------------------------------------------ */
typedef struct {
  int d, m, spectral, iters; const double *gamma; const float *wg, *wu, *wd;
  double *norms;
} gsp_ctx;

static void gsp_expert(void *vctx, long e) {
  gsp_ctx *c = (gsp_ctx *)vctx;
  int d = c->d, m = c->m;
  long off = e * (long)m * d;
  const float *wg = c->wg + off, *wu = c->wu + off, *wd = c->wd + off;
  double *n = c->norms + e * 4;
  if (!c->spectral) {
    n[0] = fro_gamma_w(d, m, c->gamma, wu);
    n[1] = fro_gamma_w_wdown(d, m, c->gamma, wg, wd);
    n[2] = fro_gamma_w(d, m, c->gamma, wg);
    n[3] = fro_gamma_w_wdown(d, m, c->gamma, wu, wd);
  } else {
    n[0] = power_factor(d, m, c->gamma, wu, MAT_GATE_OR_UP, c->iters);
    n[1] = power_product(d, m, c->gamma, wg, wd, c->iters);
    n[2] = power_factor(d, m, c->gamma, wg, MAT_GATE_OR_UP, c->iters);
    n[3] = power_product(d, m, c->gamma, wu, wd, c->iters);
  }
}

void ora_gsp(int E, int d, int m, const double *gamma, const float *wg,
             const float *wu, const float *wd, int spectral, int iters,
             double eps, double *norms, double *a_up, double *a_gate,
             double *a_tilde, double *A) {
  gsp_ctx c = {d, m, spectral, iters, gamma, wg, wu, wd, norms};
  par_for(E, gsp_expert, &c);
  double mean = 0.0;
  for (int e = 0; e < E; ++e) {
    a_up[e] = norms[e * 4 + 0] * norms[e * 4 + 1];
    a_gate[e] = norms[e * 4 + 2] * norms[e * 4 + 3];
    a_tilde[e] = sqrt(a_up[e] * a_gate[e]);
    mean += a_tilde[e];
  }
  mean /= E;
  for (int e = 0; e < E; ++e) A[e] = a_tilde[e] / (mean + eps);
}

/* ------------------------------------------------------------------------ */
/* Router-Conditioned Refinement, [ACE] "Methodology 2":                      */
/*   wtilde_e = w_e - mean_j w_j                                              */
/*   q_e      = wtilde_e / (RMS(wtilde_e) + eps) * rho                        */
/*   atilde_e = ||f_e(q_e)||_2 / (||q_e||_2 + eps)                            */
/* q_e stands where xbar stands in f, so f_e(q) applies Gamma to q.  The      */
/* layer normalisation A(e) = atilde_e / (mean_j atilde_j + eps) mirrors the  */
/* GSP one (the page prints the RCR score with A^RCR but not its formula).    */
/* ------------------------------------------------------------------------ */
typedef struct {
  int d, m; const double *gamma; const float *wg, *wu, *wd;
  const double *q; double *a_tilde; double *fnorm;
} rcr_ctx;

static void rcr_expert(void *vctx, long e) {
  rcr_ctx *c = (rcr_ctx *)vctx;
  int d = c->d, m = c->m;
  long off = e * (long)m * d;
  double *z = (double *)calloc((size_t)d, sizeof(double));
  double *h = (double *)calloc((size_t)m, sizeof(double));
  double *o = (double *)calloc((size_t)d, sizeof(double));
  const double *q = c->q + e * (long)d;
  for (int i = 0; i < d; ++i) z[i] = q[i] * c->gamma[i];
  ora_swiglu(d, m, z, c->wg + off, c->wu + off, c->wd + off, h, o);
  c->fnorm[e] = norm2(d, o);
  free(z); free(h); free(o);
}

void ora_rcr(int E, int d, int m, const double *gamma, const float *wr,
             const float *wg, const float *wu, const float *wd, double rho,
             double eps, double *q, double *fnorm, double *a_tilde, double *A) {
  double *mean_w = (double *)calloc((size_t)d, sizeof(double));
  for (int e = 0; e < E; ++e)
    for (int i = 0; i < d; ++i) mean_w[i] += (double)wr[(long)e * d + i];
  for (int i = 0; i < d; ++i) mean_w[i] /= E;
  for (int e = 0; e < E; ++e) {
    double ss = 0.0;
    for (int i = 0; i < d; ++i) {
      double wt = (double)wr[(long)e * d + i] - mean_w[i];
      q[(long)e * d + i] = wt;
      ss += wt * wt;
    }
    double rms = sqrt(ss / d);
    for (int i = 0; i < d; ++i) q[(long)e * d + i] = q[(long)e * d + i] / (rms + eps) * rho;
  }
  free(mean_w);
  rcr_ctx c = {d, m, gamma, wg, wu, wd, q, a_tilde, fnorm};
  par_for(E, rcr_expert, &c);
  double mean = 0.0;
  for (int e = 0; e < E; ++e) {
    a_tilde[e] = fnorm[e] / (norm2(d, q + (long)e * d) + eps);
    mean += a_tilde[e];
  }
  mean /= E;
  for (int e = 0; e < E; ++e) A[e] = a_tilde[e] / (mean + eps);
}

/* ------------------------------------------------------------------------ */
/* Scores and the skip decision, [ACE] "Methodology 1/2" (s = g A) and       */
/* "3. Conservative Fusion": c = max(s^GSP, s^RCR); a slot is skipped only    */
/* when both views call it low, S^ACE = S^GSP intersect S^RCR; the top-1      */
/* expert is always retained ([ACE]; [NEWS] likewise).  "Low" is s < tau.     */
/* Both forms are evaluated; the return value counts slots where the max rule */
/* and the set intersection disagree (always 0 for a correct oracle).         */
/* The pages' ablations replace the fusion rule ([ACE] "Fusion Strategy       */
/* Ablation", Table 5: Min, Mean; "Component Ablation", Table 4: one view):   */
/*   fusion 1  c = min(s^GSP, s^RCR), checked against the union of the sets  */
/*   fusion 2  c = (s^GSP + s^RCR) / 2                                       */
/*   fusion 3  c = s^GSP          fusion 4  c = s^RCR                        */
/* ------------------------------------------------------------------------ */
int ora_mask(int T, int k, const int *idx, const double *gate,
             const double *A_gsp, const double *A_rcr, double tau, int fusion,
             double *s_gsp, double *s_rcr, double *c, unsigned char *keep) {
  int disagree = 0;
  for (long s = 0; s < (long)T * k; ++s) {
    int e = idx[s];
    s_gsp[s] = gate[s] * A_gsp[e];
    s_rcr[s] = gate[s] * A_rcr[e];
    int low_g = s_gsp[s] < tau, low_r = s_rcr[s] < tau;
    switch (fusion) {
      case 1: c[s] = s_gsp[s] < s_rcr[s] ? s_gsp[s] : s_rcr[s]; break;
      case 2: c[s] = 0.5 * (s_gsp[s] + s_rcr[s]); break;
      case 3: c[s] = s_gsp[s]; break;
      case 4: c[s] = s_rcr[s]; break;
      default: c[s] = s_gsp[s] > s_rcr[s] ? s_gsp[s] : s_rcr[s]; break;
    }
    int rank = (int)(s % k);
    int skip = (c[s] < tau);
    if (fusion == 0 && (low_g && low_r) != skip) ++disagree;
    if (fusion == 1 && (low_g || low_r) != skip) ++disagree;
    keep[s] = (unsigned char)(rank == 0 || !skip);
  }
  return disagree;
}

/* ------------------------------------------------------------------------ */
/* Compaction of the kept (token, expert) slots, ordered by expert, then by  */
/* token.  counts[E], offsets[E+1]; slot_token / slot_rank per kept slot;     */
/* slot_of[T*k] = position of a kept slot, -1 for a skipped one.  Returns the */
/* number of kept slots.                                                      */
/* ------------------------------------------------------------------------ */
int ora_compact(int T, int k, int E, const int *idx, const unsigned char *keep,
                int *counts, int *offsets, int *slot_token, int *slot_rank,
                int *slot_of) {
  int S = 0;
  for (long s = 0; s < (long)T * k; ++s) slot_of[s] = -1;
  for (int e = 0; e < E; ++e) {
    offsets[e] = S;
    counts[e] = 0;
    for (int t = 0; t < T; ++t)
      for (int r = 0; r < k; ++r) {
        long s = (long)t * k + r;
        if (keep[s] && idx[s] == e) {
          slot_token[S] = t;
          slot_rank[S] = r;
          slot_of[s] = S;
          ++S;
          ++counts[e];
        }
      }
  }
  offsets[E] = S;
  return S;
}

/* ------------------------------------------------------------------------ */
/* The MoE layer output: y_t = sum over the kept slots i of token t, taken   */
/* in rank order, of g_{t,i} f_{e_i}(x_t).  Skipped slots drop out of the     */
/* sum without re-normalising the survivors.  x is the RMSNorm output.        */
/* ------------------------------------------------------------------------ */
typedef struct {
  int d, m, k; const double *x; const int *idx; const double *gate;
  const unsigned char *keep; const float *wg, *wu, *wd; double *y;
} fwd_ctx;

static void fwd_token(void *vctx, long t) {
  fwd_ctx *c = (fwd_ctx *)vctx;
  int d = c->d, m = c->m, k = c->k;
  double *h = (double *)malloc(sizeof(double) * m);
  double *o = (double *)malloc(sizeof(double) * d);
  double *y = c->y + t * d;
  for (int i = 0; i < d; ++i) y[i] = 0.0;
  for (int r = 0; r < k; ++r) {
    long s = t * k + r;
    if (!c->keep[s]) continue;
    long off = (long)c->idx[s] * m * d;
    ora_swiglu(d, m, c->x + t * d, c->wg + off, c->wu + off, c->wd + off, h, o);
    for (int i = 0; i < d; ++i) y[i] += c->gate[s] * o[i];
  }
  free(h); free(o);
}

void ora_combine(int T, int d, int m, int k, const double *x, const int *idx,
                 const double *gate, const unsigned char *keep, const float *wg,
                 const float *wu, const float *wd, double *y) {
  fwd_ctx c = {d, m, k, x, idx, gate, keep, wg, wu, wd, y};
  par_for(T, fwd_token, &c);
}
