/*
 * CPU oracle for the LeapQuant int8-state GDN/KDA decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The CUDA
 * library never includes, links or calls it, and it shares no code, header or
 * constant table with the CUDA path.
 *
 * Plain, slow, scalar C99 in fp64.  The only places that use fp32 are the ones
 * where the method stores a value (scales, smoothing factors, compensator
 * vectors are stored in fp32; codes are int8) and the quantizer's integer
 * decisions, which are taken in fp32, the precision of the kernel (the pages
 * fix none).  OpenMP is used only across independent state tiles in
 * orc_lq_batch; it changes no arithmetic.
 *
 * Sources (page title, then section):
 *  - "LeapQuant: Training-Free 8-bit Quantization for Linear Attention
 *    Recurrent States" (zhichai.net forum summary), numbered list of the three
 *    techniques: per-window quantization with a fixed low-bit state plus a
 *    high-precision buffer; Compensator Tokens for the largest outliers;
 *    smoothing of the residual.
 *  - "LeapQuant: Efficient Linear Attention with Accurate Recurrent State
 *    Quantization" (opentrain.ai), Abstract: outlier rows and columns of the
 *    state; compensators share the update path of real tokens.
 *  - globaltechnewsdesk news article on LeapQuant ("A linear-attention
 *    method cuts state ..."), paragraphs 3-5: window of 16 tokens,
 *    reconstruct and quantize once at the boundary, four Compensator Tokens,
 *    1.19 bytes per stored value.
 *  The exact recurrence S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T)
 *  + beta_t v_t k_t^T, o_t = S_t q_t is the Gated DeltaNet / Kimi Delta
 *  Attention rule those pages name; the pages do not print it.
 *
 * Readings where the pages are silent:
 *  - A Compensator Token is one whole row or one whole column of the state,
 *    chosen greedily by largest L2 energy over the d_v rows and d_k columns,
 *    stored in fp32 and removed from the residual.  Ties: the larger energy,
 *    then rows before columns, then the lower index; lines already taken are
 *    not candidates.
 *  - Smoothing: a per-key-column factor m_j = (max_i |R_ij|)^a with
 *    a in {0, 1/2, 1}; a column whose max is below the smallest normal fp32
 *    gets m_j = 1.
 *  - Quantization: symmetric int8 in [-127, 127] with one fp32 scale per
 *    state row, sigma_i = b_i / 127 where b_i is the row max of the smoothed
 *    residual; codes are rint-half-even of (R_ij * (1/m_j)) * (127/b_i),
 *    every product and quotient correctly rounded in fp32.  A row whose max
 *    is below the smallest normal fp32 gets sigma_i = 1 and zero codes.
 *  - The in-window buffer keeps, per token, the key k_i, the gate alpha_i and
 *    the delta d_i = u_i - S0 w_i, the image of the WY pair (w_i, u_i) under
 *    the fixed window-base state S0.  The WY pair itself is also carried here
 *    and checked against d_i at every step.
 *
 * Layout of a state tile: S is d_v x d_k, row-major, row i = value channel,
 * column j = key channel; o = S q.  A compensator id is i for row i and
 * d_v + j for column j.  Compensator vectors are stored with a stride of
 * max(d_k, d_v) values.
 *
 * Every entry point returns 0 on success and a negative value on a bad
 * argument.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { C_DK = 0, C_DV, C_W, C_K, C_GATE, C_QUANT, C_SMOOTH, C_NCFG };

/* Diagnostics written by the run functions.  The caller zeroes the array and
 * sets D_MIN_MARGIN to +inf before the first call. */
enum {
  D_WY_RESIDUAL = 0, /* max over steps of |d_t - (u_t - S0 w_t)| / max|d_t| */
  D_MIN_MARGIN,      /* min over selections of (best - runner-up) / best    */
  D_FOLDS,           /* number of folds performed                           */
  D_SELECTIONS,      /* number of compensator selections made               */
  D_NDIAG = 8
};

static int cfg_ok(const int *c) {
  if (!c) return 0;
  if (c[C_DK] < 1 || c[C_DV] < 1) return 0;
  if (c[C_W] < 1 || c[C_W] > 1024) return 0;
  if (c[C_K] < 0 || c[C_K] > c[C_DK] + c[C_DV]) return 0;
  if (c[C_GATE] != 0 && c[C_GATE] != 1) return 0;
  if (c[C_QUANT] != 0 && c[C_QUANT] != 1) return 0;
  if (c[C_SMOOTH] < 0 || c[C_SMOOTH] > 2) return 0;
  return 1;
}

static int dmax_of(const int *c) { return c[C_DK] > c[C_DV] ? c[C_DK] : c[C_DV]; }

/* ------------------------------------------------------------------------ */
/* Exact recurrence                                                          */
/* ------------------------------------------------------------------------ */

/* One token of the exact GDN (scalar gate) / KDA (per-key-channel gate)
 * recurrence, written as the delta rule:
 *   S <- S diag(alpha);  S <- S + beta (v - S k) k^T;  o = S q.
 * Expanding the two updates gives S_{t-1} diag(alpha)(I - beta k k^T)
 * + beta v k^T. */
static void exact_step(int dk, int dv, int gate, double *S, const double *q, const double *k,
                       const double *v, const double *alpha, double beta, double *o) {
  for (int i = 0; i < dv; ++i)
    for (int j = 0; j < dk; ++j) S[(long)i * dk + j] *= gate ? alpha[j] : alpha[0];
  for (int i = 0; i < dv; ++i) {
    double sk = 0.0;
    for (int j = 0; j < dk; ++j) sk += S[(long)i * dk + j] * k[j];
    double delta = beta * (v[i] - sk);
    for (int j = 0; j < dk; ++j) S[(long)i * dk + j] += delta * k[j];
  }
  for (int i = 0; i < dv; ++i) {
    double acc = 0.0;
    for (int j = 0; j < dk; ++j) acc += S[(long)i * dk + j] * q[j];
    o[i] = acc;
  }
}

/* Run T tokens of the exact recurrence on one tile.  Inputs of token t start
 * at q + t*sq (and so on); alpha holds 1 (GDN) or d_k (KDA) values per token;
 * beta one value per token. */
int orc_exact_run(const int *cfg, int T, double *S, const double *q, const double *k,
                  const double *v, const double *alpha, const double *beta, long sq, long sk,
                  long sv, long sa, long sb, double *o, long so) {
  if (!cfg_ok(cfg) || T < 0 || !S) return -1;
  int dk = cfg[C_DK], dv = cfg[C_DV], gate = cfg[C_GATE];
  for (int t = 0; t < T; ++t)
    exact_step(dk, dv, gate, S, q + t * sq, k + t * sk, v + t * sv, alpha + t * sa, beta[t * sb],
               o + t * so);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Quantizer: compensators, smoothing, per-row int8                          */
/* ------------------------------------------------------------------------ */

/* Line energies (sum of squares) of the residual, rows then columns. */
static void line_energies(int dk, int dv, const double *R, double *en) {
  for (int i = 0; i < dv; ++i) {
    double e = 0.0;
    for (int j = 0; j < dk; ++j) e += R[(long)i * dk + j] * R[(long)i * dk + j];
    en[i] = e;
  }
  for (int j = 0; j < dk; ++j) {
    double e = 0.0;
    for (int i = 0; i < dv; ++i) e += R[(long)i * dk + j] * R[(long)i * dk + j];
    en[dv + j] = e;
  }
}

/* Quantize a state S (d_v x d_k, fp64).
 *
 * quant = 1 (int8): the quantizer works on the fp32 rounding of S.  It pulls
 * out K compensator lines (cv, cid), then smooths (m) and quantizes (Q, sig)
 * the residual.  xq (nullable, d_v*d_k floats) receives each code's value
 * before rounding, for tie analysis.
 * quant = 0 (identity): the same compensator extraction in fp64; the residual
 * is kept exactly in Rid and the lines in cv64.  Nothing is rounded, so the
 * reconstruction equals S exactly. */
int orc_quantize(const int *cfg, const double *S, int8_t *Q, float *sig, float *m, float *cv,
                 int32_t *cid, double *Rid, double *cv64, float *xq, double *diag) {
  if (!cfg_ok(cfg) || !S || !cid) return -1;
  int dk = cfg[C_DK], dv = cfg[C_DV], K = cfg[C_K], quant = cfg[C_QUANT];
  int smooth = cfg[C_SMOOTH], dmax = dmax_of(cfg), nl = dk + dv;
  if (quant && (!Q || !sig || !m || (K > 0 && !cv))) return -1;
  if (!quant && (!Rid || (K > 0 && !cv64))) return -1;

  long nel = (long)dk * dv;
  double *R = malloc(sizeof(double) * nel);
  double *en = malloc(sizeof(double) * nl);
  char *taken = calloc(nl, 1);
  if (!R || !en || !taken) { free(R); free(en); free(taken); return -2; }
  for (long e = 0; e < nel; ++e) R[e] = quant ? (double)(float)S[e] : S[e];

  /* Compensator Tokens: K greedy picks of the highest-energy row or column. */
  for (int c = 0; c < K; ++c) {
    line_energies(dk, dv, R, en);
    int best = -1;
    for (int id = 0; id < nl; ++id) {
      if (taken[id]) continue;
      if (best < 0 || en[id] > en[best]) best = id;
    }
    double runner = -1.0;
    for (int id = 0; id < nl; ++id)
      if (!taken[id] && id != best && en[id] > runner) runner = en[id];
    if (diag) {
      diag[D_SELECTIONS] += 1.0;
      if (en[best] > 0.0 && runner >= 0.0) {
        double margin = (en[best] - runner) / en[best];
        if (margin < diag[D_MIN_MARGIN]) diag[D_MIN_MARGIN] = margin;
      }
    }
    if (best < dv) {
      for (int j = 0; j < dk; ++j) {
        double val = R[(long)best * dk + j];
        if (quant) cv[(long)c * dmax + j] = (float)val; else cv64[(long)c * dmax + j] = val;
        R[(long)best * dk + j] = 0.0;
      }
      for (int j = dk; j < dmax; ++j) {
        if (quant) cv[(long)c * dmax + j] = 0.0f; else cv64[(long)c * dmax + j] = 0.0;
      }
    } else {
      int jc = best - dv;
      for (int i = 0; i < dv; ++i) {
        double val = R[(long)i * dk + jc];
        if (quant) cv[(long)c * dmax + i] = (float)val; else cv64[(long)c * dmax + i] = val;
        R[(long)i * dk + jc] = 0.0;
      }
      for (int i = dv; i < dmax; ++i) {
        if (quant) cv[(long)c * dmax + i] = 0.0f; else cv64[(long)c * dmax + i] = 0.0;
      }
    }
    cid[c] = best;
    taken[best] = 1;
  }

  if (!quant) {
    memcpy(Rid, R, sizeof(double) * nel);
    free(R); free(en); free(taken);
    return 0;
  }

  /* Residual smoothing: one factor per key column, from the column max. */
  float *invm = malloc(sizeof(float) * dk);
  float *rt = malloc(sizeof(float) * dk);
  if (!invm || !rt) { free(R); free(en); free(taken); free(invm); free(rt); return -2; }
  for (int j = 0; j < dk; ++j) {
    float a = 0.0f;
    for (int i = 0; i < dv; ++i) {
      float x = fabsf((float)R[(long)i * dk + j]);
      if (x > a) a = x;
    }
    float mj;
    if (smooth == 0 || a < FLT_MIN) mj = 1.0f;
    else if (smooth == 1) mj = sqrtf(a);
    else mj = a;
    m[j] = mj;
    invm[j] = 1.0f / mj;
  }

  /* Symmetric int8 with one fp32 scale per row. */
  for (int i = 0; i < dv; ++i) {
    float b = 0.0f;
    for (int j = 0; j < dk; ++j) {
      rt[j] = (float)R[(long)i * dk + j] * invm[j];
      float x = fabsf(rt[j]);
      if (x > b) b = x;
    }
    if (b < FLT_MIN) {
      sig[i] = 1.0f;
      for (int j = 0; j < dk; ++j) {
        Q[(long)i * dk + j] = 0;
        if (xq) xq[(long)i * dk + j] = 0.0f;
      }
      continue;
    }
    sig[i] = b / 127.0f;
    float inv_s = 127.0f / b;
    for (int j = 0; j < dk; ++j) {
      float x = rt[j] * inv_s;
      if (xq) xq[(long)i * dk + j] = x;
      float r = rintf(x);
      if (r > 127.0f) r = 127.0f;
      if (r < -127.0f) r = -127.0f;
      Q[(long)i * dk + j] = (int8_t)r;
    }
  }
  free(R); free(en); free(taken); free(invm); free(rt);
  return 0;
}

/* Reconstruct the window-base state S0 (fp64) from a stored record:
 * S0 = diag(sig) Q diag(m) + sum of the compensator lines (int8), or
 * S0 = Rid + sum of the lines (identity). */
int orc_dequantize(const int *cfg, const int8_t *Q, const float *sig, const float *m,
                   const float *cv, const int32_t *cid, const double *Rid, const double *cv64,
                   double *S0) {
  if (!cfg_ok(cfg) || !S0) return -1;
  int dk = cfg[C_DK], dv = cfg[C_DV], K = cfg[C_K], quant = cfg[C_QUANT], dmax = dmax_of(cfg);
  if (quant && (!Q || !sig || !m || (K > 0 && (!cv || !cid)))) return -1;
  if (!quant && (!Rid || (K > 0 && (!cv64 || !cid)))) return -1;
  for (int i = 0; i < dv; ++i)
    for (int j = 0; j < dk; ++j) {
      long e = (long)i * dk + j;
      S0[e] = quant ? (double)sig[i] * (double)Q[e] * (double)m[j] : Rid[e];
    }
  for (int c = 0; c < K; ++c) {
    int id = cid[c];
    if (id < 0 || id >= dk + dv) return -1;
    if (id < dv) {
      for (int j = 0; j < dk; ++j)
        S0[(long)id * dk + j] += quant ? (double)cv[(long)c * dmax + j] : cv64[(long)c * dmax + j];
    } else {
      int jc = id - dv;
      for (int i = 0; i < dv; ++i)
        S0[(long)i * dk + jc] += quant ? (double)cv[(long)c * dmax + i] : cv64[(long)c * dmax + i];
    }
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Windowed decode                                                           */
/* ------------------------------------------------------------------------ */

/* Decay ratios Gamma_last / Gamma_s = prod_{s' = s+1 .. last} alpha_{s'} for
 * s = 0..last, as running products (never as quotients), and the window gate
 * Gamma_last = prod_{s' = 0 .. last} alpha_{s'}.  ratio is (last+1) x ga,
 * Gamma is ga values (ga = d_k for KDA, 1 for GDN).  Token s's gate is the
 * buffered ba[s], except that a non-null acur is the gate of token `last`
 * (the current token, not yet in the buffer). */
static void decay_ratios(int gate, int dk, const double *ba, const double *acur, int last,
                         double *ratio, double *Gamma) {
  int ga = gate ? dk : 1;
  for (int j = 0; j < ga; ++j) {
    double acc = 1.0;
    for (int s = last; s >= 0; --s) {
      ratio[(long)s * ga + j] = acc;
      const double *src = (acur && s == last) ? acur : ba + (long)s * ga;
      acc *= src[j];
    }
    Gamma[j] = acc;
  }
}

/* Current state inside the window: S_t = S0 diag(Gamma_t) + sum_s d_s (k_s o ratio_s)^T
 * over the n buffered tokens.  With n == 0 this is S0. */
static void window_state(int dk, int dv, int gate, const double *S0, int n, const double *bk,
                         const double *bd, const double *ba, double *S, double *ratio,
                         double *Gamma) {
  int ga = gate ? dk : 1;
  if (n > 0) decay_ratios(gate, dk, ba, NULL, n - 1, ratio, Gamma);
  else for (int j = 0; j < ga; ++j) Gamma[j] = 1.0;
  for (int i = 0; i < dv; ++i)
    for (int j = 0; j < dk; ++j) {
      double x = S0[(long)i * dk + j] * Gamma[gate ? j : 0];
      for (int s = 0; s < n; ++s)
        x += bd[(long)s * dv + i] * (bk[(long)s * dk + j] * ratio[(long)s * ga + (gate ? j : 0)]);
      S[(long)i * dk + j] = x;
    }
}

typedef struct {
  int dk, dv, W, gate;
  double *ratio, *Gamma, *gq, *gk, *yq, *yk, *cc, *aa, *d, *u, *w, *tmp;
} step_ws;

static int ws_alloc(step_ws *ws, const int *cfg) {
  ws->dk = cfg[C_DK]; ws->dv = cfg[C_DV]; ws->W = cfg[C_W]; ws->gate = cfg[C_GATE];
  int ga = ws->gate ? ws->dk : 1, dmax = dmax_of(cfg);
  ws->ratio = malloc(sizeof(double) * (long)(ws->W + 1) * ga);
  ws->Gamma = malloc(sizeof(double) * ga);
  ws->gq = malloc(sizeof(double) * ws->dk);
  ws->gk = malloc(sizeof(double) * ws->dk);
  ws->yq = malloc(sizeof(double) * ws->dv);
  ws->yk = malloc(sizeof(double) * ws->dv);
  ws->cc = malloc(sizeof(double) * (ws->W + 1));
  ws->aa = malloc(sizeof(double) * (ws->W + 1));
  ws->d = malloc(sizeof(double) * ws->dv);
  ws->u = malloc(sizeof(double) * ws->dv);
  ws->w = malloc(sizeof(double) * ws->dk);
  ws->tmp = malloc(sizeof(double) * dmax);
  return ws->ratio && ws->Gamma && ws->gq && ws->gk && ws->yq && ws->yk && ws->cc && ws->aa &&
         ws->d && ws->u && ws->w && ws->tmp;
}

static void ws_free(step_ws *ws) {
  free(ws->ratio); free(ws->Gamma); free(ws->gq); free(ws->gk); free(ws->yq); free(ws->yk);
  free(ws->cc); free(ws->aa); free(ws->d); free(ws->u); free(ws->w); free(ws->tmp);
}

/* One token inside the window, from the fixed base state S0 and the buffer.
 * With t = n buffered tokens before this one:
 *   Gamma_t = alpha_0 o ... o alpha_t,  ratio_s = prod_{s<s'<=t} alpha_{s'}
 *   y_q = S0 (Gamma_t o q),  y_k = S0 (Gamma_t o k)
 *   c_s = (k_s o ratio_s) . k,  a_s = (k_s o ratio_s) . q   (s < t)
 *   d_t = beta (v - y_k - sum_s c_s d_s)
 *   o_t = y_q + sum_s a_s d_s + (k . q) d_t
 * and the token (k, d_t, alpha) is appended.  WY form, carried for the
 * cross-check: u_t = beta (v - sum_s c_s u_s), w_t = beta (Gamma_t o k
 * - sum_s c_s w_s), and d_t must equal u_t - S0 w_t. */
static void lq_step(step_ws *ws, const double *S0, int *n, double *bk, double *bd, double *ba,
                    double *bu, double *bw, const double *q, const double *k, const double *v,
                    const double *alpha, double beta, double *o, double *diag) {
  int dk = ws->dk, dv = ws->dv, gate = ws->gate, ga = gate ? dk : 1;
  int t = *n;
  decay_ratios(gate, dk, ba, alpha, t, ws->ratio, ws->Gamma);
  for (int j = 0; j < dk; ++j) {
    double g = ws->Gamma[gate ? j : 0];
    ws->gq[j] = g * q[j];
    ws->gk[j] = g * k[j];
  }
  for (int i = 0; i < dv; ++i) {
    double aq = 0.0, ak = 0.0;
    for (int j = 0; j < dk; ++j) {
      aq += S0[(long)i * dk + j] * ws->gq[j];
      ak += S0[(long)i * dk + j] * ws->gk[j];
    }
    ws->yq[i] = aq;
    ws->yk[i] = ak;
  }
  for (int s = 0; s < t; ++s) {
    double c = 0.0, a = 0.0;
    for (int j = 0; j < dk; ++j) {
      double kt = bk[(long)s * dk + j] * ws->ratio[(long)s * ga + (gate ? j : 0)];
      c += kt * k[j];
      a += kt * q[j];
    }
    ws->cc[s] = c;
    ws->aa[s] = a;
  }
  double att = 0.0;
  for (int j = 0; j < dk; ++j) att += k[j] * q[j];
  double dnorm = 0.0;
  for (int i = 0; i < dv; ++i) {
    double x = v[i] - ws->yk[i];
    for (int s = 0; s < t; ++s) x -= ws->cc[s] * bd[(long)s * dv + i];
    ws->d[i] = beta * x;
    if (fabs(ws->d[i]) > dnorm) dnorm = fabs(ws->d[i]);
  }
  for (int i = 0; i < dv; ++i) {
    double x = ws->yq[i];
    for (int s = 0; s < t; ++s) x += ws->aa[s] * bd[(long)s * dv + i];
    o[i] = x + att * ws->d[i];
  }
  if (bu && bw) {
    for (int i = 0; i < dv; ++i) {
      double x = v[i];
      for (int s = 0; s < t; ++s) x -= ws->cc[s] * bu[(long)s * dv + i];
      ws->u[i] = beta * x;
    }
    for (int j = 0; j < dk; ++j) {
      double x = ws->gk[j];
      for (int s = 0; s < t; ++s) x -= ws->cc[s] * bw[(long)s * dk + j];
      ws->w[j] = beta * x;
    }
    double res = 0.0;
    for (int i = 0; i < dv; ++i) {
      double sw = 0.0;
      for (int j = 0; j < dk; ++j) sw += S0[(long)i * dk + j] * ws->w[j];
      double r = fabs(ws->d[i] - (ws->u[i] - sw));
      if (r > res) res = r;
    }
    if (dnorm > 0.0) res /= dnorm;
    if (diag && res > diag[D_WY_RESIDUAL]) diag[D_WY_RESIDUAL] = res;
    for (int i = 0; i < dv; ++i) bu[(long)t * dv + i] = ws->u[i];
    for (int j = 0; j < dk; ++j) bw[(long)t * dk + j] = ws->w[j];
  }
  for (int j = 0; j < dk; ++j) bk[(long)t * dk + j] = k[j];
  for (int i = 0; i < dv; ++i) bd[(long)t * dv + i] = ws->d[i];
  for (int j = 0; j < ga; ++j) ba[(long)t * ga + j] = alpha[j];
  *n = t + 1;
}

/* Record arrays of one tile, grouped to keep the signatures readable. */
typedef struct {
  int8_t *Q; float *sig, *m, *cv; int32_t *cid; double *Rid, *cv64;
} record;

/* Fold the buffered tokens into the state and quantize it again:
 * S = S0 diag(Gamma_n) + sum_{s<n} d_s (k_s o ratio_s)^T, then quantize(S).
 * The buffer is emptied. */
static int lq_fold(const int *cfg, step_ws *ws, double *S0, double *Sw, record *rec, int *n,
                   const double *bk, const double *bd, const double *ba, double *diag) {
  window_state(cfg[C_DK], cfg[C_DV], cfg[C_GATE], S0, *n, bk, bd, ba, Sw, ws->ratio, ws->Gamma);
  int rc = orc_quantize(cfg, Sw, rec->Q, rec->sig, rec->m, rec->cv, rec->cid, rec->Rid, rec->cv64,
                        NULL, diag);
  if (rc) return rc;
  *n = 0;
  if (diag) diag[D_FOLDS] += 1.0;
  return orc_dequantize(cfg, rec->Q, rec->sig, rec->m, rec->cv, rec->cid, rec->Rid, rec->cv64, S0);
}

/* Run T tokens of the windowed quantized decode on one tile, starting from
 * the given record and buffer (n tokens buffered).  Each time the buffer
 * reaches W tokens it is folded and the state requantized.  Record and buffer
 * are updated in place.  bu/bw (nullable together) carry the WY cross-check.
 * o receives the T outputs (o + t*so). */
int orc_lq_run(const int *cfg, int T, int8_t *Q, float *sig, float *m, float *cv, int32_t *cid,
               double *Rid, double *cv64, int *n, double *bk, double *bd, double *ba, double *bu,
               double *bw, const double *q, const double *k, const double *v, const double *alpha,
               const double *beta, long sq, long sk, long sv, long sa, long sb, double *o, long so,
               double *diag) {
  if (!cfg_ok(cfg) || T < 0 || !n || !bk || !bd || !ba) return -1;
  if (*n < 0 || *n >= cfg[C_W]) return -1;
  int dk = cfg[C_DK], dv = cfg[C_DV];
  record rec = {Q, sig, m, cv, cid, Rid, cv64};
  step_ws ws;
  double *S0 = malloc(sizeof(double) * (long)dk * dv);
  double *Sw = malloc(sizeof(double) * (long)dk * dv);
  int rc = (S0 && Sw && ws_alloc(&ws, cfg)) ? 0 : -2;
  if (!rc) rc = orc_dequantize(cfg, Q, sig, m, cv, cid, Rid, cv64, S0);
  for (int t = 0; t < T && !rc; ++t) {
    lq_step(&ws, S0, n, bk, bd, ba, bu, bw, q + t * sq, k + t * sk, v + t * sv, alpha + t * sa,
            beta[t * sb], o + t * so, diag);
    if (*n == cfg[C_W]) rc = lq_fold(cfg, &ws, S0, Sw, &rec, n, bk, bd, ba, diag);
  }
  ws_free(&ws);
  free(S0); free(Sw);
  return rc;
}

/* Fold a partially filled window (0 < n < W): same fold as at the boundary. */
int orc_lq_flush(const int *cfg, int8_t *Q, float *sig, float *m, float *cv, int32_t *cid,
                 double *Rid, double *cv64, int *n, const double *bk, const double *bd,
                 const double *ba, double *diag) {
  if (!cfg_ok(cfg) || !n || !bk || !bd || !ba) return -1;
  if (*n < 0 || *n > cfg[C_W]) return -1;
  if (*n == 0) return 0;
  int dk = cfg[C_DK], dv = cfg[C_DV];
  record rec = {Q, sig, m, cv, cid, Rid, cv64};
  step_ws ws;
  double *S0 = malloc(sizeof(double) * (long)dk * dv);
  double *Sw = malloc(sizeof(double) * (long)dk * dv);
  int rc = (S0 && Sw && ws_alloc(&ws, cfg)) ? 0 : -2;
  if (!rc) rc = orc_dequantize(cfg, Q, sig, m, cv, cid, Rid, cv64, S0);
  if (!rc) rc = lq_fold(cfg, &ws, S0, Sw, &rec, n, bk, bd, ba, diag);
  ws_free(&ws);
  free(S0); free(Sw);
  return rc;
}

/* The current state of a tile: the window-base state advanced by the n
 * buffered tokens (no quantization). */
int orc_lq_state(const int *cfg, const int8_t *Q, const float *sig, const float *m,
                 const float *cv, const int32_t *cid, const double *Rid, const double *cv64, int n,
                 const double *bk, const double *bd, const double *ba, double *S) {
  if (!cfg_ok(cfg) || !S || n < 0 || n > cfg[C_W]) return -1;
  if (n > 0 && (!bk || !bd || !ba)) return -1;
  int dk = cfg[C_DK], dv = cfg[C_DV], ga = cfg[C_GATE] ? dk : 1;
  double *S0 = malloc(sizeof(double) * (long)dk * dv);
  double *ratio = malloc(sizeof(double) * (long)(cfg[C_W] + 1) * ga);
  double *Gamma = malloc(sizeof(double) * ga);
  int rc = (S0 && ratio && Gamma) ? 0 : -2;
  if (!rc) rc = orc_dequantize(cfg, Q, sig, m, cv, cid, Rid, cv64, S0);
  if (!rc) window_state(dk, dv, cfg[C_GATE], S0, n, bk, bd, ba, S, ratio, Gamma);
  free(S0); free(ratio); free(Gamma);
  return rc;
}

/* ------------------------------------------------------------------------ */
/* Batch driver (CPU baseline timing): many independent tiles                */
/* ------------------------------------------------------------------------ */

/* Run T tokens on every tile of a batch of B sequences x Hv value heads, the
 * keys and queries shared by groups of Hv/Hk value heads (head hv reads key
 * head hv / (Hv/Hk)).  int8 records only.  Per-tile arrays are packed tile
 * after tile; inputs are token-major:
 *   q, k  [T][B][Hk][dk]     v, o [T][B][Hv][dv]
 *   alpha [T][B][Hv][1 or dk]  beta [T][B][Hv]
 * Buffers: n [tiles], bk [tiles][W][dk], bd [tiles][W][dv], ba [tiles][W][ga].
 * No WY cross-check.  nthreads <= 0 lets OpenMP choose.  Returns the number
 * of threads used, or a negative value on error. */
int orc_lq_batch(const int *cfg, int B, int Hk, int Hv, int T, int8_t *Q, float *sig, float *m,
                 float *cv, int32_t *cid, int *n, double *bk, double *bd, double *ba,
                 const double *q, const double *k, const double *v, const double *alpha,
                 const double *beta, double *o, int nthreads) {
  if (!cfg_ok(cfg) || !cfg[C_QUANT] || B < 0 || Hk < 1 || Hv < 1 || Hv % Hk || T < 0) return -1;
  int dk = cfg[C_DK], dv = cfg[C_DV], W = cfg[C_W], K = cfg[C_K], dmax = dmax_of(cfg);
  int ga = cfg[C_GATE] ? dk : 1, group = Hv / Hk;
  long tiles = (long)B * Hv;
  int used = 1, bad = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
  {
#pragma omp single
    used = omp_get_num_threads();
  }
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
#endif
  for (long tile = 0; tile < tiles; ++tile) {
    long b = tile / Hv, hv = tile % Hv, hk = hv / group;
    int rc = orc_lq_run(cfg, T, Q + tile * dk * dv, sig + tile * dv, m + tile * dk,
                        cv + tile * (long)K * dmax, cid + tile * K, NULL, NULL, n + tile,
                        bk + tile * (long)W * dk, bd + tile * (long)W * dv,
                        ba + tile * (long)W * ga, NULL, NULL,
                        q + (b * Hk + hk) * dk, k + (b * Hk + hk) * dk, v + tile * dv,
                        alpha + tile * ga, beta + tile, (long)B * Hk * dk, (long)B * Hk * dk,
                        tiles * dv, tiles * ga, tiles, o + tile * dv, tiles * dv, NULL);
    if (rc) bad |= 1;
  }
  return bad ? -1 : used;
}

/* Interface version, checked by the ctypes wrapper when it loads the library. */
int orc_version(void) { return 1; }
