/*
 * wk_oracle.c -- plain, slow fp64 reference of the Wukong interaction-stack forward.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product calls this code: only the
 * tests, the smoke check and the benchmark's CPU-baseline leg load it. It shares
 * no code with the CUDA path; it reads the same input bits (bf16 or fp32
 * storage, upcast exactly to double) and computes everything in double.
 *
 * Source of the method: the Wukong page (xdnf.cn repost of the Zhihu summary of
 * "Wukong: Towards a Scaling Law for Large-Scale Recommendation", arXiv
 * 2403.02545), section 2.2 and 2.3. The page's formulas were lost when it was
 * extracted; the surviving text fixes:
 *   - a Wukong layer = Factorization Machine Block (FMB) and Linear Compress
 *     Block (LCB), their outputs concatenated, plus a residual connection, then
 *     LayerNorm (section 2.2, first paragraph);
 *   - the FMB's FM is an optimised FM that first compresses the number of
 *     features to k and then computes the crossing, and the FMB outputs a matrix
 *     of n_F embeddings (section 2.2, FMB paragraph);
 *   - the LCB is a weight matrix W_L times the layer input, with n_L the number
 *     of compressed output embeddings and n_i the number of embeddings of layer
 *     i (section 2.2, LCB paragraph);
 *   - the knobs l, n_F, n_L, k and the MLP of the FMB (section 2.3).
 * The equations written out below are the reading of those sentences:
 *   FM(X)   = (X X^T) Y,          X in R^{n x d}, Y in R^{n x k}
 *             (the optimised form X (X^T Y) is the same product re-associated;
 *             the oracle deliberately takes the plain pairwise-dot-product form)
 *   FMB(X)  = reshape_{n_F x d}( MLP( LN( flatten_rowmajor( FM(X) ) ) ) )
 *   MLP     = m Linear layers h_0 = n k -> ... -> h_m = n_F d, ReLU after every
 *             Linear except the last
 *   LCB(X)  = W_L X,              W_L in R^{n_L x n}
 *   layer   = LN_rows( concat_rows(FMB(X), LCB(X)) + X ),   n_F + n_L = n
 *   LN(v)   = (v - mean) / sqrt(var + eps) * gamma + beta, biased variance,
 *             two passes; the FMB LayerNorm acts on the whole flattened n*k
 *             vector, the output LayerNorm on each embedding row (d values).
 *
 * Parity status: pinned by the identity tests of tests/test_oracle_pins.py
 * (re-association X(X^T Y), orthogonal-row and tiny exact-rational FM cases,
 * LCB with W_L = I, LayerNorm closed forms, the all-zero-weights layer reducing
 * to a library LayerNorm, MLP identity and ReLU cases, concat order). No page
 * prints a worked numeric example of a whole layer, so the composition itself
 * is pinned only through those identities.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int32_t n, d, k, n_f, n_l;
  int32_t mlp_num_linear;   /* m >= 1 */
  const int32_t* mlp_dims;  /* m+1 entries: h_0 = n*k, ..., h_m = n_f*d */
  double ln_eps;
  int32_t dtype;            /* storage of Y, W_j, W_L: 0 = fp32, 1 = bf16 bits */
} wko_config;

typedef struct {
  const void* Y;                        /* [n, k] */
  const void* const* W;                 /* m entries, [h_{j+1}, h_j] row-major */
  const float* const* b;                /* m entries, [h_{j+1}], NULL entry = zero bias */
  const float* fmb_gamma;               /* [n*k] */
  const float* fmb_beta;                /* [n*k] */
  const void* W_L;                      /* [n_l, n] */
  const float* out_gamma;               /* [d] */
  const float* out_beta;                /* [d] */
} wko_layer;

/* ---- storage ----------------------------------------------------------- */

static double load_elem(int32_t dtype, const void* p, int64_t i) {
  if (dtype == 1) {
    uint32_t u = ((uint32_t)((const uint16_t*)p)[i]) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
  }
  return (double)((const float*)p)[i];
}

/* Rounding used only by the diagnostic mode: double -> fp32 (nearest-even) ->
 * bf16 (nearest-even on the fp32 bits), the path a GPU takes when it stores an
 * fp32 accumulator as bf16. */
static double round_bf16_via_f32(double v) {
  float f = (float)v;
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7F800000u) == 0x7F800000u) return (double)f;
  uint32_t lsb = (u >> 16) & 1u;
  u = (u + 0x7FFFu + lsb) & 0xFFFF0000u;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* diagnostic rounding points (bit mask of the diag argument) */
enum { DIAG_A0 = 1, DIAG_HIDDEN = 2, DIAG_CONCAT = 4, DIAG_XOUT = 8, DIAG_XOPS = 16, DIAG_Z = 32, DIAG_F16 = 64 };

/* set by wko_layer_forward from the DIAG_F16 bit: round to fp16 instead of bf16 */
static int g_diag_f16 = 0;

/* double -> fp32 (nearest-even) -> fp16 (nearest-even, subnormals kept), diagnostic only */
static double round_f16_via_f32(double v) {
  float f = (float)v;
  double a = fabs((double)f);
  if (a == 0.0 || a >= 65520.0) return a >= 65520.0 ? copysign(INFINITY, v) : (double)f;
  int e;
  frexp(a, &e);                          /* a = m * 2^e, m in [0.5, 1) */
  int q = e - 11;                        /* spacing 2^(e-11) for 11 significant bits */
  if (q < -24) q = -24;                  /* subnormal spacing */
  double step = ldexp(1.0, q);
  double r = nearbyint((double)f / step) * step;   /* ties to even under the default mode */
  return r;
}

static double round_diag(double v) { return g_diag_f16 ? round_f16_via_f32(v) : round_bf16_via_f32(v); }

static void maybe_round(double* v, int64_t len, int diag) {
  if (!diag) return;
  for (int64_t i = 0; i < len; ++i) v[i] = round_diag(v[i]);
}

/* ---- the steps, each on one example ------------------------------------ */

/* FM: F = P Y with P[i][j] = <x_i, x_j>, the pairwise dot products of the
 * embedding rows. X [n,d], Y [n,k], F [n,k]; P is scratch [n,n]. */
void wko_fm(int32_t n, int32_t d, int32_t k, const double* X, const double* Y, double* P, double* F) {
  for (int32_t i = 0; i < n; ++i)
    for (int32_t j = 0; j < n; ++j) {
      double s = 0.0;
      for (int32_t t = 0; t < d; ++t) s += X[(int64_t)i * d + t] * X[(int64_t)j * d + t];
      P[(int64_t)i * n + j] = s;
    }
  for (int32_t i = 0; i < n; ++i)
    for (int32_t c = 0; c < k; ++c) {
      double s = 0.0;
      for (int32_t j = 0; j < n; ++j) s += P[(int64_t)i * n + j] * Y[(int64_t)j * k + c];
      F[(int64_t)i * k + c] = s;
    }
}

/* LayerNorm of one vector: y = (x - mean) / sqrt(var + eps) * gamma + beta,
 * mean and biased variance by two passes. gamma/beta may be NULL (1 and 0). */
void wko_layernorm(int64_t len, const double* x, const double* gamma, const double* beta, double eps, double* y) {
  double mean = 0.0;
  for (int64_t i = 0; i < len; ++i) mean += x[i];
  mean /= (double)len;
  double var = 0.0;
  for (int64_t i = 0; i < len; ++i) var += (x[i] - mean) * (x[i] - mean);
  var /= (double)len;
  double inv = 1.0 / sqrt(var + eps);
  for (int64_t i = 0; i < len; ++i) {
    double g = gamma ? gamma[i] : 1.0;
    double b = beta ? beta[i] : 0.0;
    y[i] = (x[i] - mean) * inv * g + b;
  }
}

/* LCB: G = W_L X, G [n_l, d]. */
void wko_lcb(int32_t n, int32_t d, int32_t n_l, const double* WL, const double* X, double* G) {
  for (int32_t r = 0; r < n_l; ++r)
    for (int32_t t = 0; t < d; ++t) {
      double s = 0.0;
      for (int32_t i = 0; i < n; ++i) s += WL[(int64_t)r * n + i] * X[(int64_t)i * d + t];
      G[(int64_t)r * d + t] = s;
    }
}

/* ---- threading helper --------------------------------------------------- */

typedef void (*range_fn)(void* ctx, int64_t begin, int64_t end);
typedef struct {
  range_fn fn;
  void* ctx;
  int64_t begin, end;
} range_job;

static void* range_worker(void* a) {
  range_job* j = (range_job*)a;
  j->fn(j->ctx, j->begin, j->end);
  return NULL;
}

static void parallel_for(int64_t count, int threads, range_fn fn, void* ctx) {
  if (count <= 0) return;
  if (threads < 1) threads = 1;
  if (threads > 256) threads = 256;
  if (threads > count) threads = (int)count;
  range_job jobs[256];
  pthread_t tid[256];
  int created[256];
  int64_t chunk = (count + threads - 1) / threads;
  for (int t = 0; t < threads; ++t) {
    jobs[t].fn = fn;
    jobs[t].ctx = ctx;
    jobs[t].begin = (int64_t)t * chunk;
    jobs[t].end = jobs[t].begin + chunk < count ? jobs[t].begin + chunk : count;
    created[t] = 0;
  }
  for (int t = 1; t < threads; ++t) {
    if (jobs[t].begin >= jobs[t].end) continue;
    created[t] = pthread_create(&tid[t], NULL, range_worker, &jobs[t]) == 0;
    if (!created[t]) range_worker(&jobs[t]);
  }
  range_worker(&jobs[0]);
  for (int t = 1; t < threads; ++t)
    if (created[t]) pthread_join(tid[t], NULL);
}

/* ---- one layer over a set of examples ----------------------------------- */

typedef struct {
  const wko_config* cfg;
  const wko_layer* w;
  int64_t n_ex;
  const double* X_in;   /* [n_ex, n, d] */
  double* X_out;        /* [n_ex, n, d] */
  double** h;           /* m+1 activation arrays, h[j] is [n_ex, h_j] */
  double* Yd;           /* [n, k] */
  double* WLd;          /* [n_l, n] */
  double* g1; double* b1; double* g2; double* b2;
  int diag;
  int j;                /* current MLP layer */
} layer_ctx;

static void fmb_front(void* c, int64_t e0, int64_t e1) {
  layer_ctx* L = (layer_ctx*)c;
  const wko_config* cfg = L->cfg;
  int32_t n = cfg->n, d = cfg->d, k = cfg->k;
  double* P = (double*)malloc(sizeof(double) * (size_t)n * n);
  double* F = (double*)malloc(sizeof(double) * (size_t)n * k);
  double* Xr = (double*)malloc(sizeof(double) * (size_t)n * d);
  for (int64_t e = e0; e < e1; ++e) {
    memcpy(Xr, L->X_in + e * (int64_t)n * d, sizeof(double) * (size_t)n * d);
    maybe_round(Xr, (int64_t)n * d, L->diag & DIAG_XOPS);
    if (L->diag & DIAG_Z) {
      /* diagnostic only: the compressed association X (X^T Y) with X^T Y rounded to bf16 */
      for (int32_t t = 0; t < d; ++t)
        for (int32_t c = 0; c < k; ++c) {
          double z = 0.0;
          for (int32_t i = 0; i < n; ++i) z += Xr[(int64_t)i * d + t] * L->Yd[(int64_t)i * k + c];
          P[(int64_t)t * k + c] = round_diag(z);
        }
      for (int32_t i = 0; i < n; ++i)
        for (int32_t c = 0; c < k; ++c) {
          double f = 0.0;
          for (int32_t t = 0; t < d; ++t) f += Xr[(int64_t)i * d + t] * P[(int64_t)t * k + c];
          F[(int64_t)i * k + c] = f;
        }
    } else {
      wko_fm(n, d, k, Xr, L->Yd, P, F);
    }
    /* flatten row-major (feature i major, compressed index c minor), LayerNorm over n*k */
    double* a0 = L->h[0] + e * (int64_t)n * k;
    wko_layernorm((int64_t)n * k, F, L->g1, L->b1, cfg->ln_eps, a0);
    maybe_round(a0, (int64_t)n * k, L->diag & DIAG_A0);
  }
  free(P);
  free(F);
  free(Xr);
}

static void mlp_rows(void* c, int64_t r0, int64_t r1) {
  layer_ctx* L = (layer_ctx*)c;
  const wko_config* cfg = L->cfg;
  int j = L->j;
  int64_t in = cfg->mlp_dims[j], out = cfg->mlp_dims[j + 1];
  int relu = j < cfg->mlp_num_linear - 1;
  const void* W = L->w->W[j];
  const float* b = L->w->b ? L->w->b[j] : NULL;
  double* wrow = (double*)malloc(sizeof(double) * (size_t)in);
  for (int64_t r = r0; r < r1; ++r) {
    for (int64_t q = 0; q < in; ++q) wrow[q] = load_elem(cfg->dtype, W, r * in + q);
    double bias = b ? (double)b[r] : 0.0;
    for (int64_t e = 0; e < L->n_ex; ++e) {
      const double* x = L->h[j] + e * in;
      double s = 0.0;
      for (int64_t q = 0; q < in; ++q) s += wrow[q] * x[q];
      s += bias;
      if (relu && s < 0.0) s = 0.0;
      L->h[j + 1][e * out + r] = s;
    }
  }
  free(wrow);
}

static void layer_back(void* c, int64_t e0, int64_t e1) {
  layer_ctx* L = (layer_ctx*)c;
  const wko_config* cfg = L->cfg;
  int32_t n = cfg->n, d = cfg->d, n_f = cfg->n_f, n_l = cfg->n_l;
  int m = cfg->mlp_num_linear;
  double* G = (double*)malloc(sizeof(double) * (size_t)n_l * d);
  double* cat = (double*)malloc(sizeof(double) * (size_t)n * d);
  double* Xr = (double*)malloc(sizeof(double) * (size_t)n * d);
  for (int64_t e = e0; e < e1; ++e) {
    const double* X = L->X_in + e * (int64_t)n * d;
    memcpy(Xr, X, sizeof(double) * (size_t)n * d);
    maybe_round(Xr, (int64_t)n * d, L->diag & DIAG_XOPS);
    wko_lcb(n, d, n_l, L->WLd, Xr, G);
    /* concat rows: FMB rows 0..n_f-1 (the last MLP output, reshaped row-major to n_f x d),
       then LCB rows n_f..n-1 */
    const double* fmb = L->h[m] + e * (int64_t)n_f * d;
    memcpy(cat, fmb, sizeof(double) * (size_t)n_f * d);
    memcpy(cat + (int64_t)n_f * d, G, sizeof(double) * (size_t)n_l * d);
    maybe_round(cat, (int64_t)n * d, L->diag & DIAG_CONCAT);
    double* Xo = L->X_out + e * (int64_t)n * d;
    for (int32_t r = 0; r < n; ++r) {
      double* y = cat + (int64_t)r * d;
      for (int32_t t = 0; t < d; ++t) y[t] += X[(int64_t)r * d + t]; /* residual */
      wko_layernorm(d, y, L->g2, L->b2, cfg->ln_eps, Xo + (int64_t)r * d);
    }
    maybe_round(Xo, (int64_t)n * d, L->diag & DIAG_XOUT);
  }
  free(G);
  free(cat);
  free(Xr);
}

static double* upcast(int32_t dtype, const void* p, int64_t len) {
  double* out = (double*)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1));
  for (int64_t i = 0; i < len; ++i) out[i] = load_elem(dtype, p, i);
  return out;
}

static double* upcast_f32(const float* p, int64_t len) {
  if (!p) return NULL;
  return upcast(0, p, len);
}

/* One Wukong layer on n_ex examples: X_out = LN_rows(concat(FMB(X_in), LCB(X_in)) + X_in).
 * diag != 0 additionally rounds to bf16 where a GPU implementation may store an
 * intermediate, selected by bits: 1 the FMB LayerNorm output, 2 each MLP
 * activation, 4 the concatenated blocks, 8 the layer output, 16 the copy of the
 * layer input that the FM and the LCB multiply (the residual keeps the unrounded
 * input), 32 the FM taken as X (X^T Y) with X^T Y rounded; bit 64 rounds to fp16
 * instead of bf16. diag = 0 is the
 * exact fp64 reference (the one parity is graded against).
 * Returns 0, or 1 on an invalid configuration. */
int wko_layer_forward(const wko_config* cfg, const wko_layer* w, int64_t n_ex, const double* X_in, double* X_out,
                      int threads, int diag) {
  if (!cfg || !w || !X_in || !X_out || n_ex < 0) return 1;
  if (cfg->n_f + cfg->n_l != cfg->n || cfg->mlp_num_linear < 1) return 1;
  if (cfg->mlp_dims[0] != cfg->n * cfg->k || cfg->mlp_dims[cfg->mlp_num_linear] != cfg->n_f * cfg->d) return 1;
  int m = cfg->mlp_num_linear;
  layer_ctx L;
  memset(&L, 0, sizeof L);
  g_diag_f16 = (diag & DIAG_F16) != 0;
  L.cfg = cfg;
  L.w = w;
  L.n_ex = n_ex;
  L.X_in = X_in;
  L.X_out = X_out;
  L.diag = diag;
  L.h = (double**)calloc((size_t)m + 1, sizeof(double*));
  for (int j = 0; j <= m; ++j) L.h[j] = (double*)malloc(sizeof(double) * (size_t)(n_ex * cfg->mlp_dims[j] + 1));
  L.Yd = upcast(cfg->dtype, w->Y, (int64_t)cfg->n * cfg->k);
  L.WLd = upcast(cfg->dtype, w->W_L, (int64_t)cfg->n_l * cfg->n);
  L.g1 = upcast_f32(w->fmb_gamma, (int64_t)cfg->n * cfg->k);
  L.b1 = upcast_f32(w->fmb_beta, (int64_t)cfg->n * cfg->k);
  L.g2 = upcast_f32(w->out_gamma, cfg->d);
  L.b2 = upcast_f32(w->out_beta, cfg->d);

  parallel_for(n_ex, threads, fmb_front, &L);
  for (int j = 0; j < m; ++j) {
    L.j = j;
    parallel_for(cfg->mlp_dims[j + 1], threads, mlp_rows, &L);
    maybe_round(L.h[j + 1], n_ex * (int64_t)cfg->mlp_dims[j + 1], diag & DIAG_HIDDEN);
  }
  parallel_for(n_ex, threads, layer_back, &L);

  for (int j = 0; j <= m; ++j) free(L.h[j]);
  free(L.h);
  free(L.Yd);
  free(L.WLd);
  free(L.g1);
  free(L.b1);
  free(L.g2);
  free(L.b2);
  return 0;
}

/* One Linear layer on a batch, exposed for the MLP pins: out[e][r] = act(sum_q W[r][q] x[e][q] + b[r]). */
void wko_linear(int64_t n_ex, int64_t in, int64_t out, int32_t dtype, const void* W, const float* b, int relu,
                const double* x, double* y) {
  for (int64_t e = 0; e < n_ex; ++e)
    for (int64_t r = 0; r < out; ++r) {
      double s = 0.0;
      for (int64_t q = 0; q < in; ++q) s += load_elem(dtype, W, r * in + q) * x[e * in + q];
      if (b) s += (double)b[r];
      if (relu && s < 0.0) s = 0.0;
      y[e * out + r] = s;
    }
}

/* The bf16 rounding of the diagnostic mode, exposed for its own test. */
double wko_round_bf16(double v) { return round_bf16_via_f32(v); }
