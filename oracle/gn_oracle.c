/*
 * gn_oracle.c - plain fp64 CPU oracle for the row-normalization and rotary-embedding path.
 *
 * TEST INFRASTRUCTURE: see gn_oracle.h for who may call it and for the sources cited below
 * as [H] (Helios kernels article), [L] (optimized kernels for LLM layers) and [J] (Janus-Pro-7B
 * inference acceleration).
 *
 * Each public function is a loop over independent rows. A row is widened to double, the
 * definition is applied to it, and the result is written out. Reductions over a row or over
 * rows are plain left-to-right sums in double. Nothing is blocked, fused or reordered.
 */
#include "gn_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---- reading inputs ------------------------------------------------------------------ */

/* Element i of a buffer of type dt, widened to double. A bfloat16 value is the upper half of
 * an IEEE binary32 pattern, so widening is a 16-bit shift. */
static double rd(const void* p, int dt, int64_t i) {
  if (dt == ORC_F64) return ((const double*)p)[i];
  if (dt == ORC_F32) return (double)((const float*)p)[i];
  {
    uint32_t u = ((uint32_t)((const uint16_t*)p)[i]) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
  }
}

static void rd_row(const void* p, int dt, int64_t start, int64_t n, double* out) {
  for (int64_t j = 0; j < n; ++j) out[j] = rd(p, dt, start + j);
}

static double* scratch(int64_t n) {
  double* p = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
  if (!p) abort();
  return p;
}

/* ---- epilogues -------------------------------------------------------------------------
 * tanh-GeLU, [L] "编写定制融合算子": 0.5 z (1 + tanh(k (z + 0.044715 z^3))). The page prints
 * k = 0.79788456, the 8-digit value of sqrt(2/pi); the oracle uses sqrt(2/pi) itself.
 * SiLU, [J] section 4.1: z * sigmoid(z). */
static const double GELU_C = 0.044715;

static double gelu_k(void) { return sqrt(2.0 / M_PI); }

double oracle_act(int act, double z) {
  if (act == ORC_ACT_GELU_TANH) {
    double t = tanh(gelu_k() * (z + GELU_C * z * z * z));
    return 0.5 * z * (1.0 + t);
  }
  if (act == ORC_ACT_SILU) return z / (1.0 + exp(-z));
  return z;
}

/* d act / dz, by differentiating the definitions above. */
double oracle_act_grad(int act, double z) {
  if (act == ORC_ACT_GELU_TANH) {
    double k = gelu_k();
    double t = tanh(k * (z + GELU_C * z * z * z));
    return 0.5 * (1.0 + t) + 0.5 * z * (1.0 - t * t) * k * (1.0 + 3.0 * GELU_C * z * z);
  }
  if (act == ORC_ACT_SILU) {
    double s = 1.0 / (1.0 + exp(-z));
    return s * (1.0 + z * (1.0 - s));
  }
  return 1.0;
}

/* ---- RMSNorm on one row ([H] "内核一 FlashNorm") ------------------------------------------
 * r = 1 / sqrt(mean(x^2) + eps); xhat = x r; z = xhat w'; y = act(z). eps sits inside the
 * square root, as in the LayerNorm example of [L]. w' is the weight with the Gemma +1 offset
 * already applied by the caller. */
static double rms_row_inv(const double* x, int64_t n, double eps) {
  double ss = 0.0;
  for (int64_t j = 0; j < n; ++j) ss += x[j] * x[j];
  return 1.0 / sqrt(ss / (double)n + eps);
}

static void rms_row_fwd(const double* x, const double* wp, int64_t n, double eps, int act,
                        double* y, double* inv_out) {
  double r = rms_row_inv(x, n, eps);
  if (y)
    for (int64_t j = 0; j < n; ++j) y[j] = oracle_act(act, x[j] * r * wp[j]);
  if (inv_out) *inv_out = r;
}

/* Gradient of sum_j dy_j y_j for one row. With g = dy act'(z) and xhat = x r:
 *   dL/dw'_j = g_j xhat_j
 *   dL/dx_k  = r (g_k w'_k - xhat_k c),  c = mean_j(g_j w'_j xhat_j)
 * (differentiate xhat_j = x_j r(x), dr/dx_k = -r^3 x_k / n). */
static void rms_row_bwd(const double* x, const double* wp, const double* dy, int64_t n,
                        double eps, int act, double* dx, double* dw_acc) {
  double r = rms_row_inv(x, n, eps);
  double c = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    double xh = x[j] * r;
    double g = dy[j] * oracle_act_grad(act, xh * wp[j]);
    c += g * wp[j] * xh;
    if (dw_acc) dw_acc[j] += g * xh;
  }
  c /= (double)n;
  if (dx)
    for (int64_t j = 0; j < n; ++j) {
      double xh = x[j] * r;
      double g = dy[j] * oracle_act_grad(act, xh * wp[j]);
      dx[j] = r * (g * wp[j] - xh * c);
    }
}

/* effective weight w' = w (plain) or 1 + w (Gemma, [H] "内核一 FlashNorm") */
static void load_weight(const void* w, int w_dt, int64_t n, int gemma, double* wp) {
  for (int64_t j = 0; j < n; ++j) wp[j] = (gemma ? 1.0 : 0.0) + rd(w, w_dt, j);
}

void oracle_rmsnorm_fwd(const void* x, int x_dt, const void* w, int w_dt, int64_t M, int64_t N,
                        double eps, int gemma, int act, double* y, double* inv_rms) {
  double* wp = scratch(N);
  double* row = scratch(N);
  load_weight(w, w_dt, N, gemma, wp);
  for (int64_t m = 0; m < M; ++m) {
    rd_row(x, x_dt, m * N, N, row);
    rms_row_fwd(row, wp, N, eps, act, y ? y + m * N : NULL, inv_rms ? inv_rms + m : NULL);
  }
  free(row);
  free(wp);
}

void oracle_rmsnorm_bwd(const void* x, int x_dt, const void* w, int w_dt, const void* dy, int dy_dt,
                        int64_t M, int64_t N, double eps, int gemma, int act, double* dx,
                        double* dw) {
  double* wp = scratch(N);
  double* row = scratch(N);
  double* grow = scratch(N);
  load_weight(w, w_dt, N, gemma, wp);
  if (dw)
    for (int64_t j = 0; j < N; ++j) dw[j] = 0.0;
  for (int64_t m = 0; m < M; ++m) {
    rd_row(x, x_dt, m * N, N, row);
    rd_row(dy, dy_dt, m * N, N, grow);
    rms_row_bwd(row, wp, grow, N, eps, act, dx ? dx + m * N : NULL, dw);
  }
  free(grow);
  free(row);
  free(wp);
}

/* ---- LayerNorm on one row ([L] "编写定制融合算子") ------------------------------------------
 * mean = sum(x)/n; var = sum((x - mean)^2)/n (biased); s = 1/sqrt(var + eps);
 * xhat = (x - mean) s; z = xhat w + b; y = act(z). The page's example sums over its whole
 * block; one row of the hidden dimension is the block here. */
static void ln_row_stats(const double* x, int64_t n, double eps, double* mean, double* rstd) {
  double s = 0.0;
  for (int64_t j = 0; j < n; ++j) s += x[j];
  double mu = s / (double)n;
  double v = 0.0;
  for (int64_t j = 0; j < n; ++j) v += (x[j] - mu) * (x[j] - mu);
  v /= (double)n;
  *mean = mu;
  *rstd = 1.0 / sqrt(v + eps);
}

/* Gradient of sum_j dy_j y_j for one row. With g = dy act'(z), xhat as above:
 *   dL/dw_j = g_j xhat_j, dL/db_j = g_j
 *   dL/dx_k = s (g_k w_k - mean_j(g_j w_j) - xhat_k mean_j(g_j w_j xhat_j)). */
static void ln_row_bwd(const double* x, const double* w, const double* b, const double* dy,
                       int64_t n, double eps, int act, double* dx, double* dw_acc,
                       double* db_acc) {
  double mu, s;
  ln_row_stats(x, n, eps, &mu, &s);
  double c1 = 0.0, c2 = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    double xh = (x[j] - mu) * s;
    double g = dy[j] * oracle_act_grad(act, xh * w[j] + b[j]);
    c1 += g * w[j];
    c2 += g * w[j] * xh;
    if (dw_acc) dw_acc[j] += g * xh;
    if (db_acc) db_acc[j] += g;
  }
  c1 /= (double)n;
  c2 /= (double)n;
  if (dx)
    for (int64_t j = 0; j < n; ++j) {
      double xh = (x[j] - mu) * s;
      double g = dy[j] * oracle_act_grad(act, xh * w[j] + b[j]);
      dx[j] = s * (g * w[j] - c1 - xh * c2);
    }
}

static void load_affine(const void* w, const void* b, int dt, int64_t n, double* wv, double* bv) {
  for (int64_t j = 0; j < n; ++j) {
    wv[j] = w ? rd(w, dt, j) : 1.0;
    bv[j] = b ? rd(b, dt, j) : 0.0;
  }
}

void oracle_layernorm_fwd(const void* x, int x_dt, const void* w, const void* b, int wb_dt,
                          int64_t M, int64_t N, double eps, int act, double* y, double* mean,
                          double* rstd) {
  double* wv = scratch(N);
  double* bv = scratch(N);
  double* row = scratch(N);
  load_affine(w, b, wb_dt, N, wv, bv);
  for (int64_t m = 0; m < M; ++m) {
    rd_row(x, x_dt, m * N, N, row);
    double mu, s;
    ln_row_stats(row, N, eps, &mu, &s);
    if (y)
      for (int64_t j = 0; j < N; ++j) y[m * N + j] = oracle_act(act, (row[j] - mu) * s * wv[j] + bv[j]);
    if (mean) mean[m] = mu;
    if (rstd) rstd[m] = s;
  }
  free(row);
  free(bv);
  free(wv);
}

void oracle_layernorm_bwd(const void* x, int x_dt, const void* w, const void* b, int wb_dt,
                          const void* dy, int dy_dt, int64_t M, int64_t N, double eps, int act,
                          double* dx, double* dw, double* db) {
  double* wv = scratch(N);
  double* bv = scratch(N);
  double* row = scratch(N);
  double* grow = scratch(N);
  load_affine(w, b, wb_dt, N, wv, bv);
  if (dw)
    for (int64_t j = 0; j < N; ++j) dw[j] = 0.0;
  if (db)
    for (int64_t j = 0; j < N; ++j) db[j] = 0.0;
  for (int64_t m = 0; m < M; ++m) {
    rd_row(x, x_dt, m * N, N, row);
    rd_row(dy, dy_dt, m * N, N, grow);
    ln_row_bwd(row, wv, bv, grow, N, eps, act, dx ? dx + m * N : NULL, dw, db);
  }
  free(grow);
  free(row);
  free(bv);
  free(wv);
}

/* ---- rotary embedding on one head row ([H] "内核二 FlashRoPE") -------------------------------
 * Pair i is (x[2i], x[2i+1]), read as the complex number a + i c and multiplied by
 * cos + i (sign sin):  out[2i] = a cos - c sign sin,  out[2i+1] = a sign sin + c cos.
 * sign = -1 is the inverse rotation, which the article uses as the backward. */
static void rope_row(const double* x, const double* cs, const double* sn, int64_t d, int sign,
                     double* out) {
  for (int64_t i = 0; i < d / 2; ++i) {
    double a = x[2 * i], c = x[2 * i + 1];
    double co = cs[i], si = (double)sign * sn[i];
    out[2 * i] = a * co - c * si;
    out[2 * i + 1] = a * si + c * co;
  }
}

void oracle_rope(const void* x, int x_dt, const void* cos_t, const void* sin_t, int tab_dt,
                 int64_t B, int64_t S, int64_t H, int64_t D, int sign, double* out) {
  double* row = scratch(D);
  double* cs = scratch(D / 2);
  double* sn = scratch(D / 2);
  for (int64_t b = 0; b < B; ++b)
    for (int64_t s = 0; s < S; ++s) {
      rd_row(cos_t, tab_dt, s * (D / 2), D / 2, cs);
      rd_row(sin_t, tab_dt, s * (D / 2), D / 2, sn);
      for (int64_t h = 0; h < H; ++h) {
        int64_t off = ((b * S + s) * H + h) * D;
        rd_row(x, x_dt, off, D, row);
        rope_row(row, cs, sn, D, sign, out + off);
      }
    }
  free(sn);
  free(cs);
  free(row);
}

/* ---- per-head RMSNorm followed by the rotary embedding ----------------------------------
 * The two kernels of [H] applied one after the other to each head row of q or k. */
void oracle_qknorm_rope_fwd(const void* x, int x_dt, const void* w, int w_dt, const void* cos_t,
                            const void* sin_t, int tab_dt, int64_t B, int64_t S, int64_t H,
                            int64_t D, double eps, int gemma, double* out, double* inv_rms) {
  double* wp = scratch(D);
  double* row = scratch(D);
  double* nrm = scratch(D);
  double* cs = scratch(D / 2);
  double* sn = scratch(D / 2);
  load_weight(w, w_dt, D, gemma, wp);
  for (int64_t b = 0; b < B; ++b)
    for (int64_t s = 0; s < S; ++s) {
      rd_row(cos_t, tab_dt, s * (D / 2), D / 2, cs);
      rd_row(sin_t, tab_dt, s * (D / 2), D / 2, sn);
      for (int64_t h = 0; h < H; ++h) {
        int64_t r = (b * S + s) * H + h;
        rd_row(x, x_dt, r * D, D, row);
        rms_row_fwd(row, wp, D, eps, ORC_ACT_NONE, nrm, inv_rms ? inv_rms + r : NULL);
        if (out) rope_row(nrm, cs, sn, D, +1, out + r * D);
      }
    }
  free(sn);
  free(cs);
  free(nrm);
  free(row);
  free(wp);
}

/* y = R(n(x)) with R an orthogonal rotation, so dL/dn = R^T dy = rope(dy, sign = -1), and the
 * RMSNorm backward takes it from there. */
void oracle_qknorm_rope_bwd(const void* x, int x_dt, const void* w, int w_dt, const void* cos_t,
                            const void* sin_t, int tab_dt, const void* dy, int dy_dt, int64_t B,
                            int64_t S, int64_t H, int64_t D, double eps, int gemma, double* dx,
                            double* dw) {
  double* wp = scratch(D);
  double* row = scratch(D);
  double* grow = scratch(D);
  double* u = scratch(D);
  double* cs = scratch(D / 2);
  double* sn = scratch(D / 2);
  load_weight(w, w_dt, D, gemma, wp);
  if (dw)
    for (int64_t j = 0; j < D; ++j) dw[j] = 0.0;
  for (int64_t b = 0; b < B; ++b)
    for (int64_t s = 0; s < S; ++s) {
      rd_row(cos_t, tab_dt, s * (D / 2), D / 2, cs);
      rd_row(sin_t, tab_dt, s * (D / 2), D / 2, sn);
      for (int64_t h = 0; h < H; ++h) {
        int64_t r = (b * S + s) * H + h;
        rd_row(x, x_dt, r * D, D, row);
        rd_row(dy, dy_dt, r * D, D, grow);
        rope_row(grow, cs, sn, D, -1, u);
        rms_row_bwd(row, wp, u, D, eps, ORC_ACT_NONE, dx ? dx + r * D : NULL, dw);
      }
    }
  free(sn);
  free(cs);
  free(u);
  free(grow);
  free(row);
  free(wp);
}

/* ---- Normalization followed by the linear layer after it -------------------------------------
 * [J] section 4.1: LayerNorm, then a linear projection, then SiLU, in one pass; the HY-Motion
 * optimization page (section 3.1) merges LayerNorm with the matrix multiplication that follows
 * it. Plain reading: xn = the normalized row without an activation (LayerNorm
 * (x - mean) s g + beta, or RMSNorm x r g'), then y[m,n] = act(sum_k xn[k] W[n,k] + bias[n])
 * with W[N,K] the layer's weight (output feature n in row n). */
void oracle_norm_linear(const void* x, int x_dt, const void* g, const void* beta, int p_dt,
                        const void* W, int w_dt, const void* bias, int bias_dt, int64_t M,
                        int64_t N, int64_t K, double eps, int norm, int gemma, int act, double* y,
                        double* mean, double* rstd) {
  double* gv = scratch(K);
  double* bv = scratch(K);
  double* row = scratch(K);
  double* xn = scratch(K);
  double* wt = scratch(N * K);
  if (norm == ORC_NORM_LN) {
    load_affine(g, beta, p_dt, K, gv, bv);
  } else if (norm == ORC_NORM_RMS) {
    load_weight(g, p_dt, K, gemma, gv);
    for (int64_t k = 0; k < K; ++k) bv[k] = 0.0;
  } else {  /* no normalization: xn = x */
    for (int64_t k = 0; k < K; ++k) gv[k] = 1.0, bv[k] = 0.0;
  }
  rd_row(W, w_dt, 0, N * K, wt);
  for (int64_t m = 0; m < M; ++m) {
    rd_row(x, x_dt, m * K, K, row);
    double mu = 0.0, s = 1.0;
    if (norm == ORC_NORM_LN)
      ln_row_stats(row, K, eps, &mu, &s);
    else if (norm == ORC_NORM_RMS)
      s = rms_row_inv(row, K, eps);
    for (int64_t k = 0; k < K; ++k) xn[k] = (row[k] - mu) * s * gv[k] + bv[k];
    if (y)
      for (int64_t n = 0; n < N; ++n) {
        double acc = bias ? rd(bias, bias_dt, n) : 0.0;
        for (int64_t k = 0; k < K; ++k) acc += xn[k] * wt[n * K + k];
        y[m * N + n] = oracle_act(act, acc);
      }
    if (mean) mean[m] = mu;
    if (rstd) rstd[m] = s;
  }
  free(wt);
  free(xn);
  free(row);
  free(bv);
  free(gv);
}

/* ---- Backward of the linear layer with an activation -----------------------------------------
 * [H] "内核三 TiledLinear": the layer y = act(z), z = x W^T + bias runs chunk by chunk along the
 * tokens and its backward recomputes each chunk; chunking changes no arithmetic of the result,
 * so the oracle is the plain gradient: g = dy act'(z), dx = g W, dW = g^T x, dbias = sum_m g.
 * x[M,K], W[N,K], dy[M,N]; dx[M*K], dW[N*K], db[N] may each be NULL. */
void oracle_linear_act_bwd(const void* x, int x_dt, const void* W, int w_dt, const void* bias, int bias_dt,
                           const void* dy, int dy_dt, int64_t M, int64_t N, int64_t K, int act, double* dx,
                           double* dW, double* db) {
  double* wt = scratch(N * K);
  double* row = scratch(K);
  double* gr = scratch(N);
  rd_row(W, w_dt, 0, N * K, wt);
  if (dW)
    for (int64_t i = 0; i < N * K; ++i) dW[i] = 0.0;
  if (db)
    for (int64_t n = 0; n < N; ++n) db[n] = 0.0;
  for (int64_t m = 0; m < M; ++m) {
    rd_row(x, x_dt, m * K, K, row);
    for (int64_t n = 0; n < N; ++n) {
      double z = bias ? rd(bias, bias_dt, n) : 0.0;
      for (int64_t k = 0; k < K; ++k) z += row[k] * wt[n * K + k];
      gr[n] = rd(dy, dy_dt, m * N + n) * oracle_act_grad(act, z);
    }
    if (dx)
      for (int64_t k = 0; k < K; ++k) {
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) acc += gr[n] * wt[n * K + k];
        dx[m * K + k] = acc;
      }
    if (dW)
      for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) dW[n * K + k] += gr[n] * row[k];
    if (db)
      for (int64_t n = 0; n < N; ++n) db[n] += gr[n];
  }
  free(gr);
  free(row);
  free(wt);
}
