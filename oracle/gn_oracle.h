/*
 * gn_oracle.h - plain fp64 CPU oracle for the row-normalization and rotary-embedding path.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the benchmark's
 * CPU-baseline / reference arm call this code. The CUDA library never includes, links or
 * calls it, and it includes nothing of the CUDA library: the two share no code.
 *
 * Every function is the plain definition of the operation, written out as a loop over rows
 * in double precision. Inputs may be float64, float32 or bfloat16 (raw 16-bit patterns);
 * each element is widened to double as it is read. Outputs are always double.
 *
 * Sources (page title, section):
 *   [H]  "Helios 性能优化全解析: 3 个 Triton 自定义内核如何让实时长视频生成提速 16%"
 *        section "内核一 FlashNorm" (one row per block, one load, sum of squares and its
 *        inverse, times the weight; Gemma +1 offset; per-row inverse statistic saved for the
 *        backward) and section "内核二 FlashRoPE" (interleaved even/odd pairs, in-place
 *        rotation; the inverse rotation is the same kernel with sin negated), and section
 *        "内核三 TiledLinear" (linear layer run chunk by chunk along the tokens, the
 *        backward recomputing each chunk).
 *   [L]  "LLM层的优化算子" (optimized kernels for LLM layers), section "编写定制融合算子"
 *        (fused LayerNorm + GeLU example: centre, biased variance, divide by sqrt(var+eps),
 *        times weight plus bias, tanh-GeLU with constant 0.79788456 and cubic 0.044715).
 *   [J]  "Janus-Pro-7B模型推理加速实战", section 4.1 (fused LayerNorm + linear + SiLU,
 *        SiLU = x * sigmoid(x)).
 *   [Y]  "HY-Motion 1.0性能优化从算法到硬件的全方位调优策略", section 3.1 (LayerNorm merged
 *        with the linear layer that follows it).
 *
 * Parity pins: every function here is pinned by the CPU tests (closed forms, invariants,
 * library special cases and central finite differences); none is "parity unpinned".
 */
#ifndef GN_ORACLE_H
#define GN_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element type of an input buffer */
enum { ORC_F64 = 0, ORC_F32 = 1, ORC_BF16 = 2 };

/* epilogue applied to z = normalized * weight (+ bias) */
enum { ORC_ACT_NONE = 0, ORC_ACT_GELU_TANH = 1, ORC_ACT_SILU = 2 };

/* scalar epilogue and its derivative, exposed for the pin tests */
double oracle_act(int act, double z);
double oracle_act_grad(int act, double z);

/* RMSNorm forward over rows x[M,N] (row-major, contiguous).
 * y = act(x * r * w'), r = 1/sqrt(mean(x^2) + eps), w' = w or 1 + w (gemma).
 * y[M*N], inv_rms[M] (= r) may each be NULL. */
void oracle_rmsnorm_fwd(const void* x, int x_dt, const void* w, int w_dt, int64_t M, int64_t N,
                        double eps, int gemma, int act, double* y, double* inv_rms);

/* RMSNorm backward: gradients of sum(dy * y) with respect to x and w.
 * dx[M*N] and dw[N] may each be NULL; dw is overwritten (not accumulated). */
void oracle_rmsnorm_bwd(const void* x, int x_dt, const void* w, int w_dt, const void* dy, int dy_dt,
                        int64_t M, int64_t N, double eps, int gemma, int act, double* dx, double* dw);

/* LayerNorm forward: y = act(((x - mean) * rstd) * w + b), rstd = 1/sqrt(var + eps) with the
 * biased variance. w == NULL means w = 1, b == NULL means b = 0. Any output may be NULL. */
void oracle_layernorm_fwd(const void* x, int x_dt, const void* w, const void* b, int wb_dt,
                          int64_t M, int64_t N, double eps, int act, double* y, double* mean,
                          double* rstd);

/* LayerNorm backward: gradients of sum(dy * y) with respect to x, w and b. Any output may be
 * NULL; dw and db are overwritten. */
void oracle_layernorm_bwd(const void* x, int x_dt, const void* w, const void* b, int wb_dt,
                          const void* dy, int dy_dt, int64_t M, int64_t N, double eps, int act,
                          double* dx, double* dw, double* db);

/* Interleaved rotary embedding of x[B,S,H,D] with tables cos/sin[S, D/2] (table row s serves
 * every batch entry and head at token s). Pair i of a head is (x[2i], x[2i+1]); it is rotated
 * by the angle whose cosine and sine are cos[s,i] and sign*sin[s,i]. sign = +1 is the forward
 * rotation, sign = -1 its inverse (the backward). Out of place: out[B*S*H*D]. */
void oracle_rope(const void* x, int x_dt, const void* cos_t, const void* sin_t, int tab_dt,
                 int64_t B, int64_t S, int64_t H, int64_t D, int sign, double* out);

/* Per-head RMSNorm over D (weight w[D], optional gemma offset) followed by the forward rotary
 * embedding, on x[B,S,H,D]. out[B*S*H*D], inv_rms[B*S*H] may each be NULL. */
void oracle_qknorm_rope_fwd(const void* x, int x_dt, const void* w, int w_dt, const void* cos_t,
                            const void* sin_t, int tab_dt, int64_t B, int64_t S, int64_t H,
                            int64_t D, double eps, int gemma, double* out, double* inv_rms);

/* Backward of oracle_qknorm_rope_fwd: dy is rotated back (sin negated), then the per-head
 * RMSNorm backward. dx[B*S*H*D] and dw[D] may each be NULL; dw is overwritten. */
void oracle_qknorm_rope_bwd(const void* x, int x_dt, const void* w, int w_dt, const void* cos_t,
                            const void* sin_t, int tab_dt, const void* dy, int dy_dt, int64_t B,
                            int64_t S, int64_t H, int64_t D, double eps, int gemma, double* dx,
                            double* dw);

/* which normalization precedes the linear layer (ORC_NORM_NONE: none, a plain linear layer) */
enum { ORC_NORM_RMS = 0, ORC_NORM_LN = 1, ORC_NORM_NONE = 2 };

/* Normalization (RMSNorm with weight g and optional gemma offset, or LayerNorm with weight g and
 * bias beta; no activation) followed by the linear layer y = act(xn W^T + bias): x[M,K],
 * W[N,K] (row n = output feature n), bias[N] or NULL, y[M*N]. mean[M] (LayerNorm; 0 for
 * RMSNorm) and rstd[M] (1/sqrt(var + eps), or the RMSNorm inverse rms) may be NULL. */
void oracle_norm_linear(const void* x, int x_dt, const void* g, const void* beta, int p_dt,
                        const void* W, int w_dt, const void* bias, int bias_dt, int64_t M,
                        int64_t N, int64_t K, double eps, int norm, int gemma, int act, double* y,
                        double* mean, double* rstd);

/* Backward of y = act(x W^T + bias): g = dy act'(z); dx[M*K] = g W; dW[N*K] = g^T x;
 * db[N] = sum over rows of g (each output may be NULL; dW and db are overwritten). */
void oracle_linear_act_bwd(const void* x, int x_dt, const void* W, int w_dt, const void* bias, int bias_dt,
                           const void* dy, int dy_dt, int64_t M, int64_t N, int64_t K, int act, double* dx,
                           double* dW, double* db);

#ifdef __cplusplus
}
#endif
#endif
