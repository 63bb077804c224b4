/*
 * gn.h - C ABI of libgn: fused row normalization and interleaved rotary position embedding
 * for NVIDIA B200 (sm_100a).
 *
 * Sources of the operations (page title, section):
 *   [H] "Helios 性能优化全解析: 3 个 Triton 自定义内核如何让实时长视频生成提速 16%"
 *       - "内核一 FlashNorm": RMSNorm / LayerNorm with mean, variance and scaling in one
 *         memory pass per row, one thread block per row, the per-row inverse statistic saved
 *         by the forward and reused by the backward, a Gemma-style +1 weight offset handled by
 *         a compile-time branch in the same kernel.
 *       - "内核二 FlashRoPE": rotary embedding on an interleaved even/odd layout, pair i read
 *         at offsets 2i and 2i+1, rotated in place without intermediate tensors; the backward
 *         is the same kernel with sin negated.
 *       - "基准实测": FlashNorm and FlashRoPE applied together (the fused qk-norm + RoPE entry
 *         points combine them per attention head).
 *       - "内核三 TiledLinear": a linear layer run chunk by chunk along the tokens, the backward
 *         recomputing each chunk instead of keeping its activations (GN_NORM_NONE and the
 *         plain products below serve it).
 *   [L] "LLM层的优化算子", section "编写定制融合算子": LayerNorm fused with a tanh-GeLU epilogue
 *       (centre, biased variance, divide by sqrt(var + eps), times weight plus bias, GeLU).
 *   [J] "Janus-Pro-7B模型推理加速实战", section 4.1: LayerNorm fused with SiLU = x * sigmoid(x),
 *       and LayerNorm, the first linear projection and SiLU fused into one kernel.
 *   [Y] "HY-Motion 1.0性能优化从算法到硬件的全方位调优策略", section 3.1: LayerNorm merged with
 *       the matrix multiplication that follows it (no round trip of the normalized activations
 *       through memory).
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers owned by the caller, except where stated. The library
 *     allocates nothing, frees nothing and never synchronizes; each call enqueues its kernels
 *     on `stream` (a cudaStream_t; NULL = the legacy default stream) and returns.
 *   - Matrices are row-major. `ld_*` is the distance in ELEMENTS between consecutive rows.
 *     Rotary tensors are contiguous [B, S, H, D]; tables are contiguous fp32 [S, D/2].
 *   - `dt` selects the element type of x, y, dy, dx, w, b, q, k (GN_F32 or GN_BF16).
 *     Saved statistics (inv_rms, mean, rstd), weight gradients and tables are always fp32.
 *   - Arithmetic is fp32 with one round-to-nearest-even per stored bf16 element.
 *   - Arguments are checked before anything is enqueued. A check that fails returns its
 *     status and enqueues nothing:
 *       GN_ERR_NULL         a required pointer is NULL
 *       GN_ERR_SHAPE        a size is negative or zero where it must be positive, ld < hidden,
 *                           D odd or not a multiple of 8, sign not +1/-1
 *       GN_ERR_ALIGN        a row/tensor base pointer or a row stride in bytes is not a
 *                           multiple of 16
 *       GN_ERR_DTYPE        unknown dtype or epilogue
 *       GN_ERR_WORKSPACE    ws is NULL or ws_bytes below the size the *_workspace query gives
 *       GN_ERR_UNSUPPORTED  a row does not fit the kernel's shared-memory stage (see each call)
 *       GN_ERR_CUDA         the CUDA runtime reported an error while querying the device or
 *                           launching (the kernels' own faults surface at the next sync)
 *   - rows == 0 (or B*S*H == 0) is valid once the other sizes check out: nothing is launched,
 *     data pointers may be NULL, and weight gradients that are not NULL are set to zero.
 *   - A kernel never spins without bound: each wait for an asynchronous copy gives up after
 *     one second, records GN_DEVERR_WAIT_TIMEOUT in the device error word (gn_device_error)
 *     and returns.
 *   - Calls are thread-safe and keep no state between calls apart from the launch counter
 *     and the device error word.
 */
#ifndef GN_H
#define GN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GN_OK = 0,
  GN_ERR_NULL = 1,
  GN_ERR_SHAPE = 2,
  GN_ERR_ALIGN = 3,
  GN_ERR_DTYPE = 4,
  GN_ERR_WORKSPACE = 5,
  GN_ERR_UNSUPPORTED = 6,
  GN_ERR_CUDA = 7
} gn_status;

typedef enum { GN_F32 = 0, GN_BF16 = 1 } gn_dtype;

/* epilogue applied to z = normalized * weight (+ bias) before the store */
typedef enum { GN_EPI_NONE = 0, GN_EPI_GELU_TANH = 1, GN_EPI_SILU = 2 } gn_epilogue;

/* the normalization in front of the fused linear layer (GN_NORM_NONE: a plain linear layer) */
typedef enum { GN_NORM_RMS = 0, GN_NORM_LN = 1, GN_NORM_NONE = 2 } gn_norm;

/* device error word bits */
#define GN_DEVERR_WAIT_TIMEOUT 1u

/* Human-readable name of a status. Never NULL. */
const char* gn_status_string(gn_status s);

/* ---------------------------------------------------------------- RMSNorm ([H] FlashNorm)
 * Forward, per row m of x[rows, hidden]:
 *   r = 1 / sqrt(mean_j(x[m,j]^2) + eps)            (eps inside the root)
 *   w'_j = w_j, or 1 + w_j when gemma != 0          (formed in fp32, not rounded to dt)
 *   y[m,j] = epi(x[m,j] * r * w'_j)
 *   inv_rms[m] = r                                  (fp32; may be NULL: not saved)
 * x, y: device, dt, rows of `hidden` elements with strides ld_x, ld_y (16-byte aligned).
 * w: device, dt, [hidden], required. y may alias x when ld_y == ld_x (in place).
 * Limit: hidden <= 16384 (bf16) / 8192 (fp32), else GN_ERR_UNSUPPORTED (each thread keeps
 * its share of the row in registers between the reduction and the store). */
gn_status gn_rmsnorm_fwd(const void* x, const void* w, void* y, float* inv_rms, int64_t rows,
                         int64_t hidden, int64_t ld_x, int64_t ld_y, float eps, int gemma,
                         gn_epilogue epi, gn_dtype dt, void* stream);

/* Workspace in bytes that gn_rmsnorm_bwd needs for these sizes on the current device
 * (per-block fp32 partial sums of dw). 0 on error or when rows == 0. */
size_t gn_rmsnorm_bwd_workspace(int64_t rows, int64_t hidden, gn_dtype dt);

/* Backward of gn_rmsnorm_fwd, reusing the saved inv_rms instead of recomputing it:
 *   z = x r w', g = dy * epi'(z), xhat = x r
 *   dx[m,j] = r * (g_j w'_j - xhat_j * mean_k(g_k w'_k xhat_k))
 *   dw[j]   = sum_m g[m,j] xhat[m,j]            (fp32, deterministic fixed-order reduction;
 *                                              the same for gemma since d w'/d w = 1)
 * inv_rms: fp32 [rows] from the forward (required). dy, dx: dt rows with ld_dy, ld_dx.
 * dw: fp32 [hidden], may be NULL (weight gradient skipped, ws then unused and may be NULL).
 * ws: device scratch of at least gn_rmsnorm_bwd_workspace(rows, hidden, dt) bytes, 16-byte
 * aligned, owned by the caller, contents ignored on entry. dx may alias dy.
 * Limit: hidden <= 8192 (bf16) / 4096 (fp32), else GN_ERR_UNSUPPORTED. */
gn_status gn_rmsnorm_bwd(const void* x, const void* w, const float* inv_rms, const void* dy,
                         void* dx, float* dw, void* ws, size_t ws_bytes, int64_t rows,
                         int64_t hidden, int64_t ld_x, int64_t ld_dy, int64_t ld_dx, int gemma,
                         gn_epilogue epi, gn_dtype dt, void* stream);

/* ---------------------------------------------------------------- LayerNorm ([H] FlashNorm, [L], [J])
 * Forward, per row m:
 *   mu = mean_j x[m,j];  var = mean_j (x[m,j] - mu)^2  (biased);  s = 1 / sqrt(var + eps)
 *   y[m,j] = epi((x[m,j] - mu) * s * w_j + b_j)
 *   mean[m] = mu, rstd[m] = s                          (fp32; each may be NULL)
 * w, b: dt [hidden]; w == NULL means 1, b == NULL means 0. Same layout rules and limits as
 * gn_rmsnorm_fwd. */
gn_status gn_layernorm_fwd(const void* x, const void* w, const void* b, void* y, float* mean,
                           float* rstd, int64_t rows, int64_t hidden, int64_t ld_x, int64_t ld_y,
                           float eps, gn_epilogue epi, gn_dtype dt, void* stream);

size_t gn_layernorm_bwd_workspace(int64_t rows, int64_t hidden, gn_dtype dt);

/* Backward of gn_layernorm_fwd from the saved mean and rstd:
 *   xhat = (x - mu) s, z = xhat w + b, g = dy * epi'(z)
 *   dx[m,j] = s * (g_j w_j - mean_k(g_k w_k) - xhat_j * mean_k(g_k w_k xhat_k))
 *   dw[j] = sum_m g xhat,  db[j] = sum_m g         (fp32; each may be NULL)
 * mean, rstd: fp32 [rows], required. b is read only to recompute z for an epilogue.
 * ws as for gn_rmsnorm_bwd (may be NULL when dw and db are both NULL). */
gn_status gn_layernorm_bwd(const void* x, const void* w, const void* b, const float* mean,
                           const float* rstd, const void* dy, void* dx, float* dw, float* db,
                           void* ws, size_t ws_bytes, int64_t rows, int64_t hidden, int64_t ld_x,
                           int64_t ld_dy, int64_t ld_dx, gn_epilogue epi, gn_dtype dt,
                           void* stream);

/* ---------------------------------------------------------------- RoPE ([H] FlashRoPE)
 * In-place rotary embedding of q and (optionally) k, both contiguous [B, S, H, D] of dt.
 * For every (b, s, h) and pair i < D/2, with c = cos[s, i], t = sign * sin[s, i]:
 *   (x[2i], x[2i+1]) <- (x[2i] c - x[2i+1] t,  x[2i] t + x[2i+1] c)
 * cos, sin: fp32 [S, D/2], row s serving token s of every batch entry and head.
 * sign = +1: forward rotation; sign = -1: its inverse, which is the backward (apply it to
 * dq, dk in place). k may be NULL. D must be even and a multiple of 8. */
gn_status gn_rope_apply_inplace(void* q, void* k, const float* cos, const float* sin, int64_t B,
                                int64_t S, int64_t H, int64_t D, int sign, gn_dtype dt,
                                void* stream);

/* ---------------------------------------------------------------- qk-norm + RoPE ([H] FlashNorm + FlashRoPE)
 * For q (and k when not NULL), contiguous [B, S, H, D] of dt, per head row (b, s, h):
 *   r = 1 / sqrt(mean_d x_d^2 + eps); n_d = x_d r w'_d   (w' = w or 1 + w with gemma)
 *   out = rope(n, cos[s], sin[s], +1)                      (out of place)
 *   inv_rms[b, s, h] = r                                   (fp32 [B, S, H]; may be NULL)
 * wq, wk: dt [D] (one weight per tensor shared by all heads). D/8 (bf16) or D/4 (fp32) must
 * be a power of two <= 32 (D in {8,...,256} bf16, {8,...,128} fp32), else
 * GN_ERR_UNSUPPORTED. */
gn_status gn_qknorm_rope_fwd(const void* q, const void* k, const void* wq, const void* wk,
                             const float* cos, const float* sin, void* q_out, void* k_out,
                             float* inv_rms_q, float* inv_rms_k, int64_t B, int64_t S, int64_t H,
                             int64_t D, float eps, int gemma, gn_dtype dt, void* stream);

size_t gn_qknorm_rope_bwd_workspace(int64_t B, int64_t S, int64_t H, int64_t D, gn_dtype dt);

/* Backward of gn_qknorm_rope_fwd from the pre-norm inputs and the saved inv_rms:
 *   u = rope(dy, cos[s], sin[s], -1)                       (inverse rotation of the gradient)
 *   dx_d = r (u_d w'_d - xhat_d mean_e(u_e w'_e xhat_e)),  xhat = x r
 *   dw_d = sum over all head rows of u_d xhat_d            (fp32, fixed-order reduction)
 * dq_out, dk_out: gradients of q_out, k_out (dt). dq, dk: outputs (dt, may alias dq_out /
 * dk_out). dwq, dwk: fp32 [D], may be NULL. ws as for gn_rmsnorm_bwd. */
gn_status gn_qknorm_rope_bwd(const void* q, const void* k, const void* wq, const void* wk,
                             const float* cos, const float* sin, const float* inv_rms_q,
                             const float* inv_rms_k, const void* dq_out, const void* dk_out,
                             void* dq, void* dk, float* dwq, float* dwk, void* ws,
                             size_t ws_bytes, int64_t B, int64_t S, int64_t H, int64_t D,
                             int gemma, gn_dtype dt, void* stream);

/* gn_qknorm_rope_bwd without a workspace argument, for callers that cannot allocate device
 * memory: for example code running inside another framework's callback or plugin whose
 * device memory is owned and budgeted by that framework, or a process whose whole memory is
 * reserved by another allocator. The source pages have no counterpart of this call; it only
 * changes where the per-block weight-gradient partials live.
 * Arguments, results and errors are those of gn_qknorm_rope_bwd. The library allocates
 * nothing for it: the partials go to a fixed 1 MiB array inside the library (256-byte
 * aligned) that every GPU which loads the library holds until the process exits. A call
 * that would need more (2 * D * 4 bytes per block of the persistent grid, e.g. more than
 * 1024 blocks at D = 128) returns GN_ERR_WORKSPACE; use gn_qknorm_rope_bwd then.
 * The first call on a device looks up that array's device address (cudaGetSymbolAddress)
 * with the device current and caches it: make that first call before any stream capture.
 * All calls share the array, so calls whose kernels overlap on the GPU (other streams,
 * other threads) race on it and must be serialised by the caller. Nothing in the array has
 * to start at zero: each call writes every partial it later reads. */
gn_status gn_qknorm_rope_bwd_noalloc(const void* q, const void* k, const void* wq,
                                     const void* wk, const float* cos, const float* sin,
                                     const float* inv_rms_q, const float* inv_rms_k,
                                     const void* dq_out, const void* dk_out, void* dq, void* dk,
                                     float* dwq, float* dwk, int64_t B, int64_t S, int64_t H,
                                     int64_t D, int gemma, gn_dtype dt, void* stream);

/* ---- normalization + linear layer on the tensor cores ([J] section 4.1, [Y] section 3.1) ----
 * y[m,n] = act( sum_k xn[m,k] W[n,k] + bias[n] ) with xn the normalized row of x[M,K]:
 *   GN_NORM_LN : xn = (x - mean) rstd g + beta   (biased variance, rstd = 1/sqrt(var + eps))
 *   GN_NORM_RMS: xn = x rstd g',  g' = g or 1 + g (gemma),  rstd = 1/sqrt(mean(x^2) + eps)
 * The normalization is folded into the layer instead of being materialised: the forward
 * multiplies the raw x by Wf = bf16(g' W) on the tcgen05 tensor cores and corrects each output
 * with the row statistics, which it accumulates from the same x tiles:
 *   y[m,n] = act( rstd_m (x Wf^T)[m,n] - rstd_m mean_m c[n] + d[n] ),
 *   c[n] = sum_k Wf[n,k],  d[n] = sum_k beta[k] W[n,k] + bias[n]   (RMSNorm: mean = 0, d = bias).
 * GN_NORM_NONE: no normalization, y = act(x W^T + bias) (a plain linear layer on the tensor
 * cores; g, beta, c, mean and rstd are not used).
 * bf16 only (GN_BF16; GN_F32 returns GN_ERR_UNSUPPORTED). */

/* Builds Wf [N, K] (bf16, row n = output feature n, contiguous), c [N] fp32 (LayerNorm; may be
 * NULL for RMSNorm) and d [N] fp32 (may be NULL when beta and bias are both absent) from the
 * layer weight W [N, K] (bf16, contiguous), the norm weight g [K] (NULL = ones), the LayerNorm
 * bias beta [K] (NULL = zeros; ignored for RMSNorm) and the layer bias [N] (NULL = zeros), all
 * bf16. Run it once per weight update; Wf, c and d are then read by every forward. The sums run
 * in a fixed order: the results are the same on every run.
 * Errors: GN_ERR_NULL (W, Wf, or c for LayerNorm), GN_ERR_SHAPE (N < 0, K <= 0, unknown norm). */
gn_status gn_norm_linear_prepare(const void* W, const void* g, const void* beta, const void* bias,
                                 void* Wf, float* c, float* d, int64_t N, int64_t K, gn_norm norm,
                                 int gemma, gn_dtype dt, void* stream);

/* Forward: y [M, N] (bf16, row stride ldy) from x [M, K] (bf16, row stride ldx) and the
 * prepared Wf, c, d. mean [M] (LayerNorm; may be NULL for RMSNorm) and rstd [M] (fp32) receive
 * the row statistics and are required: beyond 128 rows and 256 columns a streaming pre-pass
 * writes them and the matrix kernel (pairs of SMs, 256 x 512 tiles) reads them back; below that
 * one kernel computes them from its own tiles. K, ldx and ldy must be multiples of 8; x, Wf, y, c
 * and d 16-byte aligned; M up to 8388480. Ragged M, N and K are handled.
 * Errors: GN_ERR_SHAPE (sizes, strides, norm), GN_ERR_DTYPE (epilogue), GN_ERR_ALIGN,
 * GN_ERR_NULL (x, Wf, y, rstd, or c and mean for LayerNorm), GN_ERR_CUDA (tensor-map encoding
 * or launch). M == 0 or N == 0: nothing is launched. */
gn_status gn_norm_linear_fwd(const void* x, const void* Wf, const float* c, const float* d, void* y,
                             float* mean, float* rstd, int64_t M, int64_t N, int64_t K, int64_t ldx,
                             int64_t ldy, float eps, gn_norm norm, gn_epilogue epi, gn_dtype dt,
                             void* stream);

/* ---- TiledLinear backward ([H] "内核三 TiledLinear": per chunk of tokens the backward recomputes
 * the pre-activation z = x W^T + b, forms dz = dy * act'(z), then dx = dz W, dW += dz^T x,
 * db += sum dz; the calls below run these steps on this library's kernels) ---- */

/* dz [M, N] = dy [M, N] * act'(x [M, K] Wf^T + d): the chunk's recompute on the tensor-core
 * kernels (as gn_norm_linear_fwd with GN_NORM_NONE) with the activation gradient applied where the
 * accumulators are read back, so z is never written. Wf [N, K] from gn_norm_linear_prepare
 * (GN_NORM_NONE), d [N] fp32 (may be NULL = 0). bf16 only. Row strides ldx, lddy, lddz in
 * elements, multiples of 8; K a multiple of 8; x, Wf, dy, dz, d 16-byte aligned.
 * Errors: GN_ERR_SHAPE, GN_ERR_DTYPE (epilogue), GN_ERR_NULL, GN_ERR_ALIGN, GN_ERR_UNSUPPORTED
 * (fp32), GN_ERR_CUDA. M == 0 or N == 0: nothing is launched. */
gn_status gn_linear_act_grad(const void* x, const void* Wf, const float* d, const void* dy, void* dz,
                             int64_t M, int64_t N, int64_t K, int64_t ldx, int64_t lddy, int64_t lddz,
                             gn_epilogue epi, gn_dtype dt, void* stream);

/* Operand layouts of the plain products below. GN_K_MAJOR: A as [M, K], B as [N, K], the
 * contraction index contiguous (row strides lda >= K, ldb >= K; K a multiple of 8). GN_MN_MAJOR:
 * the operand stored transposed, A as [K, M], B as [K, N] (row strides lda >= M, ldb >= N; K
 * free). The weight gradient dW = dz^T x contracts over the tokens, the rows of dz [tokens, N]
 * and x [tokens, K]: both operands are MN-major there; dx = dz W reads W [N, K] as an MN-major
 * B. Row strides are multiples of 8 elements in either layout. */
typedef enum { GN_K_MAJOR = 0, GN_MN_MAJOR = 1 } gn_layout;

/* y [M, N] = A B^T (+ d) in bf16 (fp32 accumulation on the tensor-core kernels; d [N] fp32, may
 * be NULL = 0). ldy >= N, a multiple of 8; A, B, y, d 16-byte aligned.
 * Errors: GN_ERR_SHAPE (sizes, strides, layout values), GN_ERR_NULL, GN_ERR_ALIGN,
 * GN_ERR_UNSUPPORTED (fp32), GN_ERR_CUDA. M == 0 or N == 0: nothing is launched. */
gn_status gn_linear_bf16(const void* A, const void* B, const float* d, void* y, int64_t M, int64_t N,
                         int64_t K, int64_t lda, int64_t ldb, int64_t ldy, gn_layout a_layout,
                         gn_layout b_layout, gn_dtype dt, void* stream);

/* C [M, N] += A B^T with C fp32, updated in place (a weight gradient summed over token chunks:
 * no partial is rounded), A and B bf16 in the given layouts, on the tensor-core kernels. ldc >=
 * N, a multiple of 4; A, B, C 16-byte aligned. Errors as gn_linear_bf16. */
gn_status gn_linear_acc_f32(const void* A, const void* B, float* C, int64_t M, int64_t N, int64_t K,
                            int64_t lda, int64_t ldb, int64_t ldc, gn_layout a_layout,
                            gn_layout b_layout, gn_dtype dt, void* stream);

/* Column sums of a bf16 matrix src [rows, cols] (row stride ld; cols and ld even; src 4-byte
 * aligned) into fp32 out [cols]: out = sum (accumulate == 0) or out += sum (accumulate != 0), in
 * a fixed order (the same bits on every run): 64 row slices summed into the caller's workspace
 * ws (gn_colsum_bf16_workspace(cols) bytes, 16-byte aligned), then the slices in order.
 * Errors: GN_ERR_SHAPE, GN_ERR_NULL, GN_ERR_ALIGN, GN_ERR_WORKSPACE, GN_ERR_UNSUPPORTED (fp32),
 * GN_ERR_CUDA. */
size_t gn_colsum_bf16_workspace(int64_t cols);
gn_status gn_colsum_bf16(const void* src, float* out, void* ws, size_t ws_bytes, int64_t rows,
                         int64_t cols, int64_t ld, int accumulate, gn_dtype dt, void* stream);

/* Gradient of the epilogue activation, elementwise over n elements: dz = dy * act'(z) (act as
 * in the gn_epilogue values; GN_EPI_NONE gives dz = dy). z is the pre-activation, dy the
 * gradient of act(z): the step between a layer's activation and its gradient products, for a
 * caller that holds z. (The token-chunked layer never stores z: gn_linear_act_grad applies the
 * same derivative where its recompute reads the accumulators back.) z, dy, dz: contiguous, dt,
 * 16-byte aligned; dz may alias z or dy (elementwise).
 * Errors: GN_ERR_DTYPE, GN_ERR_SHAPE (n < 0), GN_ERR_NULL, GN_ERR_ALIGN, GN_ERR_CUDA. */
gn_status gn_act_grad(const void* z, const void* dy, void* dz, int64_t n, gn_epilogue epi, gn_dtype dt,
                      void* stream);

/* The epilogue activation, elementwise over n elements: y = act(z) (act as in the gn_epilogue
 * values: tanh-GeLU of "LLM层的优化算子" section "编写定制融合算子", SiLU of the Janus-Pro-7B
 * article section 4.1; GN_EPI_NONE copies). For a caller that keeps the pre-activation z of a
 * linear layer for its backward (gn_act_grad then forms dz from it) instead of recomputing it:
 * gn_norm_linear_fwd with GN_EPI_NONE writes z, this call y. z, y: contiguous, dt, 16-byte aligned;
 * y may alias z (in place).
 * Errors: GN_ERR_DTYPE, GN_ERR_SHAPE (n < 0), GN_ERR_NULL, GN_ERR_ALIGN, GN_ERR_CUDA. */
gn_status gn_act_fwd(const void* z, void* y, int64_t n, gn_epilogue epi, gn_dtype dt, void* stream);

/* ---------------------------------------------------------------- runtime queries
 * Number of kernels this process has launched through libgn (all devices, all threads). */
uint64_t gn_launch_count(void);

/* Reads (and with clear != 0 then zeroes) the device error word of the current device into
 * *word. Synchronizes the device. GN_ERR_NULL if word is NULL, GN_ERR_CUDA on a runtime
 * error. */
gn_status gn_device_error(unsigned* word, int clear);

/* Self-test of the bounded waits (no counterpart on the source pages): enqueues a one-thread
 * kernel that waits on an mbarrier phase nothing completes, gives up after limit_us
 * microseconds (1 .. 1000000), sets GN_DEVERR_WAIT_TIMEOUT in the device error word and
 * returns, leaving the context usable. GN_ERR_SHAPE for a limit out of range. */
gn_status gn_selftest_wait_timeout(uint32_t limit_us, void* stream);

/* Tuning knobs of the launch planner, for benchmarking sweeps. key is one of "stages",
 * "ctas_per_sm", "vpt", "unit_bytes", "group_rows", "fwd_warps" (warps per CTA of the
 * one-warp-per-row norm forward, at most 20), "fwd_path" (norm forward of long rows: 1 = the
 * CTA-per-row pipeline, 2 = one warp per row with two-pass LayerNorm statistics, 3 = one warp per
 * row with one shifted pass; by default RMSNorm takes the first and LayerNorm the third);
 * value 0 restores the default. Returns
 * GN_ERR_SHAPE for an unknown key or a value out of range. Not thread-safe with concurrent
 * launches. */
gn_status gn_tune(const char* key, int value);

#ifdef __cplusplus
}
#endif
#endif /* GN_H */
