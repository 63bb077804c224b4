// layernorm.cu - LayerNorm forward and backward with an optional tanh-GeLU or SiLU epilogue
// (Helios kernels article, section "内核一 FlashNorm": mean, variance and scaling in one
// memory pass per row, statistics saved for the backward; "LLM层的优化算子", section
// "编写定制融合算子": centre, biased variance, divide by sqrt(var + eps), times weight plus
// bias, tanh-GeLU in the same kernel; Janus-Pro-7B article section 4.1: SiLU epilogue).
//
//   forward : mu = mean(x), var = mean((x - mu)^2), s = rsqrt(var + eps),
//             y = epi((x - mu) s w + b), mean = mu, rstd = s
//   backward: xhat = (x - mu) s, g = dy epi'(xhat w + b),
//             dx = s (g w - mean(g w) - xhat mean(g w xhat)), dw = sum g xhat, db = sum g
//
// The row is read from HBM once and kept in registers, so the variance is taken around the
// mean (no E[x^2] - E[x]^2 cancellation): the long-row kernel reduces the sum, then the
// centred sum of squares (two barriers over the consumer warps); the short-row kernel forms
// (count, mean, M2) per thread and combines the triples with Chan et al.'s pairwise update.
#include "norm_plan.h"
#include "norm_rows.cuh"

namespace gn {
namespace {

struct LnFwdArgs {
  const void* x;
  const void* w;
  const void* b;
  void* y;
  float* mean;
  float* rstd;
  int64_t rows;
  int64_t ldx, ldy;
  int N;
  float eps;
  int stages;
  unsigned* err;
};

struct LnBwdArgs {
  const void* x;
  const void* w;
  const void* b;
  const float* mean;
  const float* rstd;
  const void* dy;
  void* dx;
  float* ws;  // [gridDim.x, 2N]: dw partials then db partials, or null
  int64_t rows;
  int64_t ldx, lddy, lddx;
  int N;
  int stages;
  unsigned* err;
};

// Chan et al. pairwise combination of (count, mean, M2) summaries.
__device__ __forceinline__ void chan_merge(float& n, float& m, float& M2, float nb, float mb, float M2b) {
  if (nb == 0.0f) return;
  if (n == 0.0f) {
    n = nb;
    m = mb;
    M2 = M2b;
    return;
  }
  const float nn = n + nb;
  const float d = mb - m;
  const float f = __fdividef(nb, nn);
  m = fmaf(d, f, m);
  M2 = M2 + M2b + d * d * n * f;
  n = nn;
}

// Summary of this thread's elements of the row: xv[j][0..E) valid for the first cnt[j].
template <int VPT, int E>
__device__ __forceinline__ void thread_stats(const float (&xv)[VPT][E], const int (&cnt)[VPT], float& n,
                                             float& m, float& M2) {
  float s = 0.0f;
  int c = 0;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
#pragma unroll
    for (int e = 0; e < E; ++e) s += xv[j][e];  // invalid elements are 0
    c += cnt[j];
  }
  n = (float)c;
  m = c ? s / (float)c : 0.0f;
  float q = 0.0f;
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float d = xv[j][e] - m;
      q = e < cnt[j] ? fmaf(d, d, q) : q;
    }
  M2 = q;
}

// tree-combine the summaries of a group of `width` lanes into its first lane
__device__ __forceinline__ void group_stats(float& n, float& m, float& M2, int width) {
  const int li = threadIdx.x & (width - 1);
  for (int off = width / 2; off > 0; off >>= 1) {
    const float nb = __shfl_down_sync(0xffffffffu, n, off, width);
    const float mb = __shfl_down_sync(0xffffffffu, m, off, width);
    const float qb = __shfl_down_sync(0xffffffffu, M2, off, width);
    if (li < off) chan_merge(n, m, M2, nb, mb, qb);
  }
}

template <typename T, int VPT>
__device__ __forceinline__ void load_affine(const LnFwdArgs& a, int base, int stride, float (&wr)[VPT][Vec<T>::N],
                                            float (&br)[VPT][Vec<T>::N]) {
  constexpr int E = Vec<T>::N;
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int col = (base + j * stride) * E + e;
      const bool in = col < a.N;
      wr[j][e] = in ? ld_param(static_cast<const T*>(a.w), col, 1.0f) : 0.0f;
      br[j][e] = in ? ld_param(static_cast<const T*>(a.b), col, 0.0f) : 0.0f;
    }
}

// ---------------------------------------------------------------- CTA path (long rows)
// Warp 0 produces (row_pipe.cuh); warps 1.. consume. Consumer thread ct owns the vectors
// v = ct + j * nct (j < VPT) of every row. Weight and bias live in shared memory. The
// arithmetic runs on element pairs with packed fp32x2 instructions.


template <typename T, int VPT, int EPI>
__global__ void __launch_bounds__(kNormCtaThreads, norm_min_blocks(VPT)) ln_fwd_cta(const LnFwdArgs a) {
  constexpr int E = Vec<T>::N, H = E / 2;
  constexpr bool FAST = fast_math_for<T>();
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int N = a.N, nfull = N / E, nvec = (N + E - 1) / E;
  const RowPipe pipe(smem, a.stages, 1, 2, N, sizeof(T), sizeof(T));
  const T* x = static_cast<const T*>(a.x);
  T* y = static_cast<T*>(a.y);
  const int ncw = (int)(blockDim.x >> 5) - 1;
  if (tid == 0) pipe.init(ncw);
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) pipe.produce(a.rows, [&](int64_t m, int) -> const void* { return x + m * a.ldx; }, a.err);
    return;
  }
  const int ct = tid - 32, nct = ncw * 32, cw = warp - 1;
  // with the tanh-GeLU epilogue the weight and bias are staged halved (exact): the affine map
  // then yields z / 2, which gelu_of_half2 takes directly
  constexpr float kParamScale = EPI == EPI_GELU_TANH ? 0.5f : 1.0f;
  stage_param<T, VPT>(pipe.param(0), static_cast<const T*>(a.w), N, nvec, 1.0f, ct, nct, kParamScale);
  stage_param<T, VPT>(pipe.param(1), static_cast<const T*>(a.b), N, nvec, 0.0f, ct, nct, kParamScale);
  pipe.red_zero(ct, nct);
  consumers_sync(nct);
  int cnt[VPT];
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int left = N - (ct + j * nct) * E;
    cnt[j] = left <= 0 ? 0 : left >= E ? E : left;
  }
  const float inv_n = 1.0f / (float)N;
  const int64_t step = gridDim.x;
  int s = 0;
  uint32_t ph = 0, rb = 0;
  for (int64_t m = blockIdx.x; m < a.rows; m += step) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&pipe.full[s], ph, a.err));
    float2 xv[VPT][H];
    float2 sx2 = dup2(0.0f);
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      load_pairs<T>(pipe.at(s, 0), x + m * a.ldx, ct + j * nct, nfull, N, ok, xv[j]);
#pragma unroll
      for (int h = 0; h < H; ++h) sx2 = add2(sx2, xv[j][h]);  // invalid elements are 0
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&pipe.empty[s]);
    // two reductions over the register-resident row: the mean, then the sum of squares
    // around it (no E[x^2] - E[x]^2 cancellation); invalid elements are masked
    const float sx = group_sum<32>(sx2.x + sx2.y);
    if (lane == 0) pipe.red_at(rb, 0)[cw] = sx;
    if (consumers_sync_or(nct, !ok)) return;
    const float mu = pipe.red_sum(rb, 0, ncw) * inv_n;
    const float2 nmu = dup2(-mu);
    float2 q2 = dup2(0.0f);
    float qt = 0.0f;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      if (cnt[j] == E) {
#pragma unroll
        for (int h = 0; h < H; ++h) {
          const float2 d = add2(xv[j][h], nmu);
          q2 = fma2(d, d, q2);
        }
      } else {
#pragma unroll
        for (int h = 0; h < H; ++h) {
          const float d0 = xv[j][h].x - mu, d1 = xv[j][h].y - mu;
          qt = 2 * h < cnt[j] ? fmaf(d0, d0, qt) : qt;
          qt = 2 * h + 1 < cnt[j] ? fmaf(d1, d1, qt) : qt;
        }
      }
    }
    const float q = group_sum<32>(q2.x + q2.y + qt);
    if (lane == 0) pipe.red_at(rb, 1)[cw] = q;
    consumers_sync(nct);
    const float tq = pipe.red_sum(rb, 1, ncw);
    rb ^= 1u;
    if (++s == a.stages) s = 0, ph ^= 1u;
    const float rs = rsqrtf(fmaf(tq, inv_n, a.eps));
    // centre, then scale: (x - mu) s keeps near-constant rows (large s) exact where the fused
    // x s - mu s would round mu s
    const float2 rs2 = dup2(rs);
    T* yrow = y + m * a.ldy;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = ct + j * nct;
      if (v < nvec) {
        float2 wv[H], bv[H], o[H];
        param_pairs<T>(pipe.param(0), v, wv);
        param_pairs<T>(pipe.param(1), v, bv);
#pragma unroll
        for (int h = 0; h < H; ++h) {
          const float2 z = fma2(mul2(add2(xv[j][h], nmu), rs2), wv[h], bv[h]);
          if constexpr (EPI == EPI_GELU_TANH)
            o[h] = gelu_of_half2<FAST>(z);
          else
            o[h] = epi_fwd2<EPI, FAST>(z);
        }
        store_pairs<T>(yrow, v, nfull, N, o);
      }
    }
    if (ct == 0) {
      if (a.mean) a.mean[m] = mu;
      if (a.rstd) a.rstd[m] = rs;
    }
  }
}

template <typename T, int VPT, int EPI>
__global__ void __launch_bounds__(kNormCtaThreads, norm_min_blocks(VPT, true)) ln_bwd_cta(const LnBwdArgs a) {
  pdl_launch_dependents();  // the column reduction that follows may launch early
  constexpr int E = Vec<T>::N, H = E / 2;
  constexpr bool FAST = fast_math_for<T>();
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int N = a.N, nfull = N / E, nvec = (N + E - 1) / E;
  const RowPipe pipe(smem, a.stages, 2, 2, N, sizeof(T), 4);
  const T* x = static_cast<const T*>(a.x);
  const T* dy = static_cast<const T*>(a.dy);
  T* dx = static_cast<T*>(a.dx);
  const int ncw = (int)(blockDim.x >> 5) - 1;
  if (tid == 0) pipe.init(ncw);
  __syncthreads();
  if (warp == 0) {
    if (lane == 0)
      pipe.produce(
          a.rows,
          [&](int64_t m, int t) -> const void* { return t == 0 ? (const void*)(x + m * a.ldx) : (const void*)(dy + m * a.lddy); },
          a.err);
    return;
  }
  const int ct = tid - 32, nct = ncw * 32, cw = warp - 1;
  // weight and bias as fp32: the per-row passes read them with no conversion
  const float* pw = reinterpret_cast<const float*>(pipe.param(0));
  const float* pb = reinterpret_cast<const float*>(pipe.param(1));
  stage_param_f32<T, VPT>(const_cast<float*>(pw), static_cast<const T*>(a.w), N, nvec, 0.0f, 1.0f, 1.0f, ct, nct);
  stage_param_f32<T, VPT>(const_cast<float*>(pb), static_cast<const T*>(a.b), N, nvec, 0.0f, 1.0f, 0.0f, ct, nct);
  pipe.red_zero(ct, nct);
  consumers_sync(nct);
  float2 dwa[VPT][H], dba[VPT][H];
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int h = 0; h < H; ++h) dwa[j][h] = dba[j][h] = dup2(0.0f);
  const float inv_n = 1.0f / (float)N;
  const int64_t step = gridDim.x;
  int s = 0;
  uint32_t ph = 0, rb = 0;
  bool failed = false;
  // the statistics of the next row are loaded one row ahead: their global-memory latency
  // then overlaps the current row instead of stalling the start of the next
  float mu_n = 0.0f, rs_n = 0.0f;
  if (blockIdx.x < a.rows) mu_n = __ldg(a.mean + blockIdx.x), rs_n = __ldg(a.rstd + blockIdx.x);
  for (int64_t m = blockIdx.x; m < a.rows; m += step) {
    const float mu = mu_n, rs = rs_n;
    if (m + step < a.rows) mu_n = __ldg(a.mean + m + step), rs_n = __ldg(a.rstd + m + step);
    // centre, then scale (as the forward): (x - mu) s
    const float2 rs2 = dup2(rs), nmu2 = dup2(-mu);
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&pipe.full[s], ph, a.err));
    uint4 xr[VPT];  // x stays packed between the two phases (unpacked on use)
    float2 gv[VPT][H];
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = ct + j * nct;
      xr[j] = load_raw<T>(pipe.at(s, 0), x + m * a.ldx, v, nfull, N, ok);
      load_pairs<T>(pipe.at(s, 1), dy + m * a.lddy, v, nfull, N, ok, gv[j]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&pipe.empty[s]);
    float2 s12 = dup2(0.0f), s22 = dup2(0.0f);
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = ct + j * nct;
      const int vv = v < nvec ? v : 0;
      float2 wv[H], bv[H], xv[H];
      prm_pairs<H>(pw, vv, nvec, wv);
      prm_pairs<H>(pb, vv, nvec, bv);
      unpack2<T>(xr[j], xv);
#pragma unroll
      for (int h = 0; h < H; ++h) {
        const float2 xh = mul2(add2(xv[h], nmu2), rs2);
        const float2 g = EPI == EPI_NONE ? gv[j][h] : mul2(gv[j][h], epi_grad2<EPI, FAST>(fma2(xh, wv[h], bv[h])));
        const float2 gw = mul2(g, wv[h]);
        gv[j][h] = gw;  // phase 2 needs only g w
        s12 = add2(s12, gw);
        s22 = fma2(gw, xh, s22);
        dwa[j][h] = fma2(g, xh, dwa[j][h]);
        dba[j][h] = add2(dba[j][h], g);
      }
    }
    const float s1 = group_sum<32>(s12.x + s12.y);
    const float s2 = group_sum<32>(s22.x + s22.y);
    if (lane == 0) pipe.red_at(rb, 0)[cw] = s1, pipe.red_at(rb, 1)[cw] = s2;
    if (consumers_sync_or(nct, !ok)) {
      failed = true;
      break;
    }
    const float t1 = pipe.red_sum(rb, 0, ncw), t2 = pipe.red_sum(rb, 1, ncw);
    rb ^= 1u;
    if (++s == a.stages) s = 0, ph ^= 1u;
    const float2 nc1 = dup2(-t1 * inv_n), nc2 = dup2(-t2 * inv_n);
    T* dxrow = dx + m * a.lddx;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = ct + j * nct;
      if (v < nvec) {
        float2 xv[H], o[H];
        unpack2<T>(xr[j], xv);
#pragma unroll
        for (int h = 0; h < H; ++h) o[h] = mul2(rs2, add2(gv[j][h], fma2(mul2(add2(xv[h], nmu2), rs2), nc2, nc1)));
        store_pairs<T>(dxrow, v, nfull, N, o);
      }
    }
  }
  if (a.ws && !failed) {
    float* part = a.ws + (int64_t)blockIdx.x * 2 * N;
#pragma unroll
    for (int j = 0; j < VPT; ++j)
#pragma unroll
      for (int h = 0; h < H; ++h) {
        const int col = (ct + j * nct) * E + 2 * h;
        if (col < N) {
          part[col] = dwa[j][h].x;
          part[N + col] = dba[j][h].x;
        }
        if (col + 1 < N) {
          part[col + 1] = dwa[j][h].y;
          part[N + col + 1] = dba[j][h].y;
        }
      }
  }
}

// ---------------------------------------------------------------- group path (short rows)

template <typename T, int VPT, int EPI>
__global__ void __launch_bounds__(kGroupThreads) ln_fwd_grp(const LnFwdArgs a, int lanes) {
  using V = Vec<T>;
  constexpr int E = V::N;
  constexpr bool FAST = fast_math_for<T>();
  const int N = a.N, nfull = N / E, nvec = (N + E - 1) / E;
  const int li = threadIdx.x % lanes, gi = threadIdx.x / lanes;
  const int64_t gpc = kGroupThreads / lanes;
  const int64_t gstep = (int64_t)gridDim.x * gpc;
  const T* x = static_cast<const T*>(a.x);
  T* y = static_cast<T*>(a.y);
  float wr[VPT][E], br[VPT][E];
  load_affine<T, VPT>(a, li, lanes, wr, br);
  int cnt[VPT];
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int left = N - (li + j * lanes) * E;
    cnt[j] = left <= 0 ? 0 : left >= E ? E : left;
  }
  const float inv_n = 1.0f / (float)N;
  for (int64_t m0 = (int64_t)blockIdx.x * gpc; m0 < a.rows; m0 += gstep) {
    const int64_t m = m0 + gi;
    const bool live = m < a.rows;
    const T* xrow = x + (live ? m : 0) * a.ldx;
    float xv[VPT][E];
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = li + j * lanes;
      if (live && v < nfull) {
        V::unpack(ld_stream(xrow + (size_t)v * E), xv[j]);
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) xv[j][e] = (live && e < cnt[j]) ? V::load1(xrow + v * E + e) : 0.0f;
      }
    }
    float n, mu, M2;
    thread_stats<VPT, E>(xv, cnt, n, mu, M2);
    group_stats(n, mu, M2, lanes);
    mu = __shfl_sync(0xffffffffu, mu, 0, lanes);
    M2 = __shfl_sync(0xffffffffu, M2, 0, lanes);
    if (!live) continue;
    const float rs = rsqrtf(fmaf(M2, inv_n, a.eps));
    T* yrow = y + m * a.ldy;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = li + j * lanes;
      if (v < nvec) {
        float o[E];
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = epi_fwd<EPI, FAST>(fmaf((xv[j][e] - mu) * rs, wr[j][e], br[j][e]));
        if (v < nfull) {
          st_stream(yrow + (size_t)v * E, V::pack(o));
        } else {
#pragma unroll
          for (int e = 0; e < E; ++e)
            if (e < cnt[j]) V::store1(yrow + v * E + e, o[e]);
        }
      }
    }
    if (li == 0) {
      if (a.mean) a.mean[m] = mu;
      if (a.rstd) a.rstd[m] = rs;
    }
  }
}

template <typename T, int VPT, int EPI>
__global__ void __launch_bounds__(kGroupThreads) ln_bwd_grp(const LnBwdArgs a, int lanes) {
  pdl_launch_dependents();  // the column reduction that follows may launch early
  using V = Vec<T>;
  constexpr int E = V::N;
  constexpr bool FAST = fast_math_for<T>();
  extern __shared__ __align__(16) float gsm[];  // [groups per CTA][2N] dw, db partials
  const int N = a.N, nfull = N / E, nvec = (N + E - 1) / E;
  const int li = threadIdx.x % lanes, gi = threadIdx.x / lanes;
  const int gpc = kGroupThreads / lanes;
  const int64_t gstep = (int64_t)gridDim.x * gpc;
  const T* x = static_cast<const T*>(a.x);
  const T* dy = static_cast<const T*>(a.dy);
  T* dx = static_cast<T*>(a.dx);
  float wr[VPT][E], br[VPT][E], dwa[VPT][E], dba[VPT][E];
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int col = (li + j * lanes) * E + e;
      const bool in = col < N;
      wr[j][e] = in ? ld_param(static_cast<const T*>(a.w), col, 1.0f) : 0.0f;
      br[j][e] = in ? ld_param(static_cast<const T*>(a.b), col, 0.0f) : 0.0f;
      dwa[j][e] = 0.0f;
      dba[j][e] = 0.0f;
    }
  const float inv_n = 1.0f / (float)N;
  for (int64_t m0 = (int64_t)blockIdx.x * gpc; m0 < a.rows; m0 += gstep) {
    const int64_t m = m0 + gi;
    const bool live = m < a.rows;
    const int64_t mm = live ? m : 0;
    const float mu = live ? __ldg(a.mean + m) : 0.0f;
    const float rs = live ? __ldg(a.rstd + m) : 0.0f;
    const T* xrow = x + mm * a.ldx;
    const T* gyrow = dy + mm * a.lddy;
    float xv[VPT][E], gv[VPT][E];
    float s1 = 0.0f, s2 = 0.0f;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = li + j * lanes;
      if (live && v < nfull) {
        V::unpack(ld_stream(xrow + (size_t)v * E), xv[j]);
        V::unpack(ld_stream(gyrow + (size_t)v * E), gv[j]);
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int col = v * E + e;
          const bool in = live && v < nvec && col < N;
          xv[j][e] = in ? V::load1(xrow + col) : 0.0f;
          gv[j][e] = in ? V::load1(gyrow + col) : 0.0f;
        }
      }
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float xh = (xv[j][e] - mu) * rs;
        const float g = gv[j][e] * epi_grad<EPI, FAST>(fmaf(xh, wr[j][e], br[j][e]));
        const float gw = g * wr[j][e];
        gv[j][e] = g;
        s1 += gw;
        s2 = fmaf(gw, xh, s2);
        dwa[j][e] = fmaf(g, xh, dwa[j][e]);
        dba[j][e] += g;
      }
    }
    s1 = group_sum_rt(s1, lanes);
    s2 = group_sum_rt(s2, lanes);
    if (!live) continue;
    const float c1 = s1 * inv_n, c2 = s2 * inv_n;
    T* dxrow = dx + m * a.lddx;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = li + j * lanes;
      if (v < nvec) {
        float o[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const float xh = (xv[j][e] - mu) * rs;
          o[e] = rs * (fmaf(gv[j][e], wr[j][e], -c1) - xh * c2);
        }
        if (v < nfull) {
          st_stream(dxrow + (size_t)v * E, V::pack(o));
        } else {
#pragma unroll
          for (int e = 0; e < E; ++e)
            if (v * E + e < N) V::store1(dxrow + v * E + e, o[e]);
        }
      }
    }
  }
  if (!a.ws) return;
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int col = (li + j * lanes) * E + e;
      if (col < N) {
        gsm[gi * 2 * N + col] = dwa[j][e];
        gsm[gi * 2 * N + N + col] = dba[j][e];
      }
    }
  __syncthreads();
  float* part = a.ws + (int64_t)blockIdx.x * 2 * N;
  for (int col = threadIdx.x; col < 2 * N; col += kGroupThreads) {
    float t = 0.0f;
    for (int g = 0; g < gpc; ++g) t += gsm[g * 2 * N + col];
    part[col] = t;
  }
}

// ---------------------------------------------------------------- dispatch

template <typename T, int VPT, bool CTA, bool BWD>
void* pick_ln(int epi) {
#define GN_PICK(E_)                                                              \
  if constexpr (BWD) {                                                           \
    if constexpr (CTA) return (void*)ln_bwd_cta<T, VPT, E_>;                     \
    else return (void*)ln_bwd_grp<T, VPT, E_>;                                   \
  } else {                                                                       \
    if constexpr (CTA) return (void*)ln_fwd_cta<T, VPT, E_>;                     \
    else return (void*)ln_fwd_grp<T, VPT, E_>;                                   \
  }
  if (epi == EPI_GELU_TANH) { GN_PICK(EPI_GELU_TANH) }
  if (epi == EPI_SILU) { GN_PICK(EPI_SILU) }
  GN_PICK(EPI_NONE)
#undef GN_PICK
}

template <typename T, bool BWD>
void* pick_ln_t(int vpt, bool cta, int epi) {
  switch (vpt) {
    case 1: return cta ? pick_ln<T, 1, true, BWD>(epi) : pick_ln<T, 1, false, BWD>(epi);
    case 2: return cta ? pick_ln<T, 2, true, BWD>(epi) : pick_ln<T, 2, false, BWD>(epi);
    case 4: return cta ? pick_ln<T, 4, true, BWD>(epi) : pick_ln<T, 4, false, BWD>(epi);
    case 8:
      if constexpr (!BWD) return cta ? pick_ln<T, 8, true, false>(epi) : nullptr;
      return nullptr;
  }
  return nullptr;
}


gn_status ln_plan(int64_t rows, int64_t hidden, gn_dtype dt, bool bwd, int epi, NormPlan* p, void** kern,
                  int* grid) {
  // 4 vectors per thread in both directions (measured: the backward's per-row overhead
  // outweighs its extra registers)
  gn_status st = plan_norm(hidden, dt_size(dt), bwd ? 2 : 1, 2, bwd ? 4 : 8, 160, p, bwd ? 4 : 0);
  if (st != GN_OK) return st;
  if (dt == GN_BF16)
    *kern = bwd ? pick_ln_t<__nv_bfloat16, true>(p->vpt, p->cta, epi) : pick_ln_t<__nv_bfloat16, false>(p->vpt, p->cta, epi);
  else
    *kern = bwd ? pick_ln_t<float, true>(p->vpt, p->cta, epi) : pick_ln_t<float, false>(p->vpt, p->cta, epi);
  if (!*kern) return GN_ERR_UNSUPPORTED;
  const int cap = g_tune.ctas_per_sm ? g_tune.ctas_per_sm : 8;
  int g = persistent_grid(*kern, p->threads, p->smem, cap);
  if (g <= 0) return GN_ERR_CUDA;
  const int64_t units = p->cta ? rows : (rows + (kGroupThreads / p->lanes) - 1) / (kGroupThreads / p->lanes);
  if (units < g) g = (int)(units > 0 ? units : 1);
  *grid = g;
  return GN_OK;
}

}  // namespace
}  // namespace gn

using namespace gn;

extern "C" gn_status gn_layernorm_fwd(const void* x, const void* w, const void* b, void* y, float* mean,
                                      float* rstd, int64_t rows, int64_t hidden, int64_t ld_x, int64_t ld_y,
                                      float eps, gn_epilogue epi, gn_dtype dt, void* stream) {
  if (!dt_ok(dt) || !epi_ok(epi)) return GN_ERR_DTYPE;
  if (rows < 0 || hidden <= 0 || ld_x < hidden || ld_y < hidden || hidden > (1 << 20)) return GN_ERR_SHAPE;
  if (rows == 0) return GN_OK;
  if (!x || !y) return GN_ERR_NULL;
  const size_t es = dt_size(dt);
  if (!aligned16(x) || !aligned16(y) || (ld_x * es) % 16 || (ld_y * es) % 16) return GN_ERR_ALIGN;
  gn_status st;
  if ((hidden * (int64_t)es + 15) / 16 > kGroupMaxVec && g_tune.fwd_path != 1) {
    // long rows: one warp per row unless the row does not fit
    st = launch_norm_fwd_warp(true, x, w, b, y, mean, rstd, rows, hidden, ld_x, ld_y, eps, false, epi, dt,
                              (cudaStream_t)stream);
    if (st != GN_ERR_UNSUPPORTED) return st;
  }
  NormPlan p;
  void* kern = nullptr;
  int grid = 0;
  st = ln_plan(rows, hidden, dt, false, epi, &p, &kern, &grid);
  if (st != GN_OK) return st;
  unsigned* err = device_err_word();
  if (!err) return GN_ERR_CUDA;
  LnFwdArgs a{x, w, b, y, mean, rstd, rows, ld_x, ld_y, (int)hidden, eps, p.stages, err};
  int lanes = p.lanes;
  void* args_cta[] = {&a};
  void* args_grp[] = {&a, &lanes};
  if (cudaLaunchKernel(kern, dim3(grid), dim3(p.threads), p.cta ? args_cta : args_grp, p.smem,
                       (cudaStream_t)stream) != cudaSuccess)
    return GN_ERR_CUDA;
  count_launches(1);
  return launch_status();
}

extern "C" size_t gn_layernorm_bwd_workspace(int64_t rows, int64_t hidden, gn_dtype dt) {
  if (rows <= 0 || hidden <= 0 || !dt_ok(dt)) return 0;
  // the epilogue variants may differ in occupancy, hence in persistent grid size: size for
  // the largest
  int grid = 0;
  for (int epi = GN_EPI_NONE; epi <= GN_EPI_SILU; ++epi) {
    NormPlan p;
    void* kern = nullptr;
    int g = 0;
    if (ln_plan(rows, hidden, dt, true, epi, &p, &kern, &g) != GN_OK) return 0;
    if (g > grid) grid = g;
  }
  return (size_t)grid * 2 * (size_t)hidden * sizeof(float);
}

extern "C" gn_status gn_layernorm_bwd(const void* x, const void* w, const void* b, const float* mean,
                                      const float* rstd, const void* dy, void* dx, float* dw, float* db,
                                      void* ws, size_t ws_bytes, int64_t rows, int64_t hidden, int64_t ld_x,
                                      int64_t ld_dy, int64_t ld_dx, gn_epilogue epi, gn_dtype dt,
                                      void* stream) {
  if (!dt_ok(dt) || !epi_ok(epi)) return GN_ERR_DTYPE;
  if (rows < 0 || hidden <= 0 || ld_x < hidden || ld_dy < hidden || ld_dx < hidden || hidden > (1 << 20))
    return GN_ERR_SHAPE;
  cudaStream_t s = (cudaStream_t)stream;
  if (rows == 0) {
    if (dw && cudaMemsetAsync(dw, 0, (size_t)hidden * sizeof(float), s) != cudaSuccess) return GN_ERR_CUDA;
    if (db && cudaMemsetAsync(db, 0, (size_t)hidden * sizeof(float), s) != cudaSuccess) return GN_ERR_CUDA;
    return GN_OK;
  }
  if (!x || !mean || !rstd || !dy || !dx) return GN_ERR_NULL;
  const size_t es = dt_size(dt);
  if (!aligned16(x) || !aligned16(dy) || !aligned16(dx) || (ld_x * es) % 16 || (ld_dy * es) % 16 ||
      (ld_dx * es) % 16)
    return GN_ERR_ALIGN;
  NormPlan p;
  void* kern = nullptr;
  int grid = 0;
  gn_status st = ln_plan(rows, hidden, dt, true, epi, &p, &kern, &grid);
  if (st != GN_OK) return st;
  const bool wgrad = dw || db;
  if (wgrad) {
    if (!ws) return GN_ERR_WORKSPACE;
    if (!aligned16(ws)) return GN_ERR_ALIGN;
    if (ws_bytes < (size_t)grid * 2 * (size_t)hidden * sizeof(float)) return GN_ERR_WORKSPACE;
  }
  unsigned* err = device_err_word();
  if (!err) return GN_ERR_CUDA;
  LnBwdArgs a{x, w, b, mean, rstd, dy, dx, wgrad ? static_cast<float*>(ws) : nullptr, rows, ld_x, ld_dy, ld_dx,
              (int)hidden, p.stages, err};
  int lanes = p.lanes;
  void* args_cta[] = {&a};
  void* args_grp[] = {&a, &lanes};
  if (cudaLaunchKernel(kern, dim3(grid), dim3(p.threads), p.cta ? args_cta : args_grp, p.smem, s) != cudaSuccess)
    return GN_ERR_CUDA;
  count_launches(1);
  if ((st = launch_status()) != GN_OK) return st;
  if (wgrad) return launch_colsum(static_cast<const float*>(ws), grid, 2 * hidden, hidden, dw, db, s);
  return GN_OK;
}
