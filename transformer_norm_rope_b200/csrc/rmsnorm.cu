// rmsnorm.cu - RMSNorm forward and backward (Helios kernels article, section
// "内核一 FlashNorm": one pass over each row, sum of squares and its inverse root, times the
// weight; Gemma +1 offset as a compile-time branch; the forward saves the per-row inverse
// RMS and the backward reuses it).
//
//   forward : r = rsqrt(mean(x^2) + eps), y = epi(x r w'), inv_rms = r
//   backward: g = dy epi'(x r w'), dx = r (g w' - x r mean(g w' x r)), dw = sum_rows g x r
//
// Both directions read each input byte from HBM once and write each output byte once. The
// weight gradient is accumulated per thread in fp32 registers over the rows a CTA owns,
// written as one partial row per CTA, and summed in a fixed order by launch_colsum.
#include "norm_plan.h"
#include "norm_rows.cuh"

namespace gn {
namespace {

struct RmsFwdArgs {
  const void* x;
  const void* w;
  void* y;
  float* inv_rms;
  int64_t rows;
  int64_t ldx, ldy;
  int N;
  float eps;
  int stages;
  unsigned* err;
};

struct RmsBwdArgs {
  const void* x;
  const void* w;
  const float* inv_rms;
  const void* dy;
  void* dx;
  float* ws;  // [gridDim.x, N] partial dw, or null
  int64_t rows;
  int64_t ldx, lddy, lddx;
  int N;
  int stages;
  unsigned* err;
};

// ---------------------------------------------------------------- CTA path (long rows)
// Warp 0 produces (row_pipe.cuh); warps 1.. consume. Consumer thread ct owns the vectors
// v = ct + j * nct (j < VPT) of every row, so its columns - and its share of the weight
// gradient - never change. The weight lives in shared memory (one copy per CTA). The
// arithmetic runs on element pairs with packed fp32x2 instructions.


template <typename T, int VPT, int EPI, bool GEMMA>
__global__ void __launch_bounds__(kNormCtaThreads, norm_min_blocks(VPT)) rms_fwd_cta(const RmsFwdArgs a) {
  constexpr int H = Vec<T>::N / 2;
  constexpr bool FAST = fast_math_for<T>();
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int N = a.N, nfull = N / Vec<T>::N, nvec = (N + Vec<T>::N - 1) / Vec<T>::N;
  const RowPipe pipe(smem, a.stages, 1, 1, N, sizeof(T), sizeof(T));
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
  stage_param<T, VPT>(pipe.param(0), static_cast<const T*>(a.w), N, nvec, 0.0f, ct, nct);
  pipe.red_zero(ct, nct);
  consumers_sync(nct);
  const float inv_n = 1.0f / (float)N;
  const int64_t step = gridDim.x;
  int s = 0;
  uint32_t ph = 0, rb = 0;
  for (int64_t m = blockIdx.x; m < a.rows; m += step) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&pipe.full[s], ph, a.err));
    float2 xv[VPT][H];
    float2 ss2 = dup2(0.0f);
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      load_pairs<T>(pipe.at(s, 0), x + m * a.ldx, ct + j * nct, nfull, N, ok, xv[j]);
#pragma unroll
      for (int h = 0; h < H; ++h) ss2 = fma2(xv[j][h], xv[j][h], ss2);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&pipe.empty[s]);
    const float ss = group_sum<32>(ss2.x + ss2.y);
    if (lane == 0) pipe.red_at(rb, 0)[cw] = ss;
    if (consumers_sync_or(nct, !ok)) return;
    const float tot = pipe.red_sum(rb, 0, ncw);
    rb ^= 1u;
    if (++s == a.stages) s = 0, ph ^= 1u;
    const float r = rsqrtf(fmaf(tot, inv_n, a.eps));
    const float2 r2 = dup2(r);
    T* yrow = y + m * a.ldy;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = ct + j * nct;
      if (v < nvec) {
        float2 wv[H], o[H];
        param_pairs<T>(pipe.param(0), v, wv);
#pragma unroll
        for (int h = 0; h < H; ++h) {
          const float2 wp = GEMMA ? add2(wv[h], dup2(1.0f)) : wv[h];
          o[h] = epi_fwd2<EPI, FAST>(mul2(mul2(xv[j][h], r2), wp));
        }
        store_pairs<T>(yrow, v, nfull, N, o);
      }
    }
    if (ct == 0 && a.inv_rms) a.inv_rms[m] = r;
  }
}

template <typename T, int VPT, int EPI, bool GEMMA>
__global__ void __launch_bounds__(kNormCtaThreads, norm_min_blocks(VPT, true)) rms_bwd_cta(const RmsBwdArgs a) {
  pdl_launch_dependents();  // the column reduction that follows may launch early
  constexpr int E = Vec<T>::N, H = E / 2;
  constexpr bool FAST = fast_math_for<T>();
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int N = a.N, nfull = N / E, nvec = (N + E - 1) / E;
  const RowPipe pipe(smem, a.stages, 2, 1, N, sizeof(T), 4);
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
  // w' = w (+1 Gemma) as fp32: the per-row passes read it with no conversion
  stage_param_f32<T, VPT>(reinterpret_cast<float*>(pipe.param(0)), static_cast<const T*>(a.w), N, nvec,
                          GEMMA ? 1.0f : 0.0f, 1.0f, 0.0f, ct, nct);
  pipe.red_zero(ct, nct);
  consumers_sync(nct);
  float2 dwa[VPT][H];
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int h = 0; h < H; ++h) dwa[j][h] = dup2(0.0f);
  const float inv_n = 1.0f / (float)N;
  const int64_t step = gridDim.x;
  int s = 0;
  uint32_t ph = 0, rb = 0;
  bool failed = false;
  // the statistic of the next row is loaded one row ahead: its global-memory latency then
  // overlaps the current row instead of stalling the start of the next
  float r_n = blockIdx.x < a.rows ? __ldg(a.inv_rms + blockIdx.x) : 0.0f;
  for (int64_t m = blockIdx.x; m < a.rows; m += step) {
    const float r = r_n;
    if (m + step < a.rows) r_n = __ldg(a.inv_rms + m + step);
    const float2 r2 = dup2(r);
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
    float2 c2 = dup2(0.0f);
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = ct + j * nct;
      float2 wv[H], xv[H];
      prm_pairs<H>(reinterpret_cast<const float*>(pipe.param(0)), v < nvec ? v : 0, nvec, wv);
      unpack2<T>(xr[j], xv);
#pragma unroll
      for (int h = 0; h < H; ++h) {
        const float2 wp = wv[h];
        const float2 xh = mul2(xv[h], r2);
        const float2 g = EPI == EPI_NONE ? gv[j][h] : mul2(gv[j][h], epi_grad2<EPI, FAST>(mul2(xh, wp)));
        const float2 gw = mul2(g, wp);
        gv[j][h] = gw;  // phase 2 needs only g w'
        c2 = fma2(gw, xh, c2);
        dwa[j][h] = fma2(g, xh, dwa[j][h]);
      }
    }
    const float c = group_sum<32>(c2.x + c2.y);
    if (lane == 0) pipe.red_at(rb, 0)[cw] = c;
    if (consumers_sync_or(nct, !ok)) {
      failed = true;
      break;
    }
    const float tot = pipe.red_sum(rb, 0, ncw);
    rb ^= 1u;
    if (++s == a.stages) s = 0, ph ^= 1u;
    const float2 ncm = dup2(-tot * inv_n);
    T* dxrow = dx + m * a.lddx;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = ct + j * nct;
      if (v < nvec) {
        float2 xv[H], o[H];
        unpack2<T>(xr[j], xv);
#pragma unroll
        for (int h = 0; h < H; ++h) o[h] = mul2(r2, fma2(mul2(xv[h], r2), ncm, gv[j][h]));
        store_pairs<T>(dxrow, v, nfull, N, o);
      }
    }
  }
  if (a.ws && !failed) {
    float* part = a.ws + (int64_t)blockIdx.x * N;
#pragma unroll
    for (int j = 0; j < VPT; ++j)
#pragma unroll
      for (int h = 0; h < H; ++h) {
        const int col = (ct + j * nct) * E + 2 * h;
        if (col < N) part[col] = dwa[j][h].x;
        if (col + 1 < N) part[col + 1] = dwa[j][h].y;
      }
  }
}

// ---------------------------------------------------------------- group path (short rows)
// `lanes` consecutive threads own one row; rows are walked grid-stride by lane groups.

template <typename T, int VPT, int EPI, bool GEMMA>
__global__ void __launch_bounds__(kGroupThreads) rms_fwd_grp(const RmsFwdArgs a, int lanes) {
  using V = Vec<T>;
  constexpr int E = V::N;
  constexpr bool FAST = fast_math_for<T>();
  const int N = a.N, nfull = N / E, nvec = (N + E - 1) / E;
  const int li = threadIdx.x % lanes;
  const int64_t gpc = kGroupThreads / lanes;
  const int gi = threadIdx.x / lanes;
  const int64_t gstep = (int64_t)gridDim.x * gpc;
  const T* x = static_cast<const T*>(a.x);
  T* y = static_cast<T*>(a.y);
  float wr[VPT][E];
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int col = (li + j * lanes) * E + e;
      wr[j][e] = col < N ? (GEMMA ? 1.0f : 0.0f) + ld_param(static_cast<const T*>(a.w), col, 0.0f) : 0.0f;
    }
  const float inv_n = 1.0f / (float)N;
  // the loop bound is the CTA's first row (uniform over the CTA), so every lane runs the
  // same iterations and the shuffles below always see the full warp
  for (int64_t m0 = (int64_t)blockIdx.x * gpc; m0 < a.rows; m0 += gstep) {
    const int64_t m = m0 + gi;
    const bool live = m < a.rows;
    const T* xrow = x + (live ? m : 0) * a.ldx;
    float xv[VPT][E];
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = li + j * lanes;
      if (live && v < nfull) {
        V::unpack(ld_stream(xrow + (size_t)v * E), xv[j]);
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int col = v * E + e;
          xv[j][e] = (live && v < nvec && col < N) ? V::load1(xrow + col) : 0.0f;
        }
      }
#pragma unroll
      for (int e = 0; e < E; ++e) ss = fmaf(xv[j][e], xv[j][e], ss);
    }
    ss = group_sum_rt(ss, lanes);
    if (!live) continue;
    const float r = rsqrtf(fmaf(ss, inv_n, a.eps));
    T* yrow = y + m * a.ldy;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = li + j * lanes;
      if (v < nvec) {
        float o[E];
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = epi_fwd<EPI, FAST>(xv[j][e] * r * wr[j][e]);
        if (v < nfull) {
          st_stream(yrow + (size_t)v * E, V::pack(o));
        } else {
#pragma unroll
          for (int e = 0; e < E; ++e)
            if (v * E + e < N) V::store1(yrow + v * E + e, o[e]);
        }
      }
    }
    if (li == 0 && a.inv_rms) a.inv_rms[m] = r;
  }
}

template <typename T, int VPT, int EPI, bool GEMMA>
__global__ void __launch_bounds__(kGroupThreads) rms_bwd_grp(const RmsBwdArgs a, int lanes) {
  pdl_launch_dependents();  // the column reduction that follows may launch early
  using V = Vec<T>;
  constexpr int E = V::N;
  constexpr bool FAST = fast_math_for<T>();
  extern __shared__ __align__(16) float gsm[];  // [groups per CTA][N] dw partials
  const int N = a.N, nfull = N / E, nvec = (N + E - 1) / E;
  const int li = threadIdx.x % lanes;
  const int gi = threadIdx.x / lanes;
  const int gpc = kGroupThreads / lanes;
  const int64_t gstep = (int64_t)gridDim.x * gpc;
  const T* x = static_cast<const T*>(a.x);
  const T* dy = static_cast<const T*>(a.dy);
  T* dx = static_cast<T*>(a.dx);
  float wr[VPT][E], dwa[VPT][E];
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int col = (li + j * lanes) * E + e;
      wr[j][e] = col < N ? (GEMMA ? 1.0f : 0.0f) + ld_param(static_cast<const T*>(a.w), col, 0.0f) : 0.0f;
      dwa[j][e] = 0.0f;
    }
  const float inv_n = 1.0f / (float)N;
  for (int64_t m0 = (int64_t)blockIdx.x * gpc; m0 < a.rows; m0 += gstep) {
    const int64_t m = m0 + gi;
    const bool live = m < a.rows;
    const int64_t mm = live ? m : 0;
    const float r = live ? __ldg(a.inv_rms + m) : 0.0f;
    const T* xrow = x + mm * a.ldx;
    const T* gyrow = dy + mm * a.lddy;
    float xv[VPT][E], gv[VPT][E];
    float c = 0.0f;
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
        const float xh = xv[j][e] * r;
        const float g = gv[j][e] * epi_grad<EPI, FAST>(xh * wr[j][e]);
        gv[j][e] = g;
        c = fmaf(g * wr[j][e], xh, c);
        dwa[j][e] = fmaf(g, xh, dwa[j][e]);
      }
    }
    c = group_sum_rt(c, lanes);
    if (!live) continue;
    const float cm = c * inv_n;
    T* dxrow = dx + m * a.lddx;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int v = li + j * lanes;
      if (v < nvec) {
        float o[E];
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = r * fmaf(gv[j][e], wr[j][e], -(xv[j][e] * r) * cm);
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
  // combine the groups of this CTA in group order, then write one partial row
#pragma unroll
  for (int j = 0; j < VPT; ++j)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int col = (li + j * lanes) * E + e;
      if (col < N) gsm[gi * N + col] = dwa[j][e];
    }
  __syncthreads();
  float* part = a.ws + (int64_t)blockIdx.x * N;
  for (int col = threadIdx.x; col < N; col += kGroupThreads) {
    float t = 0.0f;
    for (int g = 0; g < gpc; ++g) t += gsm[g * N + col];
    part[col] = t;
  }
}

// ---------------------------------------------------------------- dispatch

template <typename T, int VPT, bool CTA>
void* pick_fwd(int epi, bool gemma) {
#define GN_PICK(E_, G_) \
  if constexpr (CTA) return (void*)rms_fwd_cta<T, VPT, E_, G_>; \
  else return (void*)rms_fwd_grp<T, VPT, E_, G_>
  if (epi == EPI_GELU_TANH) { if (gemma) GN_PICK(EPI_GELU_TANH, true); else GN_PICK(EPI_GELU_TANH, false); }
  if (epi == EPI_SILU) { if (gemma) GN_PICK(EPI_SILU, true); else GN_PICK(EPI_SILU, false); }
  if (gemma) GN_PICK(EPI_NONE, true);
  GN_PICK(EPI_NONE, false);
#undef GN_PICK
}

template <typename T, int VPT, bool CTA>
void* pick_bwd(int epi, bool gemma) {
#define GN_PICK(E_, G_) \
  if constexpr (CTA) return (void*)rms_bwd_cta<T, VPT, E_, G_>; \
  else return (void*)rms_bwd_grp<T, VPT, E_, G_>
  if (epi == EPI_GELU_TANH) { if (gemma) GN_PICK(EPI_GELU_TANH, true); else GN_PICK(EPI_GELU_TANH, false); }
  if (epi == EPI_SILU) { if (gemma) GN_PICK(EPI_SILU, true); else GN_PICK(EPI_SILU, false); }
  if (gemma) GN_PICK(EPI_NONE, true);
  GN_PICK(EPI_NONE, false);
#undef GN_PICK
}

template <typename T>
void* pick_fwd_t(int vpt, bool cta, int epi, bool gemma) {
  switch (vpt) {
    case 1: return cta ? pick_fwd<T, 1, true>(epi, gemma) : pick_fwd<T, 1, false>(epi, gemma);
    case 2: return cta ? pick_fwd<T, 2, true>(epi, gemma) : pick_fwd<T, 2, false>(epi, gemma);
    case 4: return cta ? pick_fwd<T, 4, true>(epi, gemma) : pick_fwd<T, 4, false>(epi, gemma);
    case 8: return cta ? pick_fwd<T, 8, true>(epi, gemma) : nullptr;
  }
  return nullptr;
}

template <typename T>
void* pick_bwd_t(int vpt, bool cta, int epi, bool gemma) {
  switch (vpt) {
    case 1: return cta ? pick_bwd<T, 1, true>(epi, gemma) : pick_bwd<T, 1, false>(epi, gemma);
    case 2: return cta ? pick_bwd<T, 2, true>(epi, gemma) : pick_bwd<T, 2, false>(epi, gemma);
    case 4: return cta ? pick_bwd<T, 4, true>(epi, gemma) : pick_bwd<T, 4, false>(epi, gemma);
  }
  return nullptr;
}


gn_status rms_bwd_plan(int64_t rows, int64_t hidden, gn_dtype dt, NormPlan* p, void** kern, int epi,
                       bool gemma, int* grid) {
  gn_status st = plan_norm(hidden, dt_size(dt), 2, 1, 4, 320, p, 4);
  if (st != GN_OK) return st;
  *kern = dt == GN_BF16 ? pick_bwd_t<__nv_bfloat16>(p->vpt, p->cta, epi, gemma)
                        : pick_bwd_t<float>(p->vpt, p->cta, epi, gemma);
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

extern "C" gn_status gn_rmsnorm_fwd(const void* x, const void* w, void* y, float* inv_rms,
                                    int64_t rows, int64_t hidden, int64_t ld_x, int64_t ld_y,
                                    float eps, int gemma, gn_epilogue epi, gn_dtype dt,
                                    void* stream) {
  if (!dt_ok(dt) || !epi_ok(epi)) return GN_ERR_DTYPE;
  if (rows < 0 || hidden <= 0 || ld_x < hidden || ld_y < hidden || hidden > (1 << 20)) return GN_ERR_SHAPE;
  if (rows == 0) return GN_OK;
  if (!x || !w || !y) return GN_ERR_NULL;
  const size_t es = dt_size(dt);
  if (!aligned16(x) || !aligned16(y) || (ld_x * es) % 16 || (ld_y * es) % 16) return GN_ERR_ALIGN;
  NormPlan p;
  gn_status st = plan_norm(hidden, es, 1, 1, 8, 320, &p);
  if (st != GN_OK) return st;
  if (p.cta && (g_tune.fwd_path == 2 || g_tune.fwd_path == 3)) {  // long rows, one warp per row on request
    st = launch_norm_fwd_warp(false, x, w, nullptr, y, inv_rms, nullptr, rows, hidden, ld_x, ld_y, eps, gemma != 0,
                              epi, dt, (cudaStream_t)stream);
    if (st != GN_ERR_UNSUPPORTED) return st;
  }
  void* kern = dt == GN_BF16 ? pick_fwd_t<__nv_bfloat16>(p.vpt, p.cta, epi, gemma != 0)
                             : pick_fwd_t<float>(p.vpt, p.cta, epi, gemma != 0);
  if (!kern) return GN_ERR_UNSUPPORTED;
  const int cap = g_tune.ctas_per_sm ? g_tune.ctas_per_sm : 8;
  int grid = persistent_grid(kern, p.threads, p.smem, cap);
  if (grid <= 0) return GN_ERR_CUDA;
  const int64_t units = p.cta ? rows : (rows + (kGroupThreads / p.lanes) - 1) / (kGroupThreads / p.lanes);
  if (units < grid) grid = (int)units;
  unsigned* err = device_err_word();
  if (!err) return GN_ERR_CUDA;
  RmsFwdArgs a{x, w, y, inv_rms, rows, ld_x, ld_y, (int)hidden, eps, p.stages, err};
  int lanes = p.lanes;
  void* args_cta[] = {&a};
  void* args_grp[] = {&a, &lanes};
  if (cudaLaunchKernel(kern, dim3(grid), dim3(p.threads), p.cta ? args_cta : args_grp, p.smem,
                       (cudaStream_t)stream) != cudaSuccess)
    return GN_ERR_CUDA;
  count_launches(1);
  return launch_status();
}

extern "C" size_t gn_rmsnorm_bwd_workspace(int64_t rows, int64_t hidden, gn_dtype dt) {
  if (rows <= 0 || hidden <= 0 || !dt_ok(dt)) return 0;
  // the epilogue and Gemma variants may differ in occupancy, hence in persistent grid size:
  // size for the largest
  int grid = 0;
  for (int epi = GN_EPI_NONE; epi <= GN_EPI_SILU; ++epi)
    for (int gemma = 0; gemma < 2; ++gemma) {
      NormPlan p;
      void* kern = nullptr;
      int g = 0;
      if (rms_bwd_plan(rows, hidden, dt, &p, &kern, epi, gemma != 0, &g) != GN_OK) return 0;
      if (g > grid) grid = g;
    }
  return (size_t)grid * (size_t)hidden * sizeof(float);
}

extern "C" gn_status gn_rmsnorm_bwd(const void* x, const void* w, const float* inv_rms,
                                    const void* dy, void* dx, float* dw, void* ws, size_t ws_bytes,
                                    int64_t rows, int64_t hidden, int64_t ld_x, int64_t ld_dy,
                                    int64_t ld_dx, int gemma, gn_epilogue epi, gn_dtype dt,
                                    void* stream) {
  if (!dt_ok(dt) || !epi_ok(epi)) return GN_ERR_DTYPE;
  if (rows < 0 || hidden <= 0 || ld_x < hidden || ld_dy < hidden || ld_dx < hidden || hidden > (1 << 20))
    return GN_ERR_SHAPE;
  cudaStream_t s = (cudaStream_t)stream;
  if (rows == 0) {
    if (dw && cudaMemsetAsync(dw, 0, (size_t)hidden * sizeof(float), s) != cudaSuccess) return GN_ERR_CUDA;
    return GN_OK;
  }
  if (!x || !w || !inv_rms || !dy || !dx) return GN_ERR_NULL;
  const size_t es = dt_size(dt);
  if (!aligned16(x) || !aligned16(dy) || !aligned16(dx) || (ld_x * es) % 16 || (ld_dy * es) % 16 ||
      (ld_dx * es) % 16)
    return GN_ERR_ALIGN;
  NormPlan p;
  void* kern = nullptr;
  int grid = 0;
  gn_status st = rms_bwd_plan(rows, hidden, dt, &p, &kern, epi, gemma != 0, &grid);
  if (st != GN_OK) return st;
  if (dw) {
    if (!ws || !aligned16(ws)) return ws ? GN_ERR_ALIGN : GN_ERR_WORKSPACE;
    if (ws_bytes < (size_t)grid * (size_t)hidden * sizeof(float)) return GN_ERR_WORKSPACE;
  }
  unsigned* err = device_err_word();
  if (!err) return GN_ERR_CUDA;
  RmsBwdArgs a{x, w, inv_rms, dy, dx, dw ? static_cast<float*>(ws) : nullptr, rows, ld_x, ld_dy, ld_dx,
               (int)hidden, p.stages, err};
  int lanes = p.lanes;
  void* args_cta[] = {&a};
  void* args_grp[] = {&a, &lanes};
  if (cudaLaunchKernel(kern, dim3(grid), dim3(p.threads), p.cta ? args_cta : args_grp, p.smem, s) !=
      cudaSuccess)
    return GN_ERR_CUDA;
  count_launches(1);
  if ((st = launch_status()) != GN_OK) return st;
  if (dw) return launch_colsum(static_cast<const float*>(ws), grid, hidden, hidden, dw, nullptr, s);
  return GN_OK;
}
