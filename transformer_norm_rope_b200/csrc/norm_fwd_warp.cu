// norm_fwd_warp.cu - RMSNorm and LayerNorm forward with one warp per row (Helios kernels
// article, section "内核一 FlashNorm": each row read from HBM once, its statistic reduced and
// inverted on chip, the scaled row written once, the per-row inverse statistic saved;
// "LLM层的优化算子", section "编写定制融合算子": LayerNorm centres, takes the biased variance,
// divides by sqrt(var + eps), applies weight and bias and the tanh-GeLU in the same pass).
//
//   RMSNorm  : r = rsqrt(mean(x^2) + eps),            y = epi(x r w'),            inv_rms = r
//   LayerNorm: mu = mean(x), s = rsqrt(mean((x-mu)^2) + eps), y = epi((x-mu) s w + b), mean, rstd
//
// Layout of the work: a CTA of W warps per SM; warp g of the grid owns rows g, g + G, g + 2G, ...
// (G = all warps of the grid). Each warp is its own producer: one lane moves the warp's next rows
// into the warp's private shared-memory stages with 1-D TMA bulk copies (one mbarrier per stage),
// S - 1 rows ahead of the row being computed (by default S = 1: the warp loads its row, then
// computes it, while the SM's other warps load and compute theirs). A stage is refilled only
// after the warp itself has finished the row it held, so no consumer-release barrier exists, and
// no barrier spans more than one warp: the row statistics are reduced with xor shuffles inside
// the warp. The warp reads its row from shared memory once per pass (two passes: the statistics,
// then the output; the exact two-pass LayerNorm variant takes the mean and the centred sum of
// squares in separate passes, three in all), so the row stays in HBM order one 16-byte vector
// per lane and nothing of it needs to live in registers.
//
// The parameters (weight, bias) are staged once per CTA in shared memory, before the tanh-GeLU
// with the factor 1/2 folded in (exact): widened to fp32 with the Gemma +1 offset folded in for
// RMSNorm and fp32 rows (the per-row passes then read them with no conversion), kept in bf16 for
// LayerNorm on bf16 rows (half the space, so that more warps fit).
#include "gn_host.h"
#include "norm_plan.h"
#include "norm_rows.cuh"

namespace gn {
namespace {

constexpr int kWarpFwdMaxWarps = 20;
constexpr int kWarpFwdMaxStages = 4;
constexpr uint32_t kWarpFwdHeader = kWarpFwdMaxWarps * kWarpFwdMaxStages * 8;  // mbarriers

struct WarpFwdArgs {
  const void* x;
  const void* w;
  const void* b;  // LayerNorm bias (null = 0)
  void* y;
  float* stat0;   // RMSNorm: inv_rms; LayerNorm: mean (null = not saved)
  float* stat1;   // LayerNorm: rstd
  int64_t rows;
  int64_t ldx, ldy;
  int N;
  int stages;
  uint32_t slot;    // bytes per stage (one row of whole 16-byte vectors, rounded to 128)
  uint32_t pbytes;  // bytes per staged parameter vector
  float eps;
  unsigned* err;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// MODE: 0 RMSNorm; 1 LayerNorm, statistics in two passes (mean, then centred squares); 2 LayerNorm,
// statistics in one pass around a shift K (the mean of each lane's first vector over the warp):
// mean = K + S1 / N, var = S2 / N - (S1 / N)^2 with S1 = sum (x - K), S2 = sum (x - K)^2; |mean - K|
// is of the order of the row's deviation over sqrt(256), so the subtraction loses nothing measurable
template <typename T, int MODE, int EPI, bool GEMMA>
__global__ void __launch_bounds__(kWarpFwdMaxWarps * 32, 1) norm_fwd_warp(const WarpFwdArgs a) {
  constexpr bool LN = MODE != 0;
  using V = Vec<T>;
  constexpr int E = V::N, H = E / 2;
  constexpr bool FAST = fast_math_for<T>();
  constexpr bool HALF = LN && EPI == EPI_GELU_TANH;  // parameters staged halved for gelu_of_half2
  // LayerNorm on bf16 rows keeps its weight and bias in bf16 (unpacked on use): half the shared
  // memory of fp32 copies, so that 20 warps fit at hidden 5120 instead of 16
  constexpr bool P16 = LN && sizeof(T) == 2;
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (int)(blockDim.x >> 5);
  const int S = a.stages;
  const int N = a.N, nfull = N / E, nvec = (N + E - 1) / E;
  const uint32_t bulk = (uint32_t)nfull * 16u;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem) + wid * kWarpFwdMaxStages;
  float* pw = reinterpret_cast<float*>(smem + kWarpFwdHeader);
  float* pb = reinterpret_cast<float*>(smem + kWarpFwdHeader + a.pbytes);
  uint8_t* stg = smem + kWarpFwdHeader + (LN ? 2u : 1u) * a.pbytes + (size_t)wid * S * a.slot;
  const T* x = static_cast<const T*>(a.x);
  T* y = static_cast<T*>(a.y);
  const int64_t gstep = (int64_t)gridDim.x * nw;
  const int64_t m0 = (int64_t)blockIdx.x * nw + wid;

  // this warp's barriers and first rows, issued before the parameters are staged so that the
  // copies' latency overlaps the staging
  uint32_t pend = 0;  // stages holding a copy not yet consumed (bit s), their phases in pph
  uint32_t pph = 0;
  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
    mbar_fence_init();
    for (int k = 0; k < S - 1; ++k) {
      const int64_t m = m0 + (int64_t)k * gstep;
      if (m < a.rows) {
        mbar_expect_tx(&full[k], bulk);
        bulk_g2s(stg + (size_t)k * a.slot, x + m * a.ldx, bulk, &full[k]);
        pend |= 1u << k;
      }
    }
  }
  // the parameters, zero past N: fp32 (Gemma offset folded in) or, for P16, the row type
  if constexpr (P16) {
    stage_rowtype<T>(reinterpret_cast<uint8_t*>(pw), static_cast<const T*>(a.w), N, nvec, HALF ? 0.5f : 1.0f, 1.0f);
    stage_rowtype<T>(reinterpret_cast<uint8_t*>(pb), static_cast<const T*>(a.b), N, nvec, HALF ? 0.5f : 1.0f, 0.0f);
  } else {
    stage_fp32<T>(pw, static_cast<const T*>(a.w), N, nvec, GEMMA ? 1.0f : 0.0f, HALF ? 0.5f : 1.0f, 1.0f);
    if constexpr (LN) stage_fp32<T>(pb, static_cast<const T*>(a.b), N, nvec, 0.0f, HALF ? 0.5f : 1.0f, 0.0f);
  }
  __syncthreads();

  const float inv_n = 1.0f / (float)N;
  const int tv = nfull;  // index of the ragged tail vector (if N % E != 0), owned by lane tv & 31
  const int tcnt = N - nfull * E;
  int s = 0;
  uint32_t ph = 0;
  bool failed = false;
  for (int64_t m = m0; m < a.rows; m += gstep) {
    // refill: the row S - 1 ahead goes into the stage this warp finished last; every lane's reads
    // of that stage returned their values before the __syncwarp that closed the previous row
    if (lane == 0) {
      const int64_t mn = m + (int64_t)(S - 1) * gstep;
      if (mn < a.rows) {
        int sn = s + S - 1;
        if (sn >= S) sn -= S;
        const uint32_t phn = sn >= s ? ph : ph ^ 1u;
        mbar_expect_tx(&full[sn], bulk);
        bulk_g2s(stg + (size_t)sn * a.slot, x + mn * a.ldx, bulk, &full[sn]);
        pend |= 1u << sn;
        pph = (pph & ~(1u << sn)) | (phn << sn);
      }
    }
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, a.err))) {
      failed = true;
      break;
    }
    if (lane == 0) pend &= ~(1u << s);
    const uint8_t* st = stg + (size_t)s * a.slot;
    const T* xrow = x + m * a.ldx;
    // the ragged tail vector, widened from global memory (zero past N)
    float2 tail[H];
#pragma unroll
    for (int h = 0; h < H; ++h) tail[h] = dup2(0.0f);
    if (tcnt && lane == (tv & 31)) {
#pragma unroll
      for (int h = 0; h < H; ++h) {
        tail[h].x = 2 * h < tcnt ? V::load1(xrow + tv * E + 2 * h) : 0.0f;
        tail[h].y = 2 * h + 1 < tcnt ? V::load1(xrow + tv * E + 2 * h + 1) : 0.0f;
      }
    }
    float stat_a;  // RMSNorm: r; LayerNorm: rstd
    float mu = 0.0f;
    if constexpr (!LN) {
      float2 acc[H];
#pragma unroll
      for (int h = 0; h < H; ++h) acc[h] = dup2(0.0f);
#pragma unroll 4
      for (int v = lane; v < nfull; v += 32) {
        float2 f[H];
        unpack2<T>(*reinterpret_cast<const uint4*>(st + (size_t)v * 16), f);
#pragma unroll
        for (int h = 0; h < H; ++h) acc[h] = fma2(f[h], f[h], acc[h]);
      }
      if (tcnt && lane == (tv & 31))
#pragma unroll
        for (int h = 0; h < H; ++h) acc[h] = fma2(tail[h], tail[h], acc[h]);
      float2 t = acc[0];
#pragma unroll
      for (int h = 1; h < H; ++h) t = add2(t, acc[h]);
      const float ss = warp_sum(t.x + t.y);
      stat_a = rsqrtf(fmaf(ss, inv_n, a.eps));
    } else if constexpr (MODE == 2) {
      // one pass with a shift: K = the mean of the first vector of every lane that has a whole one
      float k0;
      {
        float2 f[H];
        unpack2<T>(*reinterpret_cast<const uint4*>(st + (size_t)(lane < nfull ? lane : 0) * 16), f);
        float2 t = f[0];
#pragma unroll
        for (int h = 1; h < H; ++h) t = add2(t, f[h]);
        const int nk = nfull < 32 ? nfull : 32;
        k0 = warp_sum(lane < nfull ? t.x + t.y : 0.0f) / (float)(nk * E);
      }
      const float2 nk2 = dup2(-k0);
      float2 s1[H], s2[H];
#pragma unroll
      for (int h = 0; h < H; ++h) s1[h] = s2[h] = dup2(0.0f);
#pragma unroll 4
      for (int v = lane; v < nfull; v += 32) {
        float2 f[H];
        unpack2<T>(*reinterpret_cast<const uint4*>(st + (size_t)v * 16), f);
#pragma unroll
        for (int h = 0; h < H; ++h) {
          const float2 d = add2(f[h], nk2);
          s1[h] = add2(s1[h], d);
          s2[h] = fma2(d, d, s2[h]);
        }
      }
      if (tcnt && lane == (tv & 31))
#pragma unroll
        for (int h = 0; h < H; ++h) {
          const float d0 = 2 * h < tcnt ? tail[h].x - k0 : 0.0f;
          const float d1 = 2 * h + 1 < tcnt ? tail[h].y - k0 : 0.0f;
          s1[h].x += d0, s1[h].y += d1;
          s2[h].x = fmaf(d0, d0, s2[h].x), s2[h].y = fmaf(d1, d1, s2[h].y);
        }
      float2 t1 = s1[0], t2 = s2[0];
#pragma unroll
      for (int h = 1; h < H; ++h) t1 = add2(t1, s1[h]), t2 = add2(t2, s2[h]);
      const float m1 = warp_sum(t1.x + t1.y) * inv_n;  // mean - K
      const float m2 = warp_sum(t2.x + t2.y) * inv_n;
      mu = k0 + m1;
      stat_a = rsqrtf(fmaxf(fmaf(-m1, m1, m2), 0.0f) + a.eps);
    } else {
      float2 acc[H];
#pragma unroll
      for (int h = 0; h < H; ++h) acc[h] = dup2(0.0f);
#pragma unroll 4
      for (int v = lane; v < nfull; v += 32) {
        float2 f[H];
        unpack2<T>(*reinterpret_cast<const uint4*>(st + (size_t)v * 16), f);
#pragma unroll
        for (int h = 0; h < H; ++h) acc[h] = add2(acc[h], f[h]);
      }
      if (tcnt && lane == (tv & 31))
#pragma unroll
        for (int h = 0; h < H; ++h) acc[h] = add2(acc[h], tail[h]);
      float2 t = acc[0];
#pragma unroll
      for (int h = 1; h < H; ++h) t = add2(t, acc[h]);
      mu = warp_sum(t.x + t.y) * inv_n;
      // centred sum of squares from the same shared-memory row (no E[x^2] - E[x]^2 cancellation)
      const float2 nmu = dup2(-mu);
#pragma unroll
      for (int h = 0; h < H; ++h) acc[h] = dup2(0.0f);
#pragma unroll 4
      for (int v = lane; v < nfull; v += 32) {
        float2 f[H];
        unpack2<T>(*reinterpret_cast<const uint4*>(st + (size_t)v * 16), f);
#pragma unroll
        for (int h = 0; h < H; ++h) {
          const float2 d = add2(f[h], nmu);
          acc[h] = fma2(d, d, acc[h]);
        }
      }
      if (tcnt && lane == (tv & 31))
#pragma unroll
        for (int h = 0; h < H; ++h) {
          const float d0 = 2 * h < tcnt ? tail[h].x - mu : 0.0f;
          const float d1 = 2 * h + 1 < tcnt ? tail[h].y - mu : 0.0f;
          acc[h].x = fmaf(d0, d0, acc[h].x);
          acc[h].y = fmaf(d1, d1, acc[h].y);
        }
      t = acc[0];
#pragma unroll
      for (int h = 1; h < H; ++h) t = add2(t, acc[h]);
      const float q = warp_sum(t.x + t.y);
      stat_a = rsqrtf(fmaf(q, inv_n, a.eps));
    }
    // output pass. LayerNorm centres first, then scales: (x - mu) s. The fused x s - mu s would
    // round mu s, an error of up to half an ulp of mu s in every normalized value, which for a
    // near-constant row (large s) with a mean away from 0 exceeds the output's own rounding.
    const float2 ra = dup2(stat_a), nmu2 = dup2(-mu);
    T* yrow = y + m * a.ldy;
#pragma unroll 4
    for (int v = lane; v < nvec; v += 32) {
      float2 f[H], wv[H], o[H];
      if (v < nfull) {
        unpack2<T>(*reinterpret_cast<const uint4*>(st + (size_t)v * 16), f);
      } else {
#pragma unroll
        for (int h = 0; h < H; ++h) f[h] = tail[h];
      }
      if constexpr (P16)
        param_pairs<T>(reinterpret_cast<const uint8_t*>(pw), v, wv);
      else
        prm_pairs<H>(pw, v, nvec, wv);
      if constexpr (LN) {
        float2 bv[H];
        if constexpr (P16)
          param_pairs<T>(reinterpret_cast<const uint8_t*>(pb), v, bv);
        else
          prm_pairs<H>(pb, v, nvec, bv);
#pragma unroll
        for (int h = 0; h < H; ++h) {
          const float2 z = fma2(mul2(add2(f[h], nmu2), ra), wv[h], bv[h]);
          if constexpr (EPI == EPI_GELU_TANH)
            o[h] = gelu_of_half2<FAST>(z);
          else
            o[h] = epi_fwd2<EPI, FAST>(z);
        }
      } else {
#pragma unroll
        for (int h = 0; h < H; ++h) o[h] = epi_fwd2<EPI, FAST>(mul2(mul2(f[h], ra), wv[h]));
      }
      store_pairs<T>(yrow, v, nfull, N, o);
    }
    if (lane == 0) {
      if constexpr (LN) {
        if (a.stat0) a.stat0[m] = mu;
        if (a.stat1) a.stat1[m] = stat_a;
      } else {
        if (a.stat0) a.stat0[m] = stat_a;
      }
    }
    __syncwarp();  // every lane's reads of this stage are done before it is refilled
    if (++s == S) s = 0, ph ^= 1u;
  }
  // copies still in flight (only after a timed-out wait) land before the CTA may exit
  if (lane == 0 && failed)
    for (int t = 0; t < S; ++t)
      if (pend & (1u << t)) (void)mbar_wait(&full[t], (pph >> t) & 1u, nullptr, kWaitLimitNs);
}

// ---------------------------------------------------------------- dispatch

template <typename T, int MODE>
void* pick_warp_fwd(int epi, bool gemma) {
  if constexpr (MODE != 0) {
    if (epi == EPI_GELU_TANH) return (void*)norm_fwd_warp<T, MODE, EPI_GELU_TANH, false>;
    if (epi == EPI_SILU) return (void*)norm_fwd_warp<T, MODE, EPI_SILU, false>;
    return (void*)norm_fwd_warp<T, MODE, EPI_NONE, false>;
  } else {
    if (epi == EPI_GELU_TANH)
      return gemma ? (void*)norm_fwd_warp<T, 0, EPI_GELU_TANH, true> : (void*)norm_fwd_warp<T, 0, EPI_GELU_TANH, false>;
    if (epi == EPI_SILU)
      return gemma ? (void*)norm_fwd_warp<T, 0, EPI_SILU, true> : (void*)norm_fwd_warp<T, 0, EPI_SILU, false>;
    return gemma ? (void*)norm_fwd_warp<T, 0, EPI_NONE, true> : (void*)norm_fwd_warp<T, 0, EPI_NONE, false>;
  }
}

// LayerNorm: the one-pass shifted statistics unless fwd_path 2 asks for the two-pass form
template <typename T>
void* pick_warp_fwd_t(bool ln, int epi, bool gemma) {
  if (!ln) return pick_warp_fwd<T, 0>(epi, gemma);
  return g_tune.fwd_path == 2 ? pick_warp_fwd<T, 1>(epi, gemma) : pick_warp_fwd<T, 2>(epi, gemma);
}

}  // namespace

gn_status launch_norm_fwd_warp(bool ln, const void* x, const void* w, const void* b, void* y, float* stat0,
                               float* stat1, int64_t rows, int64_t N, int64_t ldx, int64_t ldy, float eps, bool gemma,
                               int epi, gn_dtype dt, cudaStream_t stream) {
  const int64_t es = (int64_t)dt_size(dt);
  const int64_t E = 16 / es;
  const int64_t nfull = N / E;
  if (nfull < 1) return GN_ERR_UNSUPPORTED;
  const uint32_t slot = pipe_slot_bytes(nfull * 16);
  // a parameter vector: fp32 copies, or the row type for LayerNorm on bf16 rows (P16 in the kernel)
  const uint32_t pbytes = pipe_slot_bytes((N + E - 1) / E * E * (ln && dt == GN_BF16 ? 2 : 4));
  unsigned* err = device_err_word();
  if (!err) return GN_ERR_CUDA;
  const size_t limit = smem_optin();
  const size_t fixed = kWarpFwdHeader + (ln ? 2u : 1u) * (size_t)pbytes;
  // One stage per warp and as many warps as fit, in whole multiples of 4: each warp loads its
  // row, then computes it, and the other warps' loads and arithmetic fill the gap; a CTA's warps
  // are spread over the SM's 4 schedulers, and the work is per warp, so an uneven split leaves
  // the schedulers with a fifth warp the slowest. Measured on B200 (LayerNorm + GeLU, x [32768,
  // 5120] bf16, GB/s): 2 stages x 9 warps 4280; 1 stage x 8 / 15 / 16 / 17 / 18 warps 3870 / 5220
  // / 5530 / 5100 / 5280.
  int stages = g_tune.stages ? g_tune.stages : 1;
  if (stages < 1 || stages > kWarpFwdMaxStages) return GN_ERR_UNSUPPORTED;
  if (limit <= fixed) return GN_ERR_UNSUPPORTED;
  int warps = (int)((limit - fixed) / ((size_t)stages * slot));
  if (warps > kWarpFwdMaxWarps) warps = kWarpFwdMaxWarps;
  warps &= ~3;
  if (g_tune.fwd_warps && g_tune.fwd_warps < warps) warps = g_tune.fwd_warps;
  if (warps < 4) return GN_ERR_UNSUPPORTED;
  const size_t smem = fixed + (size_t)warps * stages * slot;
  void* kern = dt == GN_BF16 ? pick_warp_fwd_t<__nv_bfloat16>(ln, epi, gemma) : pick_warp_fwd_t<float>(ln, epi, gemma);
  int grid = persistent_grid(kern, warps * 32, smem, 1);
  if (grid <= 0) return GN_ERR_CUDA;
  const int64_t need = (rows + warps - 1) / warps;
  if (need < grid) grid = (int)need;
  WarpFwdArgs a{x, w, b, y, stat0, stat1, rows, ldx, ldy, (int)N, stages, slot, pbytes, eps, err};
  void* args[] = {&a};
  if (cudaLaunchKernel(kern, dim3(grid), dim3(warps * 32), args, smem, stream) != cudaSuccess) return GN_ERR_CUDA;
  count_launches(1);
  return launch_status();
}

}  // namespace gn
