// gn_common.cuh - device building blocks shared by the sm_100a kernels of libgn.
//
// * 16-byte vector I/O: 8 bf16 or 4 fp32 per access, widened to fp32 in registers.
// * 1-D TMA bulk copies (cp.async.bulk global -> shared, completion counted on an mbarrier)
//   for the row pipeline, with a bounded wait: a wait that runs past kWaitLimitNs records
//   the wait-timeout bit in the caller's error word and returns false instead of spinning.
// * warp reductions and the tanh-GeLU / SiLU epilogues with their derivatives.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gn {

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s: far above any real copy latency
constexpr unsigned kDevErrWaitTimeout = 1u;  // GN_DEVERR_WAIT_TIMEOUT in gn.h

// ---------------------------------------------------------------- element traits

template <typename T>
struct Vec;

template <>
struct Vec<float> {
  static constexpr int N = 4;  // elements per 16-byte vector
  __device__ __forceinline__ static void unpack(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
  __device__ __forceinline__ static uint4 pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
  __device__ __forceinline__ static float load1(const float* p) { return *p; }
  __device__ __forceinline__ static void store1(float* p, float v) { *p = v; }
};

template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void split(uint32_t w, float& lo, float& hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xffff0000u);
  }
  __device__ __forceinline__ static void unpack(const uint4& u, float (&f)[8]) {
    split(u.x, f[0], f[1]);
    split(u.y, f[2], f[3]);
    split(u.z, f[4], f[5]);
    split(u.w, f[6], f[7]);
  }
  __device__ __forceinline__ static uint32_t join(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even, both halves
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ __forceinline__ static uint4 pack(const float (&f)[8]) {
    return make_uint4(join(f[0], f[1]), join(f[2], f[3]), join(f[4], f[5]), join(f[6], f[7]));
  }
  __device__ __forceinline__ static float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  __device__ __forceinline__ static void store1(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// ---------------------------------------------------------------- packed fp32 pairs
// sm_100 executes one FMA / MUL / ADD on two fp32 lanes per instruction (CUDA's __ffma2_rn,
// __fmul2_rn, __fadd2_rn; round to nearest even per lane, like the scalar forms).

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 dup2(float a) { return make_float2(a, a); }

// a 16-byte vector as E/2 element pairs (elements 2i, 2i+1 in .x, .y)
template <typename T>
__device__ __forceinline__ void unpack2(const uint4& u, float2 (&f)[Vec<T>::N / 2]) {
  if constexpr (sizeof(T) == 2) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
  } else {
    f[0] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
    f[1] = make_float2(__uint_as_float(u.z), __uint_as_float(u.w));
  }
}

template <typename T>
__device__ __forceinline__ uint4 pack2(const float2 (&f)[Vec<T>::N / 2]) {
  if constexpr (sizeof(T) == 2) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __float22bfloat162_rn(f[i]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    return make_uint4(__float_as_uint(f[0].x), __float_as_uint(f[0].y), __float_as_uint(f[1].x),
                      __float_as_uint(f[1].y));
  }
}

// streaming 16-byte global access (read-once / write-once data)
__device__ __forceinline__ uint4 ld_stream(const void* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ void st_stream(void* p, const uint4& v) { __stcs(reinterpret_cast<uint4*>(p), v); }

// element i of a weight vector, widened (w == nullptr -> dflt)
template <typename T>
__device__ __forceinline__ float ld_param(const T* w, int64_t i, float dflt) {
  return w ? Vec<T>::load1(w + i) : dflt;
}

// ---------------------------------------------------------------- mbarrier + bulk copy

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// make the initialised barriers visible to the async (TMA) proxy; call before __syncthreads
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

// The thread may be suspended inside try_wait until the phase completes or about
// kSuspendHintNs pass, so a waiting warp does not spend issue slots polling.
#ifndef GN_SUSPEND_HINT_NS
#define GN_SUSPEND_HINT_NS 100000
#endif
constexpr uint32_t kSuspendHintNs = GN_SUSPEND_HINT_NS;

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of `bar` to complete, for at most limit_ns. On timeout the error
// word gets GN_DEVERR_WAIT_TIMEOUT and the function returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned* err,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      if (err) atomicOr(err, kDevErrWaitTimeout);
      return false;
    }
  }
  return true;
}

// 1-D bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from global to
// this CTA's shared memory; completion is counted on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// ---------------------------------------------------------------- programmatic dependent launch
// A backward kernel lets the launch of the grid that follows it in the stream (the weight-gradient
// column reduction, launched with programmatic stream serialization) start before it completes;
// that grid waits in pdl_wait() for this grid's completion and memory before it reads anything.

#ifndef GN_PDL
#define GN_PDL 1
#endif
__device__ __forceinline__ void pdl_launch_dependents() {
  if (GN_PDL) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
  if (GN_PDL) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------- reductions

template <int WIDTH = 32>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = WIDTH / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o, WIDTH);
  return v;
}

// runtime-width variant (width a power of two <= 32); every lane gets the same total. The
// width is uniform across the warp, so the dispatch to the unrolled forms costs one branch.
__device__ __forceinline__ float group_sum_rt(float v, int width) {
  switch (width) {
    case 32: return group_sum<32>(v);
    case 16: return group_sum<16>(v);
    case 8: return group_sum<8>(v);
    case 4: return group_sum<4>(v);
    case 2: return group_sum<2>(v);
    default: return v;
  }
}

// ---------------------------------------------------------------- epilogues
// tanh-GeLU: 0.5 z (1 + tanh(k (z + 0.044715 z^3))), k = sqrt(2/pi). SiLU: z * sigmoid(z).
// bf16 outputs use the hardware tanh.approx / ex2-based __expf (error far below bf16
// rounding); fp32 outputs use the accurate expf, the tanh-GeLU through 1 +- tanh(u) formed from
// exp(-2|u|) (one_pm_tanh).

enum Epi { EPI_NONE = 0, EPI_GELU_TANH = 1, EPI_SILU = 2 };

constexpr float kGeluK = 0.7978845608028654f;  // sqrt(2/pi)
constexpr float kGeluC = 0.044715f;

template <bool FAST>
__device__ __forceinline__ float tanh_f(float x) {
  if constexpr (FAST) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
  } else {
    return tanhf(x);
  }
}

template <bool FAST>
__device__ __forceinline__ float sigmoid_f(float x) {
  if constexpr (FAST) {
    // approximate reciprocal (2 ulp): far below the bf16 rounding of the outputs; the correctly
    // rounded __frcp_rn is a multi-instruction sequence that made the SiLU kernels ALU-bound
    return __fdividef(1.0f, 1.0f + __expf(-x));
  } else {
    return 1.0f / (1.0f + expf(-x));
  }
}

// 1 + tanh(u) and 1 - tanh(u) from a = exp(-2|u|): tanh(|u|) = (1 - a) / (1 + a), so the two are
// 2 / (1 + a) and 2a / (1 + a), the smaller one without cancellation. The fp32 tanh-GeLU and its
// derivative use this form: with tanh(u) itself, 1 + tanh(u) keeps no significant bits once
// tanh(u) rounds to -1 (u < -9, z < -5.5), where the derivative is still ~1e-6.
__device__ __forceinline__ void one_pm_tanh(float u, float& p, float& q) {
  const float a = expf(-2.0f * fabsf(u));
  const float r = 2.0f / (1.0f + a);
  const float ra = r * a;
  p = u >= 0.0f ? r : ra;  // 1 + tanh(u)
  q = u >= 0.0f ? ra : r;  // 1 - tanh(u)
}

template <int EPI, bool FAST>
__device__ __forceinline__ float epi_fwd(float z) {
  if constexpr (EPI == EPI_GELU_TANH && !FAST) {
    float p, q;
    one_pm_tanh(z * fmaf(kGeluK * kGeluC, z * z, kGeluK), p, q);
    return 0.5f * z * p;
  } else if constexpr (EPI == EPI_GELU_TANH) {
    const float z2 = z * z;
    const float t = tanh_f<FAST>(z * fmaf(kGeluK * kGeluC, z2, kGeluK));  // k (z + c z^3)
    const float h = 0.5f * z;
    return fmaf(h, t, h);
  } else if constexpr (EPI == EPI_SILU) {
    return z * sigmoid_f<FAST>(z);
  } else {
    return z;
  }
}

// d epi / dz
template <int EPI, bool FAST>
__device__ __forceinline__ float epi_grad(float z) {
  if constexpr (EPI == EPI_GELU_TANH && !FAST) {
    // 0.5 (1 + t) + 0.5 z (1 - t)(1 + t) k' = 0.5 (1 + t) (1 + z (1 - t) k'), k' = k (1 + 3 c z^2)
    const float z2 = z * z;
    float p, q;
    one_pm_tanh(z * fmaf(kGeluK * kGeluC, z2, kGeluK), p, q);
    return 0.5f * p * fmaf(z * q, fmaf(3.0f * kGeluK * kGeluC, z2, kGeluK), 1.0f);
  } else if constexpr (EPI == EPI_GELU_TANH) {
    const float z2 = z * z;
    const float t = tanh_f<FAST>(z * fmaf(kGeluK * kGeluC, z2, kGeluK));
    // 0.5 (1 + t) + 0.5 z (1 - t^2) k (1 + 3 c z^2)
    const float k3 = fmaf(3.0f * 0.5f * kGeluK * kGeluC, z2, 0.5f * kGeluK);  // 0.5 k (1 + 3 c z^2)
    return fmaf(z * fmaf(-t, t, 1.0f), k3, fmaf(0.5f, t, 0.5f));
  } else if constexpr (EPI == EPI_SILU) {
    const float s = sigmoid_f<FAST>(z);
    return s * fmaf(z, 1.0f - s, 1.0f);
  } else {
    return 1.0f;
  }
}

// The same epilogues on a pair of lanes. On bf16 rows the forward tanh-GeLU runs on packed fp32x2
// instructions with the scalar form's operations, operand order and constants lane by lane, so
// each lane rounds exactly as epi_fwd; the fp32 form and SiLU run as two scalar evaluations.
template <bool FAST>
__device__ __forceinline__ float2 tanh2(float2 u) {
  return make_float2(tanh_f<FAST>(u.x), tanh_f<FAST>(u.y));
}

template <int EPI, bool FAST>
__device__ __forceinline__ float2 epi_fwd2(float2 z) {
  if constexpr (EPI == EPI_NONE) {
    return z;
  } else if constexpr (EPI == EPI_GELU_TANH && FAST) {
    const float2 z2 = mul2(z, z);
    const float2 t = tanh2<FAST>(mul2(z, fma2(dup2(kGeluK * kGeluC), z2, dup2(kGeluK))));
    const float2 h = mul2(dup2(0.5f), z);
    return fma2(h, t, h);
  } else {
    return make_float2(epi_fwd<EPI, FAST>(z.x), epi_fwd<EPI, FAST>(z.y));
  }
}

// tanh-GeLU of z = 2 h, given h: callers whose pre-activation is an affine map fold the 1/2 into
// its parameters (scaling by a power of two is exact). With h2 = h h = z^2 / 4 the argument
// k (z + c z^3) = h (2k + 8kc h2) and GeLU(z) = h + h tanh(.) take the same roundings as
// epi_fwd(z), one multiplication fewer.
template <bool FAST>
__device__ __forceinline__ float2 gelu_of_half2(float2 h) {
  if constexpr (!FAST) {  // the fp32 form: GeLU(z) = h (1 + tanh(u)), 1 + tanh(u) without cancellation
    float p0, p1, q;
    one_pm_tanh(h.x * fmaf(8.0f * (kGeluK * kGeluC), h.x * h.x, 2.0f * kGeluK), p0, q);
    one_pm_tanh(h.y * fmaf(8.0f * (kGeluK * kGeluC), h.y * h.y, 2.0f * kGeluK), p1, q);
    return make_float2(h.x * p0, h.y * p1);
  } else {
    const float2 h2 = mul2(h, h);
    const float2 t = tanh2<FAST>(mul2(h, fma2(dup2(8.0f * (kGeluK * kGeluC)), h2, dup2(2.0f * kGeluK))));
    return fma2(h, t, h);
  }
}

// On bf16 rows the tanh-GeLU gradient runs on packed fp32x2 instructions with the scalar form's
// operations, operand order and constants lane by lane (each lane rounds exactly as epi_grad);
// the fp32 form and SiLU run as two scalar evaluations.
template <int EPI, bool FAST>
__device__ __forceinline__ float2 epi_grad2(float2 z) {
  if constexpr (EPI == EPI_NONE) {
    return dup2(1.0f);
  } else if constexpr (EPI == EPI_GELU_TANH && FAST) {
    const float2 z2 = mul2(z, z);
    const float2 t = tanh2<FAST>(mul2(z, fma2(dup2(kGeluK * kGeluC), z2, dup2(kGeluK))));
    const float2 k3 = fma2(dup2(3.0f * 0.5f * kGeluK * kGeluC), z2, dup2(0.5f * kGeluK));
    const float2 s = fma2(make_float2(-t.x, -t.y), t, dup2(1.0f));  // 1 - t^2
    return fma2(mul2(z, s), k3, fma2(dup2(0.5f), t, dup2(0.5f)));
  } else {
    return make_float2(epi_grad<EPI, FAST>(z.x), epi_grad<EPI, FAST>(z.y));
  }
}

template <typename T>
constexpr bool fast_math_for() {
  return sizeof(T) == 2;  // bf16 I/O
}

}  // namespace gn
