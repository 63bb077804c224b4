// rope.cu - interleaved rotary position embedding, in place (Helios kernels article, section
// "内核二 FlashRoPE": pair i of a head at offsets 2i and 2i+1, rotated in one pass and written
// back in place, no intermediate tensors; the backward is the same kernel with sin negated),
// and the fused per-head RMSNorm + RoPE ("内核一 FlashNorm" and "内核二 FlashRoPE" applied to
// q and k together, section "基准实测").
//
// One kernel template serves the three operations. The work unit is a slab of HC consecutive
// heads of one token (b, s) of q and of k: HC*D contiguous elements per tensor, plus the
// token's cos/sin table rows. A persistent CTA is warp-specialised:
//   * warp 0 (one lane) is the producer: it walks the CTA's units grid-stride and moves each
//     unit into a shared-memory stage with 1-D TMA bulk copies, counted on the stage's `full`
//     mbarrier; before reusing a stage it waits on the stage's `empty` mbarrier;
//   * the other C warps are consumers: they wait on `full`, compute straight from shared
//     memory one 16-byte vector at a time (few live registers, so several CTAs share an SM),
//     store the results with 16-byte streaming stores, and each warp arrives on `empty`.
// No CTA-wide barrier sits on the per-unit path. Units are ordered token-major, so the table
// row of token s is fetched by neighbouring CTAs at about the same time. Every wait is bounded.
//
//   ROPE    : x <- rot(x, cos, sign*sin)                                   (in place)
//   QK_FWD  : r = rsqrt(mean_d x^2 + eps), out = rot(x r w', cos, sin), inv_rms = r
//   QK_BWD  : u = rot(dy, cos, -sin), g = u w', dx = r (g - x r mean_d(g x r)),
//             dw_d += u_d x_d r   (per tensor, fixed-order partials + column reduction)
// Lanes of one head (D*size/16 of them, a power of two <= 32) reduce with xor shuffles.
#include <mutex>

#include "gn_host.h"
#include "row_pipe.cuh"

namespace gn {
namespace {

enum Mode { ROPE = 0, QK_FWD = 1, QK_BWD = 2 };

constexpr int kMaxConsumerWarps = 10;
constexpr int kRopeMaxThreads = 32 * (1 + kMaxConsumerWarps);
constexpr int kRopeMaxStages = 8;

struct RopeArgs {
  const void* x[2];   // q, k inputs (k may be null: one tensor)
  const void* dy[2];  // QK_BWD: gradients of the outputs
  void* out[2];       // outputs (ROPE: == x, in place)
  const void* w[2];   // QK: weights [D]
  float* stat[2];     // QK_FWD: inv_rms out; QK_BWD: inv_rms in (cast)
  const float* cos;
  const float* sin;
  float* ws;          // QK_BWD: [gridDim.x][2*D] partial dw, or null
  int B, S, H, D, HC, NC;  // NC = H / HC slabs per token
  int ntens;               // 1 or 2
  int stages;
  int lph_shift;           // log2(lanes per head) when that is a power of two, else -1
  float eps;
  float sign;
  uint32_t units;          // B * S * NC
  uint32_t tslot, tabslot; // bytes of one tensor slot / the table slot in a stage
  uint32_t statslot;       // QK_BWD: bytes of one tensor's inv_rms slot in a stage
  int stat_staged;         // QK_BWD: the producer copies the unit's inv_rms values into the stage
  unsigned* err;
};

__host__ __device__ inline uint32_t round128(uint32_t v) { return (v + 127u) / 128u * 128u; }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// named barrier 1 over the consumer warps only (the producer warp never joins it)
__device__ __forceinline__ void consumers_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// OR of `pred` over the consumer warps (named barrier 2)
__device__ __forceinline__ int consumers_any(int nthreads, int pred) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.s32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 2, %2, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred), "r"(nthreads)
      : "memory");
  return r;
}

// The CTA's walk over the units u = blockIdx.x + i * gridDim.x, u = (s * B + b) * NC + c (slab c
// of batch b, token s). The decode takes divisions once per CTA; each step then adds the
// decoded stride with carries.
struct UnitWalk {
  uint32_t u;
  int c, b, s;     // decode of u
  int dc, db, ds;  // decode of the stride gridDim.x

  __device__ __forceinline__ static void decode(const RopeArgs& a, uint32_t v, int& c, int& b, int& s) {
    c = (int)(v % (uint32_t)a.NC);
    const uint32_t t = v / (uint32_t)a.NC;
    b = (int)(t % (uint32_t)a.B);
    s = (int)(t / (uint32_t)a.B);
  }
  __device__ __forceinline__ explicit UnitWalk(const RopeArgs& a) : u(blockIdx.x) {
    decode(a, blockIdx.x, c, b, s);
    decode(a, gridDim.x, dc, db, ds);
  }
  __device__ __forceinline__ void next(const RopeArgs& a) {
    u += gridDim.x;
    c += dc;
    int carry = c >= a.NC;
    if (carry) c -= a.NC;
    b += db + carry;
    carry = b >= a.B;
    if (carry) b -= a.B;
    s += ds + carry;
  }
  __device__ __forceinline__ int64_t token() const { return s; }
  __device__ __forceinline__ int64_t first_row(const RopeArgs& a) const {  // first head row
    return ((int64_t)b * a.S + s) * a.H + (int64_t)c * a.HC;
  }
};

struct VecCtx {
  const uint8_t* sb;   // the unit's stage
  const float* tcos;   // the token's table rows in the stage
  const float* tsin;
  const float* tstat;  // QK_BWD: the unit's inv_rms values in the stage (null: read from global)
  int sstat;           // floats between the tensors' inv_rms slots
  int64_t row0;        // first head row of the unit
  int lph, lph_shift;  // vectors per head (and log2 when a power of two, else -1)
  float inv_d;
};

// A 16-byte vector as two planes over its consecutive pairs: plane 0 holds the even element
// of each pair, plane 1 the odd one, two pairs per float2 (bf16: pairs 0-3 -> 2 float2 per
// plane; fp32: pairs 0-1 -> 1 float2). Element e = 4k + 2*lane + plane sits in plane
// `plane`, float2 k, component `lane`. In this layout the rotation, scaling and gradient
// arithmetic of a pair runs on packed fp32x2 instructions.
template <typename T>
struct Planes {
  static constexpr int E = Vec<T>::N;
  static constexpr int K = E / 4;
  __device__ __forceinline__ static void load(const uint4& u, float2 (&p0)[K], float2 (&p1)[K]) {
    if constexpr (sizeof(T) == 2) {
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};  // word i = pair i (even element in the low half)
#pragma unroll
      for (int k = 0; k < K; ++k) {
        p0[k] = make_float2(__uint_as_float(w[2 * k] << 16), __uint_as_float(w[2 * k + 1] << 16));
        p1[k] = make_float2(__uint_as_float(w[2 * k] & 0xffff0000u), __uint_as_float(w[2 * k + 1] & 0xffff0000u));
      }
    } else {
      p0[0] = make_float2(__uint_as_float(u.x), __uint_as_float(u.z));
      p1[0] = make_float2(__uint_as_float(u.y), __uint_as_float(u.w));
    }
  }
  __device__ __forceinline__ static uint4 store(const float2 (&p0)[K], const float2 (&p1)[K]) {
    if constexpr (sizeof(T) == 2) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < K; ++k) {
        w[2 * k] = Vec<T>::join(p0[k].x, p1[k].x);
        w[2 * k + 1] = Vec<T>::join(p0[k].y, p1[k].y);
      }
      return make_uint4(w[0], w[1], w[2], w[3]);
    } else {
      return make_uint4(__float_as_uint(p0[0].x), __float_as_uint(p1[0].x), __float_as_uint(p0[0].y),
                        __float_as_uint(p1[0].y));
    }
  }
  // element order <-> planes (per-column weights and weight gradients)
  __device__ __forceinline__ static void split(const float (&e)[E], float2 (&p0)[K], float2 (&p1)[K]) {
#pragma unroll
    for (int k = 0; k < K; ++k) {
      p0[k] = make_float2(e[4 * k], e[4 * k + 2]);
      p1[k] = make_float2(e[4 * k + 1], e[4 * k + 3]);
    }
  }
  __device__ __forceinline__ static void merge(const float2 (&p0)[K], const float2 (&p1)[K], float (&e)[E]) {
#pragma unroll
    for (int k = 0; k < K; ++k) {
      e[4 * k] = p0[k].x, e[4 * k + 2] = p0[k].y;
      e[4 * k + 1] = p1[k].x, e[4 * k + 3] = p1[k].y;
    }
  }
};

// One 16-byte vector w of tensor TT's slab of the current unit (valid when w < nv_t).
// wt0/wt1: this lane's weights w' in planes; dw0/dw1: its weight-gradient accumulators.
// LPH: lanes (16-byte vectors) per head when known at compile time (16 for bf16 heads of 128,
// the benchmark's), so that the head index, the lane within the head and the head shuffles
// fold to constants; 0 = taken from the launch.
template <typename T, int MODE, int TT, int LPH>
__device__ __forceinline__ void rope_vec(const RopeArgs& a, const VecCtx& c, int w, int nv_t,
                                         const float2 (&wt0)[Planes<T>::K], const float2 (&wt1)[Planes<T>::K],
                                         float2 (&dw0)[Planes<T>::K], float2 (&dw1)[Planes<T>::K]) {
  using PL = Planes<T>;
  constexpr int K = PL::K;
  constexpr int P = Vec<T>::N / 2;
  const bool valid = w < nv_t;
  if (!valid) w = 0;
  int hh, l;
  if constexpr (LPH > 0) {
    hh = w / LPH;
    l = w % LPH;
  } else if (c.lph_shift >= 0) {
    hh = w >> c.lph_shift;
    l = w & (c.lph - 1);
  } else {
    hh = w / c.lph;
    l = w - hh * c.lph;
  }
  float2 x0[K], x1[K], cs[K], sn[K], o0[K], o1[K];
  PL::load(*reinterpret_cast<const uint4*>(c.sb + TT * a.tslot + (size_t)w * 16), x0, x1);
  if constexpr (P == 4) {
    const float4 c4 = *reinterpret_cast<const float4*>(c.tcos + l * P);
    const float4 s4 = *reinterpret_cast<const float4*>(c.tsin + l * P);
    cs[0] = make_float2(c4.x, c4.y), cs[1] = make_float2(c4.z, c4.w);
    sn[0] = make_float2(s4.x, s4.y), sn[1] = make_float2(s4.z, s4.w);
  } else {
    cs[0] = *reinterpret_cast<const float2*>(c.tcos + l * P);
    sn[0] = *reinterpret_cast<const float2*>(c.tsin + l * P);
  }
  if constexpr (MODE == ROPE) {
    // (x0, x1) -> (x0 c - x1 s', x0 s' + x1 c), s' = sign * s
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const float2 s = mul2(dup2(a.sign), sn[k]), ns = mul2(dup2(-a.sign), sn[k]);
      o0[k] = fma2(x1[k], ns, mul2(x0[k], cs[k]));
      o1[k] = fma2(x0[k], s, mul2(x1[k], cs[k]));
    }
  } else if constexpr (MODE == QK_FWD) {
    float2 ss2 = fma2(x0[0], x0[0], mul2(x1[0], x1[0]));
#pragma unroll
    for (int k = 1; k < K; ++k) ss2 = fma2(x1[k], x1[k], fma2(x0[k], x0[k], ss2));
    const float ss = LPH > 0 ? group_sum<LPH>(ss2.x + ss2.y) : group_sum_rt(ss2.x + ss2.y, c.lph);
    const float r = rsqrtf(fmaf(ss, c.inv_d, a.eps));
    const float2 r2 = dup2(r);
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const float2 n0 = mul2(x0[k], mul2(r2, wt0[k]));
      const float2 n1 = mul2(x1[k], mul2(r2, wt1[k]));
      const float2 ns = mul2(dup2(-1.0f), sn[k]);
      o0[k] = fma2(n1, ns, mul2(n0, cs[k]));
      o1[k] = fma2(n0, sn[k], mul2(n1, cs[k]));
    }
    if (valid && l == 0 && a.stat[TT]) a.stat[TT][c.row0 + hh] = r;
  } else {  // QK_BWD
    // r = 0: invalid lanes add nothing
    const float r = !valid ? 0.0f : c.tstat ? c.tstat[TT * c.sstat + hh] : __ldg(a.stat[TT] + c.row0 + hh);
    const float2 r2 = dup2(r);
    float2 d0[K], d1[K];
    PL::load(*reinterpret_cast<const uint4*>(c.sb + (a.ntens + TT) * a.tslot + (size_t)w * 16), d0, d1);
    float2 gw0[K], gw1[K], h0[K], h1[K], cd2 = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < K; ++k) {
      // inverse rotation of the output gradient: (d0 c + d1 s, d1 c - d0 s)
      const float2 ns = mul2(dup2(-1.0f), sn[k]);
      const float2 g0 = fma2(d1[k], sn[k], mul2(d0[k], cs[k]));
      const float2 g1 = fma2(d0[k], ns, mul2(d1[k], cs[k]));
      h0[k] = mul2(x0[k], r2);
      h1[k] = mul2(x1[k], r2);
      gw0[k] = mul2(g0, wt0[k]);
      gw1[k] = mul2(g1, wt1[k]);
      cd2 = fma2(gw1[k], h1[k], fma2(gw0[k], h0[k], cd2));
      dw0[k] = fma2(g0, h0[k], dw0[k]);
      dw1[k] = fma2(g1, h1[k], dw1[k]);
    }
    const float cd = (LPH > 0 ? group_sum<LPH>(cd2.x + cd2.y) : group_sum_rt(cd2.x + cd2.y, c.lph)) * c.inv_d;
    const float2 ncd = dup2(-cd);
#pragma unroll
    for (int k = 0; k < K; ++k) {
      o0[k] = mul2(r2, fma2(h0[k], ncd, gw0[k]));
      o1[k] = mul2(r2, fma2(h1[k], ncd, gw1[k]));
    }
  }
  if (valid) st_stream(static_cast<T*>(a.out[TT]) + c.row0 * a.D + (int64_t)w * Vec<T>::N, PL::store(o0, o1));
}

template <typename T, int MODE, bool GEMMA, int LPH>
__global__ void __launch_bounds__(kRopeMaxThreads, 2) rope_kernel(const RopeArgs a) {
  using V = Vec<T>;
  constexpr int E = V::N;      // elements per 16-byte vector
  constexpr bool BWD = MODE == QK_BWD;
  constexpr bool NORM = MODE != ROPE;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kRopeMaxStages;
  uint8_t* data = smem + 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ncw = (int)(blockDim.x >> 5) - 1;  // consumer warps
  const int D = a.D, HC = a.HC;
  const int lph = LPH > 0 ? LPH : D / E;       // vectors (lanes) per head
  const int nv_t = HC * lph;                   // vectors per tensor slab
  const uint32_t nslots = (uint32_t)a.ntens * (BWD ? 2u : 1u);
  const uint32_t sstride = nslots * a.tslot + a.tabslot + (BWD ? (uint32_t)a.ntens * a.statslot : 0u);
  const uint32_t slab_bytes = (uint32_t)(HC * D * (int)sizeof(T));
  const uint32_t tab_bytes = (uint32_t)(D / 2 * 4);
  const bool stat_staged = BWD && a.stat_staged;
  const uint32_t stat_bytes = stat_staged ? (uint32_t)(HC * 4) : 0u;
  if constexpr (BWD) pdl_launch_dependents();  // the column reduction that follows may launch early

  if (threadIdx.x == 0) {
    for (int st = 0; st < a.stages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], (uint32_t)ncw);
    }
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    int st = 0;
    uint32_t ph = 0, used = 0, lastph = 0;
    uint32_t k = 0;
    for (UnitWalk uw(a); uw.u < a.units; uw.next(a), ++k) {
      if (k >= (uint32_t)a.stages && !mbar_wait(&empty[st], ph ^ 1u, a.err)) break;
      const int64_t row0 = uw.first_row(a), s = uw.token();
      const int64_t eoff = row0 * D;
      uint8_t* sb = data + (size_t)st * sstride;
      mbar_expect_tx(&full[st], nslots * slab_bytes + 2 * tab_bytes + (uint32_t)a.ntens * stat_bytes);
      for (int t = 0; t < a.ntens; ++t) {
        bulk_g2s(sb + t * a.tslot, static_cast<const T*>(a.x[t]) + eoff, slab_bytes, &full[st]);
        if constexpr (BWD)
          bulk_g2s(sb + (a.ntens + t) * a.tslot, static_cast<const T*>(a.dy[t]) + eoff, slab_bytes, &full[st]);
      }
      uint8_t* tb = sb + nslots * a.tslot;
      bulk_g2s(tb, a.cos + (int64_t)s * (D / 2), tab_bytes, &full[st]);
      bulk_g2s(tb + tab_bytes, a.sin + (int64_t)s * (D / 2), tab_bytes, &full[st]);
      if (stat_staged)  // the HC saved statistics of the unit's head rows, per tensor
        for (int t = 0; t < a.ntens; ++t)
          bulk_g2s(tb + a.tabslot + t * a.statslot, a.stat[t] + row0, stat_bytes, &full[st]);
      used |= 1u << st;
      lastph = (lastph & ~(1u << st)) | (ph << st);
      if (++st == a.stages) st = 0, ph ^= 1u;
    }
    // every copy this CTA issued has landed before the CTA may exit (immediate when the
    // consumers consumed them all)
    for (int t = 0; t < a.stages; ++t)
      if (used & (1u << t)) (void)mbar_wait(&full[t], (lastph >> t) & 1u, a.err);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int ct = threadIdx.x - 32, nct = ncw * 32;
  const int li = a.lph_shift >= 0 ? (ct & (lph - 1)) : 0;  // NORM: lane within the head (fixed)
  constexpr int K = Planes<T>::K;
  float2 wq0[K], wq1[K], wk0[K], wk1[K], dq0[K], dq1[K], dk0[K], dk1[K];
  {
    float wq[E], wk[E];
#pragma unroll
    for (int e = 0; e < E; ++e) wq[e] = wk[e] = 0.0f;
    if constexpr (NORM) {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int d = li * E + e;
        wq[e] = (GEMMA ? 1.0f : 0.0f) + V::load1(static_cast<const T*>(a.w[0]) + d);
        if (a.ntens > 1) wk[e] = (GEMMA ? 1.0f : 0.0f) + V::load1(static_cast<const T*>(a.w[1]) + d);
      }
    }
    Planes<T>::split(wq, wq0, wq1);
    Planes<T>::split(wk, wk0, wk1);
#pragma unroll
    for (int k = 0; k < K; ++k) dq0[k] = dq1[k] = dk0[k] = dk1[k] = make_float2(0.0f, 0.0f);
  }
  const float inv_d = 1.0f / (float)D;
  int failed = 0;
  int st = 0;
  uint32_t ph = 0;
  for (UnitWalk uw(a); uw.u < a.units; uw.next(a)) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[st], ph, a.err));
    if (!ok) {
      failed = 1;
      break;
    }
    const int64_t row0 = uw.first_row(a);  // first head row of the unit
    const uint8_t* sb = data + (size_t)st * sstride;
    const float* tcos = reinterpret_cast<const float*>(sb + nslots * a.tslot);
    const float* tstat = stat_staged ? reinterpret_cast<const float*>(sb + nslots * a.tslot + a.tabslot) : nullptr;
    const VecCtx ctx{sb, tcos, tcos + D / 2, tstat, (int)(a.statslot / 4), row0, lph, a.lph_shift, inv_d};
    // Each pass covers one tensor (the tensor is a compile-time argument of the body); the
    // trip count is the same for every lane of a warp, so the head shuffles see full warps.
    for (int vb = 0; vb < nv_t; vb += nct) rope_vec<T, MODE, 0, LPH>(a, ctx, vb + ct, nv_t, wq0, wq1, dq0, dq1);
    if (a.ntens > 1)
      for (int vb = 0; vb < nv_t; vb += nct) rope_vec<T, MODE, 1, LPH>(a, ctx, vb + ct, nv_t, wk0, wk1, dk0, dk1);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    if (++st == a.stages) st = 0, ph ^= 1u;
  }

  if constexpr (BWD) {
    // combine the consumers' dw partials in thread order (the stages are idle now)
    if (consumers_any(nct, failed) || !a.ws) return;
    consumers_sync(nct);
    float* red = reinterpret_cast<float*>(data);  // [nct][2][E]
    float dwq[E], dwk[E];
    Planes<T>::merge(dq0, dq1, dwq);
    Planes<T>::merge(dk0, dk1, dwk);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      red[(ct * 2 + 0) * E + e] = dwq[e];
      red[(ct * 2 + 1) * E + e] = dwk[e];
    }
    consumers_sync(nct);
    float* part = a.ws + (int64_t)blockIdx.x * 2 * D;
    for (int col = ct; col < 2 * D; col += nct) {
      const int t = col / D, d = col - t * D, l = d / E, e = d - l * E;
      float acc = 0.0f;
      for (int th = l; th < nct; th += lph) acc += red[(th * 2 + t) * E + e];
      part[col] = acc;
    }
  }
}

// ---------------------------------------------------------------- planning

struct RopePlan {
  int HC, NC, cwarps, threads, stages, lph_shift;
  uint32_t tslot, tabslot, statslot;
  size_t smem;
};

gn_status plan_rope(int64_t B, int64_t S, int64_t H, int64_t D, int ntens, int mode, size_t es, RopePlan* p) {
  const int vec = (int)(16 / es);
  const int lph = (int)(D / vec);
  const int nslots = ntens * (mode == QK_BWD ? 2 : 1);
  const int64_t budget = g_tune.unit_bytes ? g_tune.unit_bytes : 48 * 1024;
  int HC = 1;
  for (int hc = (int)H; hc >= 1; --hc) {
    if (H % hc) continue;
    if ((int64_t)nslots * hc * D * (int64_t)es > budget && hc > 1) continue;
    HC = hc;
    break;
  }
  p->HC = HC;
  p->NC = (int)(H / HC);
  // consumer warps: the most (10 down to 4) whose 32*C threads divide one tensor slab's
  // vectors, so that no pass over a slab leaves lanes idle; 8 when none does
  const int64_t nv_t = (int64_t)HC * lph;
  int cw = 8;
  for (int c = kMaxConsumerWarps; c >= 4; --c)
    if (nv_t % (32 * c) == 0) {
      cw = c;
      break;
    }
  // the plain rotation (one CTA per SM) streams best with 8 consumer warps, two per scheduler,
  // even where a pass over the slab then leaves lanes idle (B200, q and k [1, 32760, 40, 128]:
  // 10 warps 6250-6390 GB/s, 8 warps 6410-6500); the qk-norm passes do more arithmetic per
  // vector and keep the divisor rule (8 warps: 5690-5920 against 5860-6050 forward)
  if (mode == ROPE && nv_t >= 32 * 8) cw = 8;
  if (g_tune.group_rows) cw = g_tune.group_rows > kMaxConsumerWarps ? kMaxConsumerWarps : g_tune.group_rows;
  p->cwarps = cw;
  p->threads = 32 * (1 + cw);
  p->lph_shift = (lph & (lph - 1)) == 0 ? __builtin_ctz((unsigned)lph) : -1;
  p->tslot = round128((uint32_t)(HC * D * (int64_t)es));
  p->tabslot = round128((uint32_t)(D * 4));
  p->statslot = mode == QK_BWD ? round128((uint32_t)(HC * 4)) : 0u;
  const size_t sstride = (size_t)nslots * p->tslot + p->tabslot + (size_t)ntens * p->statslot;
  // stage depth per CTA (measured on B200): the plain rotation computes so little that one
  // CTA per SM with ~4 stages of q and k streams best (deeper pipelines and more CTAs per SM
  // were slower: ~5750 against ~6340 GB/s at [1, 32760, 40, 128]); the qk-norm passes keep
  // ~64-96 KiB per CTA so that 2-3 CTAs share an SM
  const size_t depth = mode == ROPE ? 84 * 1024 : mode == QK_FWD ? 64 * 1024 : 96 * 1024;
  int stages = g_tune.stages ? g_tune.stages : (int)(depth / sstride);
  stages = stages < 2 ? 2 : stages > kRopeMaxStages ? kRopeMaxStages : stages;
  const size_t limit = smem_optin();
  while (stages > 1 && 128 + stages * sstride > limit) --stages;
  p->stages = stages;
  p->smem = 128 + stages * sstride;
  // the backward reuses the stages for the [consumers][2][vec] partial-sum table
  const size_t red = (size_t)32 * cw * 2 * vec * 4;
  if (mode == QK_BWD && red > stages * sstride) p->smem = 128 + red;
  if (p->smem > limit) return GN_ERR_UNSUPPORTED;
  if (B * S * p->NC >= (int64_t)1 << 31) return GN_ERR_UNSUPPORTED;
  return GN_OK;
}

template <typename T, int LPH>
void* pick_t(int mode, bool gemma) {
  if (mode == ROPE) return (void*)rope_kernel<T, ROPE, false, LPH>;
  if (mode == QK_FWD) return gemma ? (void*)rope_kernel<T, QK_FWD, true, LPH> : (void*)rope_kernel<T, QK_FWD, false, LPH>;
  return gemma ? (void*)rope_kernel<T, QK_BWD, true, LPH> : (void*)rope_kernel<T, QK_BWD, false, LPH>;
}

// heads of 16 vectors (bf16 D = 128, fp32 D = 64) take the instance with the head geometry
// folded in
void* pick(gn_dtype dt, int mode, bool gemma, int64_t D) {
  if (dt == GN_BF16) return D == 128 ? pick_t<__nv_bfloat16, 16>(mode, gemma) : pick_t<__nv_bfloat16, 0>(mode, gemma);
  return D == 64 ? pick_t<float, 16>(mode, gemma) : pick_t<float, 0>(mode, gemma);
}

gn_status setup(int64_t B, int64_t S, int64_t H, int64_t D, int ntens, int mode, gn_dtype dt, bool gemma,
                RopePlan* p, void** kern, int* grid) {
  gn_status st = plan_rope(B, S, H, D, ntens, mode, dt_size(dt), p);
  if (st != GN_OK) return st;
  *kern = pick(dt, mode, gemma, D);
  const int cap = g_tune.ctas_per_sm ? g_tune.ctas_per_sm : mode == ROPE ? 1 : 8;
  int g = persistent_grid(*kern, p->threads, p->smem, cap);
  if (g <= 0) return GN_ERR_CUDA;
  const int64_t units = B * S * p->NC;
  if (units < g) g = (int)(units > 0 ? units : 1);
  *grid = g;
  return GN_OK;
}

gn_status check_common(int64_t B, int64_t S, int64_t H, int64_t D, gn_dtype dt) {
  if (!dt_ok(dt)) return GN_ERR_DTYPE;
  if (B < 0 || S < 0 || H < 0 || D <= 0 || D % 8 || D > 4096) return GN_ERR_SHAPE;
  return GN_OK;
}

bool norm_head_ok(int64_t D, gn_dtype dt) {
  const int64_t lph = D * (int64_t)dt_size(dt) / 16;
  return lph >= 1 && lph <= 32 && (lph & (lph - 1)) == 0;
}

gn_status launch(void* kern, int grid, const RopePlan& p, RopeArgs& a, cudaStream_t s) {
  a.HC = p.HC;
  a.NC = p.NC;
  a.stages = p.stages;
  a.tslot = p.tslot;
  a.tabslot = p.tabslot;
  a.statslot = p.statslot;
  // the unit's saved statistics move with the unit when each unit's HC values start on a
  // 16-byte boundary (bulk copies need 16-byte aligned addresses and sizes); otherwise the
  // consumers read them from global memory
  a.stat_staged = p.statslot && p.HC % 4 == 0 && a.H % 4 == 0 && aligned16(a.stat[0]) &&
                  (a.ntens < 2 || aligned16(a.stat[1]));
  a.lph_shift = p.lph_shift;
  a.units = (uint32_t)((int64_t)a.B * a.S * p.NC);
  a.err = device_err_word();
  if (!a.err) return GN_ERR_CUDA;
  void* args[] = {&a};
  if (cudaLaunchKernel(kern, dim3(grid), dim3(p.threads), args, p.smem, s) != cudaSuccess) return GN_ERR_CUDA;
  count_launches(1);
  return launch_status();
}

}  // namespace
}  // namespace gn

using namespace gn;

extern "C" gn_status gn_rope_apply_inplace(void* q, void* k, const float* cos, const float* sin, int64_t B,
                                           int64_t S, int64_t H, int64_t D, int sign, gn_dtype dt,
                                           void* stream) {
  gn_status st = check_common(B, S, H, D, dt);
  if (st != GN_OK) return st;
  if (sign != 1 && sign != -1) return GN_ERR_SHAPE;
  if (B * S * H == 0) return GN_OK;
  if (!q || !cos || !sin) return GN_ERR_NULL;
  if (!aligned16(q) || (k && !aligned16(k)) || !aligned16(cos) || !aligned16(sin)) return GN_ERR_ALIGN;
  const int ntens = k ? 2 : 1;
  RopePlan p;
  void* kern = nullptr;
  int grid = 0;
  if ((st = setup(B, S, H, D, ntens, ROPE, dt, false, &p, &kern, &grid)) != GN_OK) return st;
  RopeArgs a{};
  a.x[0] = q;
  a.x[1] = k;
  a.out[0] = q;
  a.out[1] = k;
  a.cos = cos;
  a.sin = sin;
  a.B = (int)B, a.S = (int)S, a.H = (int)H, a.D = (int)D;
  a.ntens = ntens;
  a.sign = (float)sign;
  return launch(kern, grid, p, a, (cudaStream_t)stream);
}

extern "C" gn_status gn_qknorm_rope_fwd(const void* q, const void* k, const void* wq, const void* wk,
                                        const float* cos, const float* sin, void* q_out, void* k_out,
                                        float* inv_rms_q, float* inv_rms_k, int64_t B, int64_t S, int64_t H,
                                        int64_t D, float eps, int gemma, gn_dtype dt, void* stream) {
  gn_status st = check_common(B, S, H, D, dt);
  if (st != GN_OK) return st;
  if (!norm_head_ok(D, dt)) return GN_ERR_UNSUPPORTED;
  if (B * S * H == 0) return GN_OK;
  if (!q || !wq || !cos || !sin || !q_out) return GN_ERR_NULL;
  if (k && (!wk || !k_out)) return GN_ERR_NULL;
  if (!aligned16(q) || !aligned16(q_out) || (k && (!aligned16(k) || !aligned16(k_out))) || !aligned16(cos) ||
      !aligned16(sin))
    return GN_ERR_ALIGN;
  const int ntens = k ? 2 : 1;
  RopePlan p;
  void* kern = nullptr;
  int grid = 0;
  if ((st = setup(B, S, H, D, ntens, QK_FWD, dt, gemma != 0, &p, &kern, &grid)) != GN_OK) return st;
  RopeArgs a{};
  a.x[0] = q, a.x[1] = k;
  a.out[0] = q_out, a.out[1] = k_out;
  a.w[0] = wq, a.w[1] = wk;
  a.stat[0] = inv_rms_q, a.stat[1] = inv_rms_k;
  a.cos = cos, a.sin = sin;
  a.B = (int)B, a.S = (int)S, a.H = (int)H, a.D = (int)D;
  a.ntens = ntens;
  a.eps = eps;
  a.sign = 1.0f;
  return launch(kern, grid, p, a, (cudaStream_t)stream);
}

extern "C" size_t gn_qknorm_rope_bwd_workspace(int64_t B, int64_t S, int64_t H, int64_t D, gn_dtype dt) {
  if (check_common(B, S, H, D, dt) != GN_OK || !norm_head_ok(D, dt) || B * S * H == 0) return 0;
  // sized for two tensors (a call with k == NULL uses no more) and for the larger grid of
  // the plain and Gemma variants, whose occupancy may differ
  int grid = 0;
  for (int gemma = 0; gemma < 2; ++gemma) {
    RopePlan p;
    void* kern = nullptr;
    int g = 0;
    if (setup(B, S, H, D, 2, QK_BWD, dt, gemma != 0, &p, &kern, &g) != GN_OK) return 0;
    if (g > grid) grid = g;
  }
  return (size_t)grid * 2 * (size_t)D * sizeof(float);
}

extern "C" gn_status gn_qknorm_rope_bwd(const void* q, const void* k, const void* wq, const void* wk,
                                        const float* cos, const float* sin, const float* inv_rms_q,
                                        const float* inv_rms_k, const void* dq_out, const void* dk_out, void* dq,
                                        void* dk, float* dwq, float* dwk, void* ws, size_t ws_bytes, int64_t B,
                                        int64_t S, int64_t H, int64_t D, int gemma, gn_dtype dt, void* stream) {
  gn_status st = check_common(B, S, H, D, dt);
  if (st != GN_OK) return st;
  if (!norm_head_ok(D, dt)) return GN_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  if (B * S * H == 0) {
    if (dwq && cudaMemsetAsync(dwq, 0, (size_t)D * sizeof(float), s) != cudaSuccess) return GN_ERR_CUDA;
    if (dwk && cudaMemsetAsync(dwk, 0, (size_t)D * sizeof(float), s) != cudaSuccess) return GN_ERR_CUDA;
    return GN_OK;
  }
  if (!q || !wq || !cos || !sin || !inv_rms_q || !dq_out || !dq) return GN_ERR_NULL;
  if (k && (!wk || !inv_rms_k || !dk_out || !dk)) return GN_ERR_NULL;
  if (!aligned16(q) || !aligned16(dq_out) || !aligned16(dq) || !aligned16(cos) || !aligned16(sin) ||
      (k && (!aligned16(k) || !aligned16(dk_out) || !aligned16(dk))))
    return GN_ERR_ALIGN;
  const int ntens = k ? 2 : 1;
  RopePlan p;
  void* kern = nullptr;
  int grid = 0;
  if ((st = setup(B, S, H, D, ntens, QK_BWD, dt, gemma != 0, &p, &kern, &grid)) != GN_OK) return st;
  const bool wgrad = dwq || (k && dwk);
  if (wgrad) {
    if (!ws) return GN_ERR_WORKSPACE;
    if (!aligned16(ws)) return GN_ERR_ALIGN;
    if (ws_bytes < (size_t)grid * 2 * (size_t)D * sizeof(float)) return GN_ERR_WORKSPACE;
  }
  RopeArgs a{};
  a.x[0] = q, a.x[1] = k;
  a.dy[0] = dq_out, a.dy[1] = dk_out;
  a.out[0] = dq, a.out[1] = dk;
  a.w[0] = wq, a.w[1] = wk;
  a.stat[0] = const_cast<float*>(inv_rms_q), a.stat[1] = const_cast<float*>(inv_rms_k);
  a.cos = cos, a.sin = sin;
  a.ws = wgrad ? static_cast<float*>(ws) : nullptr;
  a.B = (int)B, a.S = (int)S, a.H = (int)H, a.D = (int)D;
  a.ntens = ntens;
  a.sign = 1.0f;
  if ((st = launch(kern, grid, p, a, s)) != GN_OK) return st;
  if (wgrad) return launch_colsum(a.ws, grid, 2 * D, D, dwq, k ? dwk : nullptr, s);
  return GN_OK;
}

// ---------------------------------------------------------------- fixed-scratch backward
// gn_qknorm_rope_bwd_noalloc: the same backward for callers that cannot allocate device
// memory. Its weight-gradient partials go to this file-scope array instead of a caller
// workspace. Every device that loads the library holds the array until the process exits.
// In host code the array's name is only a host-side stand-in; the device address comes from
// cudaGetSymbolAddress, taken once per device with that device current.

static constexpr size_t kQkFixedScratchBytes = 1u << 20;  // 1 MiB
static __device__ __align__(256) float gn_qk_fixed_scratch[kQkFixedScratchBytes / sizeof(float)];

namespace gn {
namespace {
constexpr int kScratchDevices = 64;
std::mutex g_scratch_mu;
float* g_scratch_ptr[kScratchDevices];

// device address of gn_qk_fixed_scratch on the current device (nullptr on error)
float* fixed_scratch() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kScratchDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, gn_qk_fixed_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  return g_scratch_ptr[dev];
}
}  // namespace
}  // namespace gn

extern "C" gn_status gn_qknorm_rope_bwd_noalloc(const void* q, const void* k, const void* wq, const void* wk,
                                                const float* cos, const float* sin, const float* inv_rms_q,
                                                const float* inv_rms_k, const void* dq_out, const void* dk_out,
                                                void* dq, void* dk, float* dwq, float* dwk, int64_t B, int64_t S,
                                                int64_t H, int64_t D, int gemma, gn_dtype dt, void* stream) {
  gn_status st = check_common(B, S, H, D, dt);
  if (st != GN_OK) return st;
  if (!norm_head_ok(D, dt)) return GN_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  if (B * S * H == 0) {
    if (dwq && cudaMemsetAsync(dwq, 0, (size_t)D * sizeof(float), s) != cudaSuccess) return GN_ERR_CUDA;
    if (dwk && cudaMemsetAsync(dwk, 0, (size_t)D * sizeof(float), s) != cudaSuccess) return GN_ERR_CUDA;
    return GN_OK;
  }
  if (!q || !wq || !cos || !sin || !inv_rms_q || !dq_out || !dq) return GN_ERR_NULL;
  if (k && (!wk || !inv_rms_k || !dk_out || !dk)) return GN_ERR_NULL;
  if (!aligned16(q) || !aligned16(dq_out) || !aligned16(dq) || !aligned16(cos) || !aligned16(sin) ||
      (k && (!aligned16(k) || !aligned16(dk_out) || !aligned16(dk))))
    return GN_ERR_ALIGN;
  const int ntens = k ? 2 : 1;
  RopePlan p;
  void* kern = nullptr;
  int grid = 0;
  if ((st = setup(B, S, H, D, ntens, QK_BWD, dt, gemma != 0, &p, &kern, &grid)) != GN_OK) return st;
  const bool wgrad = dwq || (k && dwk);
  float* scratch = nullptr;
  if (wgrad) {
    // one partial row of 2*D floats per block; every row read afterwards is written first
    if ((size_t)grid * 2 * (size_t)D * sizeof(float) > kQkFixedScratchBytes) return GN_ERR_WORKSPACE;
    scratch = fixed_scratch();
    if (!scratch) return GN_ERR_CUDA;
  }
  RopeArgs a{};
  a.x[0] = q, a.x[1] = k;
  a.dy[0] = dq_out, a.dy[1] = dk_out;
  a.out[0] = dq, a.out[1] = dk;
  a.w[0] = wq, a.w[1] = wk;
  a.stat[0] = const_cast<float*>(inv_rms_q), a.stat[1] = const_cast<float*>(inv_rms_k);
  a.cos = cos, a.sin = sin;
  a.ws = scratch;
  a.B = (int)B, a.S = (int)S, a.H = (int)H, a.D = (int)D;
  a.ntens = ntens;
  a.sign = 1.0f;
  if ((st = launch(kern, grid, p, a, s)) != GN_OK) return st;
  if (wgrad) return launch_colsum(scratch, grid, 2 * D, D, dwq, k ? dwk : nullptr, s);
  return GN_OK;
}
