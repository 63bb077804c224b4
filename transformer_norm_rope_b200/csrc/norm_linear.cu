// norm_linear.cu - normalization fused into the linear layer that follows it, on the tcgen05
// tensor cores (Janus-Pro inference page, section 4.1: LayerNorm, the first linear projection
// and SiLU in one kernel; HY-Motion optimization page, section 3.1: LayerNorm merged with the
// matrix multiplication after it, which saves the round trip of the normalized activations
// through HBM).
//
// The normalization is folded into the operands instead of being applied to the A tiles:
//   LayerNorm: xn[k] = (x[k] - mu) s g[k] + beta[k], so
//     y[m,n] = act( s_m * sum_k x[m,k] Wf[n,k] - s_m mu_m c[n] + d[n] )
//     with Wf[n,k] = bf16(g[k] W[n,k]), c[n] = sum_k Wf[n,k], d[n] = sum_k beta[k] W[n,k] + bias[n];
//   RMSNorm:   y[m,n] = act( r_m * sum_k x[m,k] Wf[n,k] + d[n] ), Wf = bf16(g'[k] W[n,k]), d = bias;
//   no norm:   y[m,n] = act( sum_k x[m,k] W[n,k] + bias[n] )   (the plain layer; TiledLinear).
// gn_norm_linear_prepare builds Wf, c and d once per weight (a memory-bound pass over W). The
// forward kernels stream the raw bf16 x and Wf through TMA straight into the tensor cores and
// apply the row statistics, the column terms and the activation when the fp32 accumulators
// are read back from tensor memory.
//
// Three kernels, by shape:
//   * norm_linear_pair_kernel (more than 128 rows and 256 columns): a cluster of two CTAs on
//     two SMs per 256 x 512 tile, tcgen05.mma.cta_group::2; the row statistics come from
//     norm_stats_kernel, a streaming pre-pass (see the comment above the pair kernel);
//   * norm_linear_kernel<MH> (otherwise): one CTA per 128 x 256 (MH = 1) or 256 x 256 (MH = 2)
//     tile, 2 + 4*MH warps:
//       warp 0      TMA producer: A tile [128*MH rows x 64 k] and B tile [256 rows x 64 k] per
//                   stage, 128-byte swizzled, as many stages as fit in shared memory;
//       warp 1      allocates the tensor memory; one lane issues tcgen05.mma (M=128, N=256,
//                   K=16, bf16 in, fp32 accumulate; MH instructions share each B tile) and
//                   commits each stage back to the producer, then the accumulators to the
//                   epilogue;
//       warps 2..   per-row statistics from the A tiles (thread = row; each copies its row of
//                   the tile to registers, consumes it and releases the stage), then the
//                   epilogue: tcgen05.ld of 32 accumulator columns at a time, corrections,
//                   activation, bf16 stores. A warp may only read the tensor-memory lanes
//                   32*(warp%4)..+31, so warp w owns rows 128h + 32*(w%4).. of the tile.
// Every mbarrier wait is bounded (kWaitLimitNs); a timeout records the error bit, the CTA skips
// its stores, waits for its own tensor-core work and copies, frees its tensor memory and exits.
#include <cuda.h>  // CUtensorMap and the cuTensorMapEncodeTiled prototype (types only)

#include <mutex>

#include "gn_common.cuh"
#include "gn_host.h"

namespace gn {
namespace {

#ifndef GN_NL_BK
#define GN_NL_BK 64
#endif
#ifndef GN_NL_BN
#define GN_NL_BN 256
#endif
constexpr int kUM = 128, kBN = GN_NL_BN, kBK = GN_NL_BK, kUK = 16;  // instruction M, tile N, tile K, instruction K
constexpr int kAccCols = 256;  // tensor-memory columns between the two accumulators
constexpr uint32_t kLine = kBK * 2;  // bytes of one tile row: 64 (BK 32, 64-byte swizzle) or 128
constexpr int kChunks = kLine / 16;  // 16-byte chunks per tile row
constexpr uint32_t kBBytes = kBN * kLine;

// A CTA computes MH x 128 rows by 256 columns: MH instructions of M = 128 share each B tile, so
// MH = 2 moves 64 KiB of operands per 8.4 MFLOP where MH = 1 moves 48 KiB per 4.2 MFLOP (the
// copies in flight per SM then cover the L2 latency at full tensor rate). Accumulator h sits in
// tensor-memory columns 256h..256h+255, lanes = rows 128h.. of the tile.
template <int MH>
struct Tile {
  static constexpr int BM = kUM * MH;
  // as many stages as fit in 227 KiB next to the barriers and column terms (at most 8)
  static constexpr int StagesFit = (int)((232448 - 1024 - 256 - 2 * kBN * 4) / (BM * kLine + kBN * kLine));
  static constexpr int Stages = StagesFit > 8 ? 8 : StagesFit;
  static constexpr int Threads = 64 + 128 * MH;  // producer, MMA, 4*MH statistics/epilogue warps
  static constexpr uint32_t ABytes = BM * kLine;
  static constexpr uint32_t StageBytes = ABytes + kBBytes;
  static constexpr uint32_t TmemCols = MH == 1 ? (kBN <= 128 ? 128 : 256) : 512;  // power of two >= kAccCols*(MH-1)+kBN
  static constexpr size_t Smem = 1024 /* alignment slack */ + (size_t)Stages * StageBytes + 256 + 2 * kBN * 4;
};

// Operand layouts in global (and shared) memory, bit 0 for A (x), bit 1 for B (Wf):
//   K-major  : A [M, K] / B [N, K] with K contiguous (the layer's natural layout);
//   MN-major : the operand stored transposed, A as [K, M] / B as [K, N] with M / N contiguous (a
//              product that contracts over the tokens, dW = dz^T x, reads both operands so,
//              and dx = dz W reads the weight so).
enum NlMajor { MAJ_A_MN = 1, MAJ_B_MN = 2 };

// instruction descriptor of tcgen05.mma kind::f16: D fp32 (bits 4-5 = 1), A and B bf16 (bits 7-9,
// 10-12 = 1), A / B MN-major (bits 15 / 16), N >> 3 at bit 17, M >> 4 at bit 24
constexpr uint32_t idesc_f16(int m, int n, int maj) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((maj & MAJ_A_MN) ? 1u << 15 : 0u) | ((maj & MAJ_B_MN) ? 1u << 16 : 0u) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

struct NlArgs {
  const float* c;  // [N] (LayerNorm)
  const float* d;  // [N] or null
  __nv_bfloat16* y;
  float* mean;  // [M] or null
  float* rstd;  // [M] or null
  int M, N, K;
  int64_t ldy;
  float eps;
  unsigned* err;
  const __nv_bfloat16* dy;  // OUT_DGRAD: gradient of the activation's output [M, N], row stride lddy
  int64_t lddy;
  float* y32;               // OUT_ACC32: fp32 accumulator [M, N], row stride ldy
};

// What the epilogue writes:
//   OUT_BF16  : y = act(rstd (x Wf^T) - rstd mean c + d) in bf16 (the layer's forward);
//   OUT_DGRAD : y = dy * act'(x Wf^T + d) in bf16 (no norm: the TiledLinear recompute of a chunk's
//               pre-activation with its gradient applied; the pre-activation is never stored);
//   OUT_ACC32 : y32 += x Wf^T in fp32 (no norm, no bias, no activation: a weight gradient summed
//               over token chunks).
enum NlOut { OUT_BF16 = 0, OUT_DGRAD = 1, OUT_ACC32 = 2 };

// The 32 columns col0.. of row m of the epilogue's output from the 32 accumulator values v:
// o = the corrected pre-activation (OUT_BF16: already activated).
// OUT_DGRAD: o <- dy[m, col0 ..] * act'(o) for the 32 columns (0 past N; row m < M)
template <int EPI>
__device__ __forceinline__ void nl_dgrad32(const NlArgs& a, int m, int col0, float (&o)[32]) {
  const __nv_bfloat16* g = a.dy + (int64_t)m * a.lddy + col0;
  if (col0 + 32 <= a.N) {
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
      float f8[8];
      Vec<__nv_bfloat16>::unpack(ld_stream(g + i), f8);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[i + e] = f8[e] * epi_grad<EPI, true>(o[i + e]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] = col0 + i < a.N ? __bfloat162float(g[i]) * epi_grad<EPI, true>(o[i]) : 0.0f;
  }
}

template <int OUT, int EPI>
__device__ __forceinline__ void nl_store32(const NlArgs& a, int m, int col0, const float (&o)[32]) {
  const bool whole = col0 + 32 <= a.N;
  if constexpr (OUT == OUT_ACC32) {
    float* row = a.y32 + (int64_t)m * a.ldy + col0;
    if (whole) {
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float4 t = *reinterpret_cast<const float4*>(row + i);
        t.x += o[i], t.y += o[i + 1], t.z += o[i + 2], t.w += o[i + 3];
        *reinterpret_cast<float4*>(row + i) = t;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (col0 + i < a.N) row[i] += o[i];
    }
  } else {
    float r[32];
    if constexpr (OUT == OUT_DGRAD) {
      const __nv_bfloat16* g = a.dy + (int64_t)m * a.lddy + col0;
      if (whole) {
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          float f8[8];
          Vec<__nv_bfloat16>::unpack(ld_stream(g + i), f8);
#pragma unroll
          for (int e = 0; e < 8; ++e) r[i + e] = f8[e] * epi_grad<EPI, true>(o[i + e]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          r[i] = col0 + i < a.N ? __bfloat162float(g[i]) * epi_grad<EPI, true>(o[i]) : 0.0f;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = o[i];
    }
    __nv_bfloat16* yrow = a.y + (int64_t)m * a.ldy;
    if (whole) {
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        const float f8[8] = {r[i], r[i + 1], r[i + 2], r[i + 3], r[i + 4], r[i + 5], r[i + 6], r[i + 7]};
        st_stream(yrow + col0 + i, Vec<__nv_bfloat16>::pack(f8));
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (col0 + i < a.N) yrow[col0 + i] = __float2bfloat16_rn(r[i]);
    }
  }
}

// ---------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// bring a tile into L2 ahead of its load (no shared memory involved)
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T for one M=128, N=256, K=16 step
template <int MAJ>
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc_f16(kUM, kBN, MAJ)), "r"(accumulate)
      : "memory");
}

// arrive once on `bar` when every tcgen05.mma this thread issued before has completed
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// Shared-memory matrix descriptor of a K-major tile of kLine-byte rows in the matching swizzle
// layout (the one TMA writes): start address >> 4 (bits 0-13), leading-dimension offset 16 B
// (encoded 1, bits 16-29; unused by these layouts), stride between 8-row groups 8 * kLine bytes
// (bits 32-45, in 16-byte units), descriptor version 1 (bits 46-47), layout (bits 61-63):
// SWIZZLE_128B = 2, SWIZZLE_64B = 4. Tiles start on 1024-byte boundaries (base offset 0).
__device__ __forceinline__ uint64_t tile_desc(const void* tile) {
  constexpr uint64_t layout = kLine == 128 ? 2 : 4;
  return (uint64_t)((smem_addr(tile) & 0x3FFFFu) >> 4) | (1ull << 16) | ((uint64_t)(8 * kLine / 16) << 32) |
         (1ull << 46) | (layout << 61);
}

// MN-major tiles (kBK = 64 only): the tile is a row of TMA boxes, each 64 M/N elements (128 bytes,
// the swizzle span) wide and kBK k-rows deep, 128-byte swizzled. Descriptor: the next 64 M/N
// elements one box further (leading-dimension offset = box bytes), the next 8 k-rows one 1024-byte
// swizzle atom further (stride offset), SWIZZLE_128B. One K=16 instruction step is 16 k-rows =
// 2048 bytes down the tile.
constexpr uint32_t kMnBox = 64 * kLine;  // bytes of one 64 x kBK box
__device__ __forceinline__ uint64_t tile_desc_mn(const void* tile) {
  return (uint64_t)((smem_addr(tile) & 0x3FFFFu) >> 4) | ((uint64_t)(kMnBox >> 4) << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
// descriptor units (16 bytes) between consecutive K=16 steps of a K-major / MN-major tile
template <bool MN>
constexpr uint64_t ksub_step() {
  return MN ? 2048 / 16 : 32 / 16;
}

// one stage's tile of an operand: a K-major tile is one box of `rows` x kBK; an MN-major tile is
// rows / 64 boxes of 64 x kBK at consecutive kMnBox offsets (coordinates: M/N first, then K)
template <bool MN>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, int k0, int r0, int rows, uint64_t* bar) {
  if constexpr (MN) {
    for (int i = 0; i < rows / 64; ++i) tma_load_2d(dst + i * kMnBox, map, r0 + 64 * i, k0, bar);
  } else {
    tma_load_2d(dst, map, k0, r0, bar);
  }
}

template <bool MN>
__device__ __forceinline__ void prefetch_tile(const CUtensorMap* map, int k0, int r0, int rows) {
  if constexpr (MN) {
    for (int i = 0; i < rows / 64; ++i) tma_prefetch_2d(map, r0 + 64 * i, k0);
  } else {
    tma_prefetch_2d(map, k0, r0);
  }
}

// 16-byte chunk c of row r sits at chunk position c ^ swz(r) of the row: the swizzle XORs
// address bits 4.. with bits 7.. of the offset inside the tile
__device__ __forceinline__ uint32_t swz(int r) {
  return kLine == 128 ? (uint32_t)(r & 7) : (uint32_t)((r >> 1) & 3);
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void mbar_arrive1(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// the epilogue's activation: the tanh-GeLU of gn_common; SiLU with the approximate divide
// (relative error ~1e-7, far below the bf16 rounding of the output)
template <int EPI>
__device__ __forceinline__ float nl_act(float z) {
  if constexpr (EPI == EPI_SILU)
    return __fdividef(z, 1.0f + __expf(-z));
  else
    return epi_fwd<EPI, true>(z);
}

// ---------------------------------------------------------------- forward kernel

template <int MH, int NORM, int EPI, int OUT = OUT_BF16, int MAJ = 0>
__global__ void __launch_bounds__(Tile<MH>::Threads, 1)
    norm_linear_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const NlArgs a) {
  using TL = Tile<MH>;
  constexpr bool AMN = (MAJ & MAJ_A_MN) != 0, BMN = (MAJ & MAJ_B_MN) != 0;
  static_assert(MAJ == 0 || (NORM == GN_NORM_NONE && kLine == 128), "MN-major operands: no norm, 64-wide k tiles");
  constexpr int kStages = TL::Stages;
  constexpr int kPrefetch = 2 * kStages;
  constexpr uint32_t kABytes = TL::ABytes, kStageBytes = TL::StageBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  float* col_c = reinterpret_cast<float*>(smem + kStages * kStageBytes + 256);  // c, d of the tile's columns
  float* col_d = col_c + kBN;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kBN, m0 = blockIdx.y * TL::BM;
  const int nk = (a.K + kBK - 1) / kBK;
  auto A = [&](int s) { return smem + s * kStageBytes; };
  auto B = [&](int s) { return smem + s * kStageBytes + kABytes; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NORM == GN_NORM_NONE ? 1 : 1 + 4 * MH);  // the MMA commit and the statistics warps
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tslot, TL::TmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t lastph = 0, used = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
        if (kb >= kStages && !mbar_wait(&empty[s], ph ^ 1u, a.err)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        mbar_expect_tx(&full[s], kStageBytes);
        // x is read from DRAM once per row block (the other column tiles hit in L2, W stays in
        // L2): fetch it into L2 a ring of stages ahead so the loads wait for L2, not DRAM
        if (kb + kPrefetch < nk) prefetch_tile<AMN>(&tmA, (kb + kPrefetch) * kBK, m0, TL::BM);
        load_tile<AMN>(A(s), &tmA, kb * kBK, m0, TL::BM, &full[s]);
        load_tile<BMN>(B(s), &tmB, kb * kBK, n0, kBN, &full[s]);
        used |= 1u << s;
        lastph = (lastph & ~(1u << s)) | (ph << s);
      }
      // every copy issued has landed before the CTA may exit
      for (int s = 0; s < kStages; ++s)
        if (used & (1u << s)) (void)mbar_wait(&full[s], (lastph >> s) & 1u, a.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
        if (!mbar_wait(&full[s], ph, a.err) || *abort_flag) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint64_t ad = AMN ? tile_desc_mn(A(s)) : tile_desc(A(s));
        const uint64_t bd = BMN ? tile_desc_mn(B(s)) : tile_desc(B(s));
#pragma unroll
        for (int k = 0; k < kBK / kUK; ++k)  // K-major: +32 bytes inside the swizzled rows
#pragma unroll
          for (int h = 0; h < MH; ++h)  // rows 128h.. of the A tile start 128 * kLine bytes further
            umma_bf16<MAJ>(tmem + (uint32_t)(kAccCols * h), ad + ksub_step<AMN>() * k + (uint64_t)(8 * kLine * h),
                           bd + ksub_step<BMN>() * k, (kb | k) != 0);
        umma_commit(&empty[s]);
      }
      umma_commit(accf);  // also after an abort: the epilogue waits for the work in flight
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ statistics + epilogue
    const int q = warp & 3;          // tensor-memory lane quadrant this warp may read
    const int h = (warp - 2) >> 2;   // accumulator (row half) of this warp
    const int r = kUM * h + 32 * q + lane;  // row of the tile
    const uint32_t sw = swz(r);  // 16-byte chunk permutation of this row
    // Row statistics over the streamed tiles. LayerNorm: each k-tile's mean and centred sum of
    // squares (two passes over the 64 register-resident values), merged into the running
    // (count, mean, M2) with Chan's update - two-pass accuracy in one sweep. RMSNorm: sum of
    // squares, one partial per k-tile added to the running total.
    // the tile's column terms, staged once (zero past N); read back after the mainloop
    for (int i = threadIdx.x - 64; i < kBN; i += 128 * MH) {
      const int n = n0 + i;
      col_c[i] = (NORM == GN_NORM_LN && n < a.N) ? a.c[n] : 0.0f;
      col_d[i] = (a.d && n < a.N) ? a.d[n] : 0.0f;
    }
    asm volatile("bar.sync 1, %0;" ::"r"(128 * MH) : "memory");  // the statistics warps only
    float cnt = 0.0f, mean = 0.0f, m2 = 0.0f;
    bool ok = true;
    for (int kb = 0; kb < (NORM == GN_NORM_NONE ? 0 : nk); ++kb) {  // no statistics without a norm
      const int s = kb % kStages;
      const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
      ok = __all_sync(0xffffffffu, mbar_wait(&full[s], ph, a.err)) && !*abort_flag;
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      // reading the row's chunks in logical order (position c ^ swz(r)) spreads the rows that
      // share a bank group over all 32 banks
      const uint8_t* line = A(s) + r * kLine;
      uint4 u[kChunks];
#pragma unroll
      for (int c = 0; c < kChunks; ++c) u[c] = *reinterpret_cast<const uint4*>(line + (((uint32_t)c ^ sw) << 4));
      const int kleft = a.K - kb * kBK;  // valid elements of this row in the tile
      const bool whole = kleft >= kBK;
      auto pair = [&](int c, int i) {  // element pair i of logical chunk c, invalid -> 0
        const uint32_t w = i == 0 ? u[c].x : i == 1 ? u[c].y : i == 2 ? u[c].z : u[c].w;
        float2 v = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
        if (!whole) {
          const int valid = kleft - 8 * c;
          v.x = 2 * i < valid ? v.x : 0.0f;
          v.y = 2 * i + 1 < valid ? v.y : 0.0f;
        }
        return v;
      };
      // every loaded value is consumed before the stage is released (the next TMA write into
      // this stage must not overtake a load still in flight)
      float2 t = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 v = pair(c, i);
          t = NORM == GN_NORM_LN ? add2(t, v) : fma2(v, v, t);
        }
      __syncwarp();
      if (lane == 0) mbar_arrive1(&empty[s]);
      if (NORM == GN_NORM_LN) {
        const float nb = whole ? (float)kBK : (float)max(kleft, 0);
        const float bm = nb > 0.0f ? (t.x + t.y) / nb : 0.0f;
        const float2 nbm = dup2(-bm);
        float2 q2 = make_float2(0.0f, 0.0f);
        float qt = 0.0f;
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 dv = add2(pair(c, i), nbm);
            if (whole) {
              q2 = fma2(dv, dv, q2);
            } else {  // zero-filled elements past the row are not centred values: skip them
              const int valid = kleft - 8 * c;
              qt = 2 * i < valid ? fmaf(dv.x, dv.x, qt) : qt;
              qt = 2 * i + 1 < valid ? fmaf(dv.y, dv.y, qt) : qt;
            }
          }
        if (nb > 0.0f) {
          const float n = cnt + nb, dlt = bm - mean;
          mean = fmaf(dlt, nb / n, mean);
          m2 += q2.x + q2.y + qt + dlt * dlt * (cnt * nb / n);
          cnt = n;
        }
      } else {
        m2 += t.x + t.y;
      }
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(accf, 0, a.err));
    tc_fence_after();
    if (ok && !*abort_flag) {
      const float inv_k = 1.0f / (float)a.K;
      float mu = 0.0f, rs;
      if (NORM == GN_NORM_LN) {
        mu = mean;
        rs = rsqrtf(fmaf(m2, inv_k, a.eps));  // biased variance M2 / K
      } else if (NORM == GN_NORM_RMS) {
        rs = rsqrtf(fmaf(m2, inv_k, a.eps));
      } else {
        rs = 1.0f;  // plain linear layer
      }
      const float nsm = -rs * mu;
      const int m = m0 + r;
      for (int j = 0; j < kBN / 32; ++j) {
        const int col0 = n0 + 32 * j;
        if (col0 >= a.N) break;  // uniform over the warp
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(kAccCols * h + 32 * j), v);
        float o[32];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 c4 = *reinterpret_cast<const float4*>(col_c + 32 * j + i);
          const float4 d4 = *reinterpret_cast<const float4*>(col_d + 32 * j + i);
          o[i + 0] = fmaf(rs, v[i + 0], fmaf(nsm, c4.x, d4.x));
          o[i + 1] = fmaf(rs, v[i + 1], fmaf(nsm, c4.y, d4.y));
          o[i + 2] = fmaf(rs, v[i + 2], fmaf(nsm, c4.z, d4.z));
          o[i + 3] = fmaf(rs, v[i + 3], fmaf(nsm, c4.w, d4.w));
        }
        if constexpr (OUT == OUT_BF16)
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = nl_act<EPI>(o[i]);
        if (m < a.M) nl_store32<OUT, EPI>(a, m, col0, o);
      }
      if (NORM != GN_NORM_NONE && blockIdx.x == 0 && m < a.M) {
        if (a.mean) a.mean[m] = mu;
        if (a.rstd) a.rstd[m] = rs;
      }
    }
  }

  // teardown: tensor memory is freed after every warp is done with it
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TL::TmemCols);
  }
}

// ---------------------------------------------------------------- pair-of-SMs forward kernel
// The same computation on a pair of CTAs on two SMs (a cluster of 2) that share each MMA: the
// leader CTA issues tcgen05.mma.cta_group::2 with M = 256 (rows 0-127 from its own shared memory,
// 128-255 from its peer's) and N = 256 (columns 0-127 of the B tile from the leader, 128-255
// from the peer), twice per k-step for a 256 x 512 pair tile. Each SM then loads 16 KiB of x and
// 32 KiB of W per 8.4 MFLOP (the single-SM 256 x 256 tile loads 64 KiB), and each SM's tensor
// memory holds its own 128 rows x 512 columns. Both CTAs' TMA loads count on the leader's `full`
// barrier; the MMA commits arrive on both CTAs' `empty` and accumulator barriers. The row
// statistics come from norm_stats_kernel, run just before: reading them from the x tiles here
// would need a signal from the leader to the peer on every stage, and a remote arrive on the
// pipeline's critical path cost more than the whole pre-pass (measured on B200).
constexpr int kPairN = 512;            // output columns of a pair tile
constexpr int kPairStages = 4;         // 48 KiB per stage and SM
constexpr uint32_t kPairABytes = kUM * kLine;           // 16 KiB: this CTA's 128 rows
constexpr uint32_t kPairBBytes = 2 * 128 * kLine;       // 32 KiB: this CTA's 2 x 128 B rows
constexpr uint32_t kPairStageBytes = kPairABytes + kPairBBytes;
constexpr int kPairThreads = 320;      // producer, MMA, 8 statistics/epilogue warps
constexpr size_t kPairSmem = 1024 + (size_t)kPairStages * kPairStageBytes + 256 + 2 * kPairN * 4;

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// TMA load into this CTA's shared memory whose completion counts on an mbarrier of either CTA
// of the pair (here: the leader's)
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int x, int y, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}

template <bool MN>
__device__ __forceinline__ void load_tile_pair(uint8_t* dst, const CUtensorMap* map, int k0, int r0, int rows,
                                               uint32_t bar_cluster) {
  if constexpr (MN) {
    for (int i = 0; i < rows / 64; ++i) tma_load_2d_pair(dst + i * kMnBox, map, r0 + 64 * i, k0, bar_cluster);
  } else {
    tma_load_2d_pair(dst, map, k0, r0, bar_cluster);
  }
}

// TMA store of a box from this CTA's shared memory (bulk-group completion), and the waits on this
// thread's bulk groups: until at most N remain reading shared memory
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(smem_addr(src))
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// TMA reduce: add a box of fp32 values from shared memory to the global tensor (done in L2)
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(smem_addr(src))
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {  // whole warp, both CTAs
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {  // whole warp, both CTAs
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// instruction shape of the pair: M = 256 (128 rows from each CTA), N = 256
template <int MAJ>
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc_f16(256, 256, MAJ)), "r"(accumulate)
      : "memory");
}

// arrive once on the barrier at this offset in both CTAs when the issued MMAs have completed
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_addr(bar)),
      "h"(mask)
      : "memory");
}

template <int NORM, int EPI, int OUT = OUT_BF16, int MAJ = 0>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    norm_linear_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmY, const NlArgs a) {
  constexpr bool AMN = (MAJ & MAJ_A_MN) != 0, BMN = (MAJ & MAJ_B_MN) != 0;
  static_assert(MAJ == 0 || (NORM == GN_NORM_NONE && kLine == 128), "MN-major operands: no norm, 64-wide k tiles");
  constexpr int kPrefetch = 2 * kPairStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tail = smem + kPairStages * kPairStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);   // leader: both CTAs' tiles landed
  uint64_t* empty = full + kPairStages;                   // the pair's MMAs done with the stage
  uint64_t* accf = empty + kPairStages;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  float* col_c = reinterpret_cast<float*>(tail + 256);
  float* col_d = col_c + kPairN;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int n0 = (blockIdx.x >> 1) * kPairN;         // the pair's first output column
  const int m0 = blockIdx.y * 256 + kUM * (int)rank;  // this CTA's first row
  const int nk = (a.K + kBK - 1) / kBK;
  auto A = [&](int s) { return smem + s * kPairStageBytes; };
  auto B = [&](int s) { return smem + s * kPairStageBytes + kPairABytes; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc_pair(tslot, 512);
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before any load counts on them
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      uint32_t lastph = 0, used = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kPairStages;
        const uint32_t ph = (uint32_t)(kb / kPairStages) & 1u;
        if (kb >= kPairStages && !mbar_wait(&empty[s], ph ^ 1u, a.err)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        const uint32_t bar = cluster_addr(&full[s], 0);
        if (leader) mbar_expect_tx(&full[s], 2 * kPairStageBytes);  // both CTAs' bytes
        if (kb + kPrefetch < nk) prefetch_tile<AMN>(&tmA, (kb + kPrefetch) * kBK, m0, kUM);
        load_tile_pair<AMN>(A(s), &tmA, kb * kBK, m0, kUM, bar);
        load_tile_pair<BMN>(B(s), &tmB, kb * kBK, n0 + 128 * (int)rank, 128, bar);
        load_tile_pair<BMN>(B(s) + 128 * kLine, &tmB, kb * kBK, n0 + 256 + 128 * (int)rank, 128, bar);
        used |= 1u << s;
        lastph = (lastph & ~(1u << s)) | (ph << s);
      }
      // the leader's barriers count both CTAs' copies: every copy issued has landed once they
      // complete (bounded waits)
      if (leader)
        for (int s = 0; s < kPairStages; ++s)
          if (used & (1u << s)) (void)mbar_wait(&full[s], (lastph >> s) & 1u, a.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kPairStages;
        const uint32_t ph = (uint32_t)(kb / kPairStages) & 1u;
        if (!mbar_wait(&full[s], ph, a.err) || *abort_flag) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint64_t ad = AMN ? tile_desc_mn(A(s)) : tile_desc(A(s));
        const uint64_t bd = BMN ? tile_desc_mn(B(s)) : tile_desc(B(s));
#pragma unroll
        for (int k = 0; k < kBK / kUK; ++k)
#pragma unroll
          for (int j = 0; j < 2; ++j)  // B rows 128j.. of each CTA's tile: columns 256j.. of the pair
            umma_bf16_pair<MAJ>(tmem + (uint32_t)(kAccCols * j), ad + ksub_step<AMN>() * k,
                                bd + ksub_step<BMN>() * k + (uint64_t)(8 * kLine * j), (kb | k) != 0);
        umma_commit_pair(&empty[s]);
      }
      umma_commit_pair(accf);  // also after an abort: both epilogues wait for the work in flight
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;          // tensor-memory lane quadrant
    const int j = (warp - 2) >> 2;   // accumulator (512 columns = 2 x 256) this warp drains
    const int r = 32 * q + lane;     // row of this CTA's 128
    const int m = m0 + r;
    for (int i = threadIdx.x - 64; i < kPairN; i += 256) {
      const int n = n0 + i;
      col_c[i] = (NORM == GN_NORM_LN && n < a.N) ? a.c[n] : 0.0f;
      col_d[i] = (a.d && n < a.N) ? a.d[n] : 0.0f;
    }
    const float mu = (NORM == GN_NORM_LN && m < a.M) ? __ldg(a.mean + m) : 0.0f;
    const float rs = NORM == GN_NORM_NONE ? 1.0f : m < a.M ? __ldg(a.rstd + m) : 0.0f;
    asm volatile("bar.sync 1, 256;" ::: "memory");  // column terms in place
    const bool ok = __all_sync(0xffffffffu, mbar_wait(accf, 0, a.err)) && !*abort_flag;
    tc_fence_after();
    if (ok) {
      const float nsm = -rs * mu;
      // bf16 outputs (y, or dz of OUT_DGRAD) leave through shared memory and TMA stores: each
      // warp turns 64 columns of its 32 rows into one 32 x 128-byte box (128-byte swizzle:
      // 16-byte chunk c of row r at position c ^ (r % 8)), two boxes in flight per warp, written
      // to y with the rows and columns past M and N clipped by the store. The pipeline stages
      // are free once every MMA has completed (accf), so the boxes reuse them. Measured (B200):
      // the fused LayerNorm + linear + SiLU 1.291 -> 1.258 ms, a dx chunk product 0.191 -> 0.180
      // ms against one 16-byte store per thread and row.
      uint8_t* box = smem + (size_t)(warp - 2) * 2 * 4096;
      for (int cb = 0; cb < 256 / 32; ++cb) {
        const int lc = 256 * j + 32 * cb;  // column of the pair tile
        const int col0 = n0 + lc;
        if (col0 >= a.N) break;  // uniform over the warp
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(kAccCols * j + 32 * cb), v);
        float o[32];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 c4 = *reinterpret_cast<const float4*>(col_c + lc + i);
          const float4 d4 = *reinterpret_cast<const float4*>(col_d + lc + i);
          o[i + 0] = fmaf(rs, v[i + 0], fmaf(nsm, c4.x, d4.x));
          o[i + 1] = fmaf(rs, v[i + 1], fmaf(nsm, c4.y, d4.y));
          o[i + 2] = fmaf(rs, v[i + 2], fmaf(nsm, c4.z, d4.z));
          o[i + 3] = fmaf(rs, v[i + 3], fmaf(nsm, c4.w, d4.w));
        }
        if constexpr (OUT != OUT_ACC32) {
          if constexpr (OUT == OUT_BF16) {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = nl_act<EPI>(o[i]);
          } else if (m < a.M) {  // OUT_DGRAD: the gradient applied (rows past M are clipped anyway)
            nl_dgrad32<EPI>(a, m, col0, o);
          }
          uint8_t* bx = box + (size_t)((cb >> 1) & 1) * 4096;
          if ((cb & 1) == 0 && cb >= 4) {  // this box's previous store has finished reading it
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
          }
          uint8_t* row = bx + lane * 128;
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            const float f8[8] = {o[i], o[i + 1], o[i + 2], o[i + 3], o[i + 4], o[i + 5], o[i + 6], o[i + 7]};
            const int c = (cb & 1) * 4 + i / 8;  // 16-byte chunk of the 128-byte box row
            *reinterpret_cast<uint4*>(row + ((c ^ (lane & 7)) << 4)) = Vec<__nv_bfloat16>::pack(f8);
          }
          if ((cb & 1) == 1 || col0 + 32 >= a.N) {  // the box is complete (or the row ends in it)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) tma_store_2d(&tmY, bx, n0 + 256 * j + 64 * (cb >> 1), m0 + 32 * q);
          }
        } else {
          // fp32 accumulator (OUT_ACC32): one 32-column box per chunk, added to y32 by a TMA
          // reduce in L2, so the epilogue never waits for the old values (each element gets one
          // addition per launch, in stream order: deterministic). Measured (B200): a TiledLinear
          // dW chunk product 0.244 -> 0.185 ms against the threads' own read-add-write.
          uint8_t* bx = box + (size_t)(cb & 1) * 4096;
          if (cb >= 2) {  // this box's previous reduce has finished reading it
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
          }
          uint8_t* row = bx + lane * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4*>(row + ((c ^ (lane & 7)) << 4)) =
                make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) tma_reduce_add_2d(&tmY, bx, col0, m0 + 32 * q);
        }
      }
      if (lane == 0) bulk_wait_read<0>();  // the boxes are read before the CTA may leave
      __syncwarp();
    }
  }

  // teardown: neither CTA leaves while the pair's MMAs may still touch its shared or tensor
  // memory; then both free the pair's tensor memory
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ---------------------------------------------------------------- row statistics pre-pass
// One warp per row of x [M, K] bf16: each lane folds its 16-byte vectors (lane, lane + 32, ...)
// into (count, mean, M2) - per vector a two-pass mean and centred sum of squares of the 8
// values, merged with Chan's update - then the lanes merge with xor shuffles (Chan's update
// again) so every lane holds the row's statistics. RMSNorm needs only the sum of squares.
// Writes mean (LayerNorm) and rstd = 1/sqrt(var + eps) (RMSNorm: 1/sqrt(mean(x^2) + eps)).
template <int NORM>
__global__ void __launch_bounds__(256) norm_stats_kernel(const __nv_bfloat16* __restrict__ x, int64_t ldx, int M, int K,
                                                          float eps, float* __restrict__ mean, float* __restrict__ rstd) {
  const int lane = threadIdx.x & 31;
  const int64_t m = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (m >= M) return;
  const __nv_bfloat16* row = x + m * ldx;
  const int nv = K / 8;  // whole 16-byte vectors (K is a multiple of 8)
  float cnt = 0.0f, mu = 0.0f, m2 = 0.0f;
#pragma unroll 4
  for (int v = lane; v < nv; v += 32) {
    const uint4 u = ld_stream(row + (int64_t)v * 8);
    float f[8];
    Vec<__nv_bfloat16>::unpack(u, f);
    if (NORM == GN_NORM_LN) {
      float t = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) t += f[e];
      const float bm = t * 0.125f;
      float q = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) q = fmaf(f[e] - bm, f[e] - bm, q);
      const float n = cnt + 8.0f, dlt = bm - mu;
      mu = fmaf(dlt, 8.0f / n, mu);
      m2 += q + dlt * dlt * (cnt * 8.0f / n);
      cnt = n;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) m2 = fmaf(f[e], f[e], m2);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float c2 = __shfl_xor_sync(0xffffffffu, cnt, o);
    const float mu2 = __shfl_xor_sync(0xffffffffu, mu, o);
    const float q2 = __shfl_xor_sync(0xffffffffu, m2, o);
    if (NORM == GN_NORM_LN) {
      const float n = cnt + c2;
      if (n > 0.0f) {
        const float dlt = mu2 - mu;
        m2 += q2 + dlt * dlt * (cnt * c2 / n);
        mu = fmaf(dlt, c2 / n, mu);
      }
      cnt = n;
    } else {
      m2 += q2;
    }
  }
  if (lane == 0) {
    if (NORM == GN_NORM_LN) mean[m] = mu;
    rstd[m] = rsqrtf(fmaf(m2, 1.0f / (float)K, eps));
  }
}

// ---------------------------------------------------------------- weight preparation
// One CTA per output feature n: Wf[n,k] = bf16(g'[k] W[n,k]); c[n] = sum_k Wf[n,k] (of the
// rounded values the GEMM multiplies); d[n] = sum_k beta[k] W[n,k] + bias[n]. The sums run in a
// fixed order (per-thread strided partials, then a fixed tree), so they are deterministic.
template <int NORM>
__global__ void __launch_bounds__(256) norm_linear_prepare_kernel(const __nv_bfloat16* __restrict__ W,
                                                                   const __nv_bfloat16* __restrict__ g,
                                                                   const __nv_bfloat16* __restrict__ beta,
                                                                   const __nv_bfloat16* __restrict__ bias,
                                                                   __nv_bfloat16* __restrict__ Wf, float* __restrict__ c,
                                                                   float* __restrict__ d, int K, int gemma) {
  __shared__ float red[2][256];
  const int n = blockIdx.x, t = threadIdx.x;
  const __nv_bfloat16* wrow = W + (int64_t)n * K;
  __nv_bfloat16* frow = Wf + (int64_t)n * K;
  float cs = 0.0f, ds = 0.0f;
  for (int k = t; k < K; k += 256) {
    const float w = __bfloat162float(wrow[k]);
    const float gk = NORM == GN_NORM_NONE ? 1.0f
                                          : (g ? __bfloat162float(g[k]) : 1.0f) + (NORM == GN_NORM_RMS && gemma ? 1.0f : 0.0f);
    const __nv_bfloat16 f = __float2bfloat16_rn(gk * w);
    frow[k] = f;
    cs += __bfloat162float(f);
    if (NORM == GN_NORM_LN && beta) ds = fmaf(__bfloat162float(beta[k]), w, ds);
  }
  red[0][t] = cs;
  red[1][t] = ds;
  __syncthreads();
  for (int h = 128; h > 0; h >>= 1) {
    if (t < h) {
      red[0][t] += red[0][t + h];
      red[1][t] += red[1][t + h];
    }
    __syncthreads();
  }
  if (t == 0) {
    if (c) c[n] = red[0][0];
    if (d) d[n] = red[1][0] + (bias ? __bfloat162float(bias[n]) : 0.0f);
  }
}

// ---------------------------------------------------------------- host side

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static std::once_flag once;
  static EncodeTiled fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  });
  return fn;
}

// 2-D bf16 tensor map of rows x cols (row stride ld elements), box box_rows x 64 columns,
// 128-byte swizzle; reads outside the tensor return zeros
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld, uint32_t box_rows) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, kLine == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map of the pair kernel's epilogue stores: rows x cols (row stride ld elements) of bf16
// (f32 false) or fp32, boxes of 128 bytes (64 bf16 or 32 fp32 columns) x 32 rows, 128-byte swizzle
bool make_out_map(CUtensorMap* map, void* base, int64_t rows, int64_t cols, int64_t ld, bool f32) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  const size_t es = f32 ? 4 : 2;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld * es)};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / es), 32u};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The kernel instances, by launch shape: one CTA per tile (MH = 1 or 2 accumulators) or a pair.
template <int MH>
struct SingleKernels {
  static constexpr size_t kSmem = Tile<MH>::Smem;
  template <int NORM, int EPI, int OUT, int MAJ>
  static void* get() {
    return (void*)norm_linear_kernel<MH, NORM, EPI, OUT, MAJ>;
  }
};
struct PairKernels {
  static constexpr size_t kSmem = kPairSmem;
  template <int NORM, int EPI, int OUT, int MAJ>
  static void* get() {
    return (void*)norm_linear_pair_kernel<NORM, EPI, OUT, MAJ>;
  }
};

// Built combinations: the layer's forward with every norm and activation (K-major operands);
// without a norm, the activation-gradient epilogue (K-major), and the plain bf16 product and the
// fp32-accumulating product in every operand layout. Others return null.
template <class KS, int MAJ>
void* pick_plain(int out) {
  return out == OUT_ACC32 ? KS::template get<GN_NORM_NONE, EPI_NONE, OUT_ACC32, MAJ>()
                          : KS::template get<GN_NORM_NONE, EPI_NONE, OUT_BF16, MAJ>();
}

template <class KS, int NORM>
void* pick_epi(int epi, int out, int maj) {
  if constexpr (NORM == GN_NORM_NONE) {
    if (maj != 0) {
      if (out == OUT_DGRAD || (out == OUT_BF16 && epi != GN_EPI_NONE)) return nullptr;
      return maj == 1 ? pick_plain<KS, 1>(out) : maj == 2 ? pick_plain<KS, 2>(out) : pick_plain<KS, 3>(out);
    }
    if (out == OUT_DGRAD) {
      if (epi == GN_EPI_GELU_TANH) return KS::template get<NORM, EPI_GELU_TANH, OUT_DGRAD, 0>();
      if (epi == GN_EPI_SILU) return KS::template get<NORM, EPI_SILU, OUT_DGRAD, 0>();
      return KS::template get<NORM, EPI_NONE, OUT_DGRAD, 0>();
    }
    if (out == OUT_ACC32) return KS::template get<NORM, EPI_NONE, OUT_ACC32, 0>();
  } else if (out != OUT_BF16 || maj != 0) {
    return nullptr;
  }
  if (epi == GN_EPI_GELU_TANH) return KS::template get<NORM, EPI_GELU_TANH, OUT_BF16, 0>();
  if (epi == GN_EPI_SILU) return KS::template get<NORM, EPI_SILU, OUT_BF16, 0>();
  return KS::template get<NORM, EPI_NONE, OUT_BF16, 0>();
}

template <class KS>
void* pick(int norm, int epi, int out, int maj) {
  return norm == GN_NORM_LN    ? pick_epi<KS, GN_NORM_LN>(epi, out, maj)
         : norm == GN_NORM_RMS ? pick_epi<KS, GN_NORM_RMS>(epi, out, maj)
                               : pick_epi<KS, GN_NORM_NONE>(epi, out, maj);
}

template <class KS>
bool set_smem_attr() {
  for (int norm = 0; norm < 3; ++norm)
    for (int epi = 0; epi < 3; ++epi)
      for (int out = 0; out < 3; ++out)
        for (int maj = 0; maj < 4; ++maj) {
          void* k = pick<KS>(norm, epi, out, maj);
          if (k && cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KS::kSmem) != cudaSuccess)
            return false;
        }
  return true;
}

#ifndef GN_NL_MH
#define GN_NL_MH 2
#endif
#ifndef GN_NL_PAIR
#define GN_NL_PAIR 1
#endif

// The launch shared by the forward and the TiledLinear backward products: y (bf16, OUT_BF16 and
// OUT_DGRAD) or y32 (fp32, OUT_ACC32) [M, N] from x and Wf: x [M, K] (K-major) or [K, M] (MN-major,
// maj bit 0), row stride ldx; Wf [N, K] or [K, N] (maj bit 1), row stride ldw. Arguments validated
// by the caller.
gn_status nl_run(const void* x, int64_t ldx, const void* Wf, int64_t ldw, const float* c, const float* d, void* y,
                 float* y32, int64_t ldy, const void* dy, int64_t lddy, float* mean, float* rstd, int64_t M,
                 int64_t N, int64_t K, float eps, int norm, int epi, int out, int maj, cudaStream_t stream) {
  // pairs of SMs sharing 256 x 512 tiles once there are more than 128 rows and 256 columns;
  // one SM per 256 x 256 tile (two accumulators) for fewer columns; 128 x 256 for few rows
  const bool pair = GN_NL_PAIR && M > kUM && N > kBN;
  const int mh = M > kUM ? GN_NL_MH : 1;
  const int bm = pair ? 2 * kUM : kUM * mh;
  // an MN-major operand is read as boxes of 64 M/N elements x 64 k-rows of the [K, M/N] matrix
  CUtensorMap ta, tb;
  const bool amn = (maj & MAJ_A_MN) != 0, bmn = (maj & MAJ_B_MN) != 0;
  if (!(amn ? make_map(&ta, x, K, M, ldx, 64u) : make_map(&ta, x, M, K, ldx, pair ? (uint32_t)kUM : (uint32_t)bm)) ||
      !(bmn ? make_map(&tb, Wf, K, N, ldw, 64u) : make_map(&tb, Wf, N, K, ldw, pair ? 128u : (uint32_t)kBN)))
    return GN_ERR_CUDA;
  void* kern = pair      ? pick<PairKernels>(norm, epi, out, maj)
               : mh == 2 ? pick<SingleKernels<2>>(norm, epi, out, maj)
                         : pick<SingleKernels<1>>(norm, epi, out, maj);
  if (!kern) return GN_ERR_UNSUPPORTED;
  // the dynamic shared-memory limits are attributes of the kernels on the current device: set
  // them once per device (0 = not yet, 1 = set, -1 = failed)
  static std::mutex attr_mu;
  static signed char attr_state[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GN_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lk(attr_mu);
    if (!attr_state[dev])
      attr_state[dev] =
          set_smem_attr<SingleKernels<1>>() && set_smem_attr<SingleKernels<2>>() && set_smem_attr<PairKernels>() ? 1 : -1;
    if (attr_state[dev] < 0) return GN_ERR_CUDA;
  }
  NlArgs a{};
  a.c = c, a.d = d;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.y32 = y32;
  a.dy = static_cast<const __nv_bfloat16*>(dy);
  a.lddy = lddy;
  a.mean = mean, a.rstd = rstd;
  a.M = (int)M, a.N = (int)N, a.K = (int)K;
  a.ldy = ldy;
  a.eps = eps;
  a.err = device_err_word();
  if (!a.err) return GN_ERR_CUDA;
  if (pair && norm != GN_NORM_NONE) {  // the pair kernel reads the row statistics: compute them first
    const unsigned sblocks = (unsigned)((M + 7) / 8);
    if (norm == GN_NORM_LN)
      norm_stats_kernel<GN_NORM_LN><<<sblocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), ldx, (int)M,
                                                                 (int)K, eps, mean, rstd);
    else
      norm_stats_kernel<GN_NORM_RMS><<<sblocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), ldx, (int)M,
                                                                  (int)K, eps, mean, rstd);
    count_launches(1);
    if (launch_status() != GN_OK) return GN_ERR_CUDA;
  }
  const dim3 grid(pair ? (unsigned)(2 * ((N + kPairN - 1) / kPairN)) : (unsigned)((N + kBN - 1) / kBN),
                  (unsigned)((M + bm - 1) / bm));
  // the pair kernel writes its outputs through TMA: a map of y (bf16) or y32 (fp32, added to) [M, N]
  CUtensorMap ty = ta;
  if (pair && !make_out_map(&ty, out == OUT_ACC32 ? (void*)y32 : y, M, N, ldy, out == OUT_ACC32)) return GN_ERR_CUDA;
  void* args_pair[] = {&ta, &tb, &ty, &a};
  void* args_one[] = {&ta, &tb, &a};
  void** args = pair ? args_pair : args_one;
  const int threads = pair ? kPairThreads : mh == 2 ? Tile<2>::Threads : Tile<1>::Threads;
  const size_t smem = pair ? kPairSmem : mh == 2 ? Tile<2>::Smem : Tile<1>::Smem;
  if (cudaLaunchKernel(kern, grid, dim3(threads), args, smem, stream) != cudaSuccess) return GN_ERR_CUDA;
  count_launches(1);
  return launch_status();
}

// shape checks shared by the entry points: K (the contraction) and every row stride a multiple of
// 8 elements (16-byte rows for the tensor maps)
bool nl_shape_ok(int64_t M, int64_t N, int64_t K) {
  return M >= 0 && N >= 0 && K > 0 && K % 8 == 0 && M <= (int64_t)65535 * kUM && N <= INT32_MAX && K <= INT32_MAX;
}

}  // namespace
}  // namespace gn

using namespace gn;

extern "C" gn_status gn_norm_linear_prepare(const void* W, const void* g, const void* beta, const void* bias, void* Wf,
                                            float* c, float* d, int64_t N, int64_t K, gn_norm norm, int gemma,
                                            gn_dtype dt, void* stream) {
  if (dt != GN_BF16) return dt_ok(dt) ? GN_ERR_UNSUPPORTED : GN_ERR_DTYPE;
  if (norm != GN_NORM_RMS && norm != GN_NORM_LN && norm != GN_NORM_NONE) return GN_ERR_SHAPE;
  if (N < 0 || K <= 0 || K > INT32_MAX || N > INT32_MAX) return GN_ERR_SHAPE;
  if (N == 0) return GN_OK;
  if (!W || !Wf) return GN_ERR_NULL;
  if (norm == GN_NORM_LN && !c) return GN_ERR_NULL;
  cudaStream_t s = (cudaStream_t)stream;
  const auto* Wb = static_cast<const __nv_bfloat16*>(W);
  const auto* gb = static_cast<const __nv_bfloat16*>(g);
  const auto* bb = static_cast<const __nv_bfloat16*>(beta);
  const auto* cb = static_cast<const __nv_bfloat16*>(bias);
  auto* fb = static_cast<__nv_bfloat16*>(Wf);
  if (norm == GN_NORM_LN)
    norm_linear_prepare_kernel<GN_NORM_LN><<<(unsigned)N, 256, 0, s>>>(Wb, gb, bb, cb, fb, c, d, (int)K, 0);
  else if (norm == GN_NORM_NONE)
    norm_linear_prepare_kernel<GN_NORM_NONE><<<(unsigned)N, 256, 0, s>>>(Wb, nullptr, nullptr, cb, fb, c, d, (int)K, 0);
  else
    norm_linear_prepare_kernel<GN_NORM_RMS><<<(unsigned)N, 256, 0, s>>>(Wb, gb, nullptr, cb, fb, c, d, (int)K,
                                                                        gemma != 0);
  count_launches(1);
  return launch_status();
}

extern "C" gn_status gn_norm_linear_fwd(const void* x, const void* Wf, const float* c, const float* d, void* y,
                                        float* mean, float* rstd, int64_t M, int64_t N, int64_t K, int64_t ldx,
                                        int64_t ldy, float eps, gn_norm norm, gn_epilogue epi, gn_dtype dt,
                                        void* stream) {
  if (dt != GN_BF16) return dt_ok(dt) ? GN_ERR_UNSUPPORTED : GN_ERR_DTYPE;
  if (!epi_ok(epi)) return GN_ERR_DTYPE;
  if (norm != GN_NORM_RMS && norm != GN_NORM_LN && norm != GN_NORM_NONE) return GN_ERR_SHAPE;
  if (!nl_shape_ok(M, N, K) || ldx < K || ldy < N || ldx % 8 || ldy % 8) return GN_ERR_SHAPE;
  if (M == 0 || N == 0) return GN_OK;
  if (!x || !Wf || !y || (norm != GN_NORM_NONE && !rstd) || (norm == GN_NORM_LN && (!c || !mean))) return GN_ERR_NULL;
  if (!aligned16(x) || !aligned16(Wf) || !aligned16(y) || (c && !aligned16(c)) || (d && !aligned16(d)))
    return GN_ERR_ALIGN;
  return nl_run(x, ldx, Wf, K, c, d, y, nullptr, ldy, nullptr, 0, mean, rstd, M, N, K, eps, norm, epi, OUT_BF16, 0,
                (cudaStream_t)stream);
}

extern "C" gn_status gn_linear_act_grad(const void* x, const void* Wf, const float* d, const void* dy, void* dz,
                                        int64_t M, int64_t N, int64_t K, int64_t ldx, int64_t lddy, int64_t lddz,
                                        gn_epilogue epi, gn_dtype dt, void* stream) {
  if (dt != GN_BF16) return dt_ok(dt) ? GN_ERR_UNSUPPORTED : GN_ERR_DTYPE;
  if (!epi_ok(epi)) return GN_ERR_DTYPE;
  if (!nl_shape_ok(M, N, K) || ldx < K || lddy < N || lddz < N || ldx % 8 || lddy % 8 || lddz % 8)
    return GN_ERR_SHAPE;
  if (M == 0 || N == 0) return GN_OK;
  if (!x || !Wf || !dy || !dz) return GN_ERR_NULL;
  if (!aligned16(x) || !aligned16(Wf) || !aligned16(dy) || !aligned16(dz) || (d && !aligned16(d))) return GN_ERR_ALIGN;
  return nl_run(x, ldx, Wf, K, nullptr, d, dz, nullptr, lddz, dy, lddy, nullptr, nullptr, M, N, K, 0.0f, GN_NORM_NONE,
                epi, OUT_DGRAD, 0, (cudaStream_t)stream);
}

namespace {
// operand checks of the plain products: a K-major operand [rows, K] needs K contiguous and a
// multiple of 8 (16-byte rows); an MN-major one [K, rows] needs its rows within the stride.
// Returns the layout bits for nl_run, or -1.
int plain_layouts(int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb, gn_layout al, gn_layout bl) {
  if ((al != GN_K_MAJOR && al != GN_MN_MAJOR) || (bl != GN_K_MAJOR && bl != GN_MN_MAJOR)) return -1;
  if (M < 0 || N < 0 || K <= 0 || M > (int64_t)65535 * kUM || N > INT32_MAX || K > INT32_MAX) return -1;
  if ((al == GN_K_MAJOR || bl == GN_K_MAJOR) && K % 8) return -1;
  if (lda % 8 || ldb % 8) return -1;
  if (lda < (al == GN_K_MAJOR ? K : M) || ldb < (bl == GN_K_MAJOR ? K : N)) return -1;
  return (al == GN_MN_MAJOR ? MAJ_A_MN : 0) | (bl == GN_MN_MAJOR ? MAJ_B_MN : 0);
}
}  // namespace

extern "C" gn_status gn_linear_bf16(const void* A, const void* B, const float* d, void* y, int64_t M, int64_t N,
                                    int64_t K, int64_t lda, int64_t ldb, int64_t ldy, gn_layout a_layout,
                                    gn_layout b_layout, gn_dtype dt, void* stream) {
  if (dt != GN_BF16) return dt_ok(dt) ? GN_ERR_UNSUPPORTED : GN_ERR_DTYPE;
  const int maj = plain_layouts(M, N, K, lda, ldb, a_layout, b_layout);
  if (maj < 0 || ldy < N || ldy % 8) return GN_ERR_SHAPE;
  if (M == 0 || N == 0) return GN_OK;
  if (!A || !B || !y) return GN_ERR_NULL;
  if (!aligned16(A) || !aligned16(B) || !aligned16(y) || (d && !aligned16(d))) return GN_ERR_ALIGN;
  return nl_run(A, lda, B, ldb, nullptr, d, y, nullptr, ldy, nullptr, 0, nullptr, nullptr, M, N, K, 0.0f, GN_NORM_NONE,
                GN_EPI_NONE, OUT_BF16, maj, (cudaStream_t)stream);
}

extern "C" gn_status gn_linear_acc_f32(const void* A, const void* B, float* C, int64_t M, int64_t N, int64_t K,
                                       int64_t lda, int64_t ldb, int64_t ldc, gn_layout a_layout, gn_layout b_layout,
                                       gn_dtype dt, void* stream) {
  if (dt != GN_BF16) return dt_ok(dt) ? GN_ERR_UNSUPPORTED : GN_ERR_DTYPE;
  const int maj = plain_layouts(M, N, K, lda, ldb, a_layout, b_layout);
  if (maj < 0 || ldc < N || ldc % 4) return GN_ERR_SHAPE;
  if (M == 0 || N == 0) return GN_OK;
  if (!A || !B || !C) return GN_ERR_NULL;
  if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return GN_ERR_ALIGN;
  return nl_run(A, lda, B, ldb, nullptr, nullptr, nullptr, C, ldc, nullptr, 0, nullptr, nullptr, M, N, K, 0.0f,
                GN_NORM_NONE, GN_EPI_NONE, OUT_ACC32, maj, (cudaStream_t)stream);
}
