// row_pipe.cuh - the warp-specialised TMA row pipeline of the one-CTA-per-row kernels.
//
// A persistent CTA walks the rows m = blockIdx.x + i * gridDim.x. Warp 0 is the producer:
// one lane moves each row (each staged tensor's whole 16-byte vectors; a ragged tail of fewer
// than 16 bytes is read from global memory by the consumer that owns it) into stage
// i % stages with 1-D TMA bulk copies counted on the stage's `full` mbarrier, and waits on the
// stage's `empty` mbarrier before reusing it. The other warps are consumers: they wait on
// `full`, copy their vectors of the row into registers, and each warp arrives on `empty` at
// once, so the producer refills the stage while the consumers are still reducing the row.
// The row statistic is reduced with shuffles within warps and one named barrier over the
// consumer warps (the producer warp never joins it).
//
// Shared memory layout (dynamic, 128-byte aligned):
//   [0, 64)           full mbarriers, one per stage (stages <= 8)
//   [64, 128)         empty mbarriers
//   [128, 1152)       reduction scratch: 2 row parities x 4 quantities x 32 warps of float
//   [1152, ...)       nparams parameter vectors (weight, bias) of the row length, in the row type
//                     (forward) or as fp32 (backward)
//   then              stages x ntens row slots (row bytes rounded up to 128)
#pragma once

#include "gn_common.cuh"

namespace gn {

constexpr int kMaxStages = 8;
constexpr uint32_t kPipeHeader = 128 + 2 * 32 * 16;

__host__ __device__ inline uint32_t pipe_slot_bytes(int64_t row_bytes) {
  return (uint32_t)((row_bytes + 127) / 128 * 128);
}

// parameter vectors: one element of pes bytes (the row type's size, or 4 for fp32 copies) per
// row element, padded to whole 16-byte row vectors and to 128 bytes
__host__ __device__ inline uint32_t pipe_param_bytes(int64_t n, int64_t es, int64_t pes) {
  return pipe_slot_bytes((n * es + 15) / 16 * (16 / es) * pes);
}

__host__ __device__ inline size_t pipe_smem_bytes(int stages, int ntens, int nparams, int64_t n, int64_t es,
                                                  int64_t pes) {
  return kPipeHeader + (size_t)nparams * pipe_param_bytes(n, es, pes) + (size_t)stages * ntens * pipe_slot_bytes(n * es);
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Barrier 1 over the `n` consumer threads, returning the OR of `pred` over them.
__device__ __forceinline__ int consumers_sync_or(int n, int pred) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.s32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred), "r"(n)
      : "memory");
  return r;
}

__device__ __forceinline__ void consumers_sync(int n) { asm volatile("bar.sync 1, %0;" ::"r"(n) : "memory"); }

struct RowPipe {
  uint64_t* full;
  uint64_t* empty;
  float4* red;      // [2][32]
  uint8_t* params;  // nparams parameter vectors
  uint8_t* data;
  int stages;
  int ntens;
  uint32_t slot;    // bytes per (stage, tensor) slot
  uint32_t pslot;   // bytes per parameter vector
  uint32_t bulk;    // bytes bulk-copied per tensor (whole 16-byte vectors of the row)

  __device__ __forceinline__ RowPipe(uint8_t* smem, int stages_, int ntens_, int nparams, int64_t n, int64_t es,
                                     int64_t pes)
      : full(reinterpret_cast<uint64_t*>(smem)),
        empty(reinterpret_cast<uint64_t*>(smem) + kMaxStages),
        red(reinterpret_cast<float4*>(smem + 128)),
        params(smem + kPipeHeader),
        data(smem + kPipeHeader + (size_t)nparams * pipe_param_bytes(n, es, pes)),
        stages(stages_),
        ntens(ntens_),
        slot(pipe_slot_bytes(n * es)),
        pslot(pipe_param_bytes(n, es, pes)),
        bulk((uint32_t)(n * es / 16 * 16)) {}

  // Cross-warp partials of the per-row reductions, as float [2 row parities][4 quantities][32
  // warps]: warp w's partial of quantity q sits at index w, so a sum over the consumer warps reads
  // four partials per 16-byte load. Slots past the consumer warps stay zero (red_zero).
  __device__ __forceinline__ float* red_at(uint32_t rb, int q) const {
    return reinterpret_cast<float*>(red) + (rb * 4 + q) * 32;
  }
  __device__ __forceinline__ void red_zero(int ct, int nct) const {
    for (int i = ct; i < 256; i += nct) reinterpret_cast<float*>(red)[i] = 0.0f;
  }
  // the fixed-order sum of quantity q over the ncw consumer warps (same order in every thread)
  __device__ __forceinline__ float red_sum(uint32_t rb, int q, int ncw) const {
    const float4* p = reinterpret_cast<const float4*>(red_at(rb, q));
    float t = 0.0f;
    for (int i = 0; i < ((ncw + 3) >> 2); ++i) {
      const float4 v = p[i];
      t += (v.x + v.y) + (v.z + v.w);
    }
    return t;
  }

  __device__ __forceinline__ const uint8_t* at(int s, int t) const {
    return data + ((size_t)s * ntens + t) * slot;
  }
  __device__ __forceinline__ uint8_t* param(int i) const { return params + (size_t)i * pslot; }

  // thread 0, before the first __syncthreads of the kernel
  __device__ __forceinline__ void init(int consumer_warps) const {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], (uint32_t)consumer_warps);
    }
    mbar_fence_init();
  }

  // Producer lane: stage every row of this CTA's walk; src(m, t) is the start of row m of
  // staged tensor t. Returns after every copy it issued has landed (bounded waits).
  template <class Src>
  __device__ __forceinline__ void produce(int64_t rows, Src src, unsigned* err) const {
    const int64_t step = gridDim.x;
    int s = 0;
    uint32_t ph = 0, used = 0, lastph = 0;
    int64_t k = 0;
    for (int64_t m = blockIdx.x; m < rows; m += step, ++k) {
      if (k >= stages && !mbar_wait(&empty[s], ph ^ 1u, err)) break;
      mbar_expect_tx(&full[s], bulk * (uint32_t)ntens);
      for (int t = 0; t < ntens; ++t) bulk_g2s(const_cast<uint8_t*>(at(s, t)), src(m, t), bulk, &full[s]);
      used |= 1u << s;
      lastph = (lastph & ~(1u << s)) | (ph << s);
      if (++s == stages) s = 0, ph ^= 1u;
    }
    for (int t = 0; t < stages; ++t)
      if (used & (1u << t)) (void)mbar_wait(&full[t], (lastph >> t) & 1u, err);
  }
};

}  // namespace gn
