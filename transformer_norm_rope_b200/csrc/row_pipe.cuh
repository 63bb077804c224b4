// row_pipe.cuh - the multi-stage TMA row pipeline used by the one-CTA-per-row kernels.
//
// A persistent CTA walks the rows m = blockIdx.x + i * gridDim.x. Row i of the CTA lands in
// stage i % stages: one thread issues one 1-D bulk copy per input tensor (the row's whole
// 16-byte vectors; a ragged tail of fewer than 16 bytes is read directly from global memory
// by the thread that owns it) and every thread waits on the stage's mbarrier. Up to `stages`
// rows are in flight per CTA, which is what keeps HBM busy without holding the rows in
// registers while they travel.
//
// Shared memory layout (dynamic, 128-byte aligned):
//   [0, 128)             mbarriers, one per stage (stages <= 16)
//   [128, 128 + 1024)    reduction scratch: 2 row parities x 32 warps x float4
//   [1152, ...)          stages x ntens x slot bytes (slot = row bytes rounded up to 128)
#pragma once

#include "gn_common.cuh"

namespace gn {

constexpr int kMaxStages = 16;
constexpr uint32_t kPipeHeader = 128 + 2 * 32 * 16;

__host__ __device__ inline uint32_t pipe_slot_bytes(int64_t row_bytes) {
  return (uint32_t)((row_bytes + 127) / 128 * 128);
}

__host__ __device__ inline size_t pipe_smem_bytes(int stages, int ntens, int64_t row_bytes) {
  return kPipeHeader + (size_t)stages * ntens * pipe_slot_bytes(row_bytes);
}

struct RowPipe {
  uint64_t* bar;
  float4* red;      // [2][32]
  uint8_t* data;
  int stages;
  int ntens;
  uint32_t slot;    // bytes per (stage, tensor) slot
  uint32_t bulk;    // bytes bulk-copied per tensor (whole 16-byte vectors of the row)

  __device__ __forceinline__ RowPipe(uint8_t* smem, int stages_, int ntens_, int64_t row_bytes)
      : bar(reinterpret_cast<uint64_t*>(smem)),
        red(reinterpret_cast<float4*>(smem + 128)),
        data(smem + kPipeHeader),
        stages(stages_),
        ntens(ntens_),
        slot(pipe_slot_bytes(row_bytes)),
        bulk((uint32_t)(row_bytes / 16 * 16)) {}

  __device__ __forceinline__ const uint8_t* at(int s, int t) const {
    return data + ((size_t)s * ntens + t) * slot;
  }

  // thread 0, before the first __syncthreads of the kernel
  __device__ __forceinline__ void init() const {
    for (int s = 0; s < stages; ++s) mbar_init(&bar[s], 1);
    mbar_fence_init();
  }

  // thread 0: start the copies of one row into stage s (s0..s3 = row start of tensors 0..3;
  // only the first ntens are used)
  __device__ __forceinline__ void issue(int s, const void* s0, const void* s1 = nullptr,
                                        const void* s2 = nullptr, const void* s3 = nullptr) const {
    mbar_expect_tx(&bar[s], bulk * (uint32_t)ntens);
    bulk_g2s(const_cast<uint8_t*>(at(s, 0)), s0, bulk, &bar[s]);
    if (ntens > 1) bulk_g2s(const_cast<uint8_t*>(at(s, 1)), s1, bulk, &bar[s]);
    if (ntens > 2) bulk_g2s(const_cast<uint8_t*>(at(s, 2)), s2, bulk, &bar[s]);
    if (ntens > 3) bulk_g2s(const_cast<uint8_t*>(at(s, 3)), s3, bulk, &bar[s]);
  }

  // wait for the stage-s copy whose completion flips the barrier to phase parity `ph`
  __device__ __forceinline__ bool wait(int s, uint32_t ph, unsigned* err) const {
    return mbar_wait(&bar[s], ph, err);
  }

  // thread 0, after a failed wait for row m (stage s, parity ph) of a grid-stride walk with
  // stride `step` over `rows`: wait (bounded) for the copies still in flight, so that none
  // lands in shared memory after the CTA has exited.
  __device__ __forceinline__ void drain(int64_t m, int64_t step, int64_t rows, int s, uint32_t ph,
                                        unsigned* err) const {
    for (int k = 0; k < stages && m < rows; ++k, m += step) {
      (void)wait(s, ph, err);
      if (++s == stages) {
        s = 0;
        ph ^= 1u;
      }
    }
  }
};

}  // namespace gn
