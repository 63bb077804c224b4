// norm_plan.h - launch planning for the row-normalization kernels (host side).
//
// Two shapes, chosen by row length (few threads for short rows, a whole CTA for long rows,
// following the FlashNorm block-size rule of the Helios kernels article, section
// "内核一 FlashNorm"):
//   * group path (<= 128 16-byte vectors per row): `lanes` (a power of two <= 32) threads own
//     a row, hold it in registers and reduce with shuffles; 256-thread CTAs, grid-stride.
//   * CTA path: a persistent warp-specialised CTA (row_pipe.cuh): one producer warp stages
//     rows with TMA bulk copies, up to 10 consumer warps hold `vpt` vectors each of the row in
//     registers and reduce with shuffles plus one named barrier per row. Up to 1280 vectors
//     per row (10240 bf16 / 5120 fp32 elements) at 2 CTAs per SM, 2560 (forward only) at 1.
#pragma once

#include "gn_host.h"
#include "row_pipe.cuh"

namespace gn {

constexpr int kGroupThreads = 256;
constexpr int kGroupMaxVec = 128;      // group path up to 128 vectors per row (vpt <= 4 at 32 lanes)
constexpr int kNormMaxConsumers = 320;  // consumer threads of a CTA-path block
constexpr int kNormCtaThreads = 32 + kNormMaxConsumers;

// blocks per SM the CTA-path kernels are compiled for (register budget per thread): two
// while a thread's share of the row fits in about 90 registers
__host__ __device__ constexpr int norm_min_blocks(int vpt, bool bwd = false) { return vpt <= (bwd ? 2 : 4) ? 2 : 1; }

struct NormPlan {
  bool cta = false;
  int vpt = 1;
  int threads = 0;
  int lanes = 32;
  int stages = 0;
  size_t smem = 0;
};

inline int pow2_ceil(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

// ntens: row tensors staged per row (1 forward, 2 backward); nparams: per-column parameter
// vectors kept in shared memory (weight, bias), pes bytes per element (the row type's size, or 4
// for fp32 copies); max_vpt: 8 forward, 4 backward; target: preferred consumer threads (the
// forward keeps more of the row per thread, which spreads the per-row reduction over more
// elements).
inline gn_status plan_norm(int64_t N, size_t es, int ntens, int nparams, int max_vpt, int target, NormPlan* p,
                           size_t pes = 0) {
  if (!pes) pes = es;
  const int vec = (int)(16 / es);
  const int64_t nvec = (N + vec - 1) / vec;
  if (nvec <= kGroupMaxVec) {
    p->cta = false;
    p->lanes = pow2_ceil((int)nvec) < 32 ? pow2_ceil((int)nvec) : 32;
    p->vpt = (int)((nvec + p->lanes - 1) / p->lanes);
    if (p->vpt == 3) p->vpt = 4;
    p->threads = kGroupThreads;
    // backward: per-group dw (and db) partials are combined in shared memory
    p->smem = ntens > 1 ? (size_t)(kGroupThreads / p->lanes) * (size_t)(p->vpt * p->lanes * vec) * 2 * 4 : 0;
    return GN_OK;
  }
  p->cta = true;
  int vpt = g_tune.vpt;
  if (vpt == 0) {
    vpt = 1;
    while (vpt < max_vpt && (nvec + vpt - 1) / vpt > target) vpt <<= 1;
  }
  if (vpt > max_vpt) return GN_ERR_UNSUPPORTED;
  const int64_t consumers = ((nvec + vpt - 1) / vpt + 31) / 32 * 32;
  if (consumers > kNormMaxConsumers) return GN_ERR_UNSUPPORTED;
  p->vpt = vpt;
  p->threads = (int)consumers + 32;
  const int64_t row_bytes = N * (int64_t)es;
  const size_t slot = pipe_slot_bytes(row_bytes);
  int stages = g_tune.stages;
  if (stages == 0) {
    // forward: shallow pipelines leave room for more CTAs per SM, which hides the per-row
    // reduction latency better; backward: ~40 KiB in flight per CTA (2 stages of x and dy at
    // hidden 5120 bf16; 3 or 4 were 1-2 % slower). Measured on B200.
    stages = (int)((ntens > 1 ? 40960 : 24576) / (slot * ntens));
    stages = stages < 2 ? 2 : stages > kMaxStages ? kMaxStages : stages;
  }
  if (stages > kMaxStages) stages = kMaxStages;
  const size_t limit = smem_optin();
  while (stages > 1 && pipe_smem_bytes(stages, ntens, nparams, N, (int64_t)es, (int64_t)pes) > limit) --stages;
  if (pipe_smem_bytes(stages, ntens, nparams, N, (int64_t)es, (int64_t)pes) > limit) return GN_ERR_UNSUPPORTED;
  p->stages = stages;
  p->smem = pipe_smem_bytes(stages, ntens, nparams, N, (int64_t)es, (int64_t)pes);
  return GN_OK;
}

// Forward of long rows with one warp per row (norm_fwd_warp.cu): RMSNorm (ln = false: stat0 =
// inv_rms) or LayerNorm (ln = true: stat0 = mean, stat1 = rstd, b = bias). Arguments validated by
// the caller. GN_ERR_UNSUPPORTED when the row does not fit its shared-memory stages (the caller
// then uses the CTA-per-row kernel).
gn_status launch_norm_fwd_warp(bool ln, const void* x, const void* w, const void* b, void* y, float* stat0,
                               float* stat1, int64_t rows, int64_t N, int64_t ldx, int64_t ldy, float eps, bool gemma,
                               int epi, gn_dtype dt, cudaStream_t stream);

}  // namespace gn
