// norm_plan.h - launch planning for the row-normalization kernels (host side).
//
// Two shapes, chosen by row length (one warp-sized lane group per row for short rows, one
// CTA per row for long rows, following the FlashNorm block-size rule of the Helios kernels
// article, section "内核一 FlashNorm": few threads for small rows, full blocks for large ones):
//   * group path (<= 128 16-byte vectors per row): `lanes` (a power of two <= 32) threads own
//     a row, hold it in registers and reduce with shuffles; 256-thread CTAs, grid-stride.
//   * CTA path: a persistent CTA owns one row at a time; rows arrive through the multi-stage
//     TMA pipeline (row_pipe.cuh); each thread holds `vpt` vectors of the row in registers,
//     and the row statistic is reduced with shuffles plus one CTA barrier.
#pragma once

#include "gn_host.h"
#include "row_pipe.cuh"

namespace gn {

constexpr int kGroupThreads = 256;
constexpr int kGroupMaxVec = 128;  // group path up to 128 vectors per row (vpt <= 4 at 32 lanes)

// most threads a CTA-path kernel instance may be launched with (its __launch_bounds__);
// backward kernels hold twice the row data per thread, so they stop at 512
__host__ __device__ constexpr int norm_max_threads(int vpt, bool bwd = false) {
  return vpt <= 1 ? (bwd ? 512 : 1024) : vpt == 2 ? 512 : 256;
}

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

// ntens: row tensors staged per row (1 forward, 2 backward). max_vpt: 8 forward, 4 backward.
inline gn_status plan_norm(int64_t N, size_t es, int ntens, int max_vpt, int default_threads,
                           NormPlan* p) {
  const bool bwd = ntens > 1;
  const int vec = (int)(16 / es);
  const int64_t nvec = (N + vec - 1) / vec;
  if (nvec <= kGroupMaxVec) {
    p->cta = false;
    p->lanes = pow2_ceil((int)nvec) < 32 ? pow2_ceil((int)nvec) : 32;
    p->vpt = (int)((nvec + p->lanes - 1) / p->lanes);
    if (p->vpt == 3) p->vpt = 4;
    p->threads = kGroupThreads;
    // backward: per-group dw partials are combined in shared memory
    p->smem = ntens > 1 ? (size_t)(kGroupThreads / p->lanes) * (size_t)(p->vpt * p->lanes * vec) * 2 * 4 : 0;
    return GN_OK;
  }
  p->cta = true;
  int vpt = g_tune.vpt;
  if (vpt == 0) {
    vpt = 1;
    while (vpt < max_vpt && (nvec + vpt - 1) / vpt > default_threads) vpt <<= 1;
  }
  if (vpt > max_vpt) return GN_ERR_UNSUPPORTED;
  int64_t threads = ((nvec + vpt - 1) / vpt + 31) / 32 * 32;
  while (threads > norm_max_threads(vpt, bwd) && vpt < max_vpt) {
    vpt <<= 1;
    threads = ((nvec + vpt - 1) / vpt + 31) / 32 * 32;
  }
  if (threads > norm_max_threads(vpt, bwd)) return GN_ERR_UNSUPPORTED;
  p->vpt = vpt;
  p->threads = (int)threads;
  const int64_t row_bytes = N * (int64_t)es;
  const size_t slot = pipe_slot_bytes(row_bytes);
  int stages = g_tune.stages;
  if (stages == 0) {
    stages = (int)(65536 / (slot * ntens));
    stages = stages < 2 ? 2 : stages > 8 ? 8 : stages;
  }
  const size_t limit = smem_optin();
  while (stages > 1 && pipe_smem_bytes(stages, ntens, row_bytes) > limit) --stages;
  if (pipe_smem_bytes(stages, ntens, row_bytes) > limit || row_bytes > 200 * 1024) return GN_ERR_UNSUPPORTED;
  p->stages = stages;
  p->smem = pipe_smem_bytes(stages, ntens, row_bytes);
  return GN_OK;
}

}  // namespace gn
