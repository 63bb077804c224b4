// gn_host.h - host-side internals shared by the translation units of libgn.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gn.h"

namespace gn {

// Tuning knobs (0 = planner default); set through gn_tune().
struct Tuning {
  int stages;
  int ctas_per_sm;
  int vpt;
  int unit_bytes;
  int group_rows;
  int fwd_warps;  // warps per CTA of the one-warp-per-row forward
  int fwd_path;   // norm forward of long rows: 1 = CTA-per-row pipeline, 2 = one warp per row with
                  // two-pass LayerNorm statistics, 3 = one warp per row with one shifted pass
};
extern Tuning g_tune;

// Address of the device error word on the current device (nullptr if it cannot be had).
unsigned* device_err_word();

// Launch bookkeeping.
void count_launches(int n);

// Properties of the current device, cached per device.
int sm_count();
size_t smem_optin();

// cudaGetLastError -> status.
gn_status launch_status();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t dt_size(gn_dtype dt) { return dt == GN_BF16 ? 2 : 4; }
inline bool dt_ok(int dt) { return dt == GN_F32 || dt == GN_BF16; }
inline bool epi_ok(int e) { return e == GN_EPI_NONE || e == GN_EPI_GELU_TANH || e == GN_EPI_SILU; }

// Deterministic column reduction of per-block partials: out0[c] = sum_g ws[g*ncols + c] for
// c < split, out1[c - split] for c >= split (either output may be null to skip its part).
gn_status launch_colsum(const float* ws, int64_t G, int64_t ncols, int64_t split, float* out0,
                        float* out1, cudaStream_t s);

// Sets a kernel's launch attributes on the current device once (the dynamic shared-memory limit
// when smem exceeds 48 KiB, and the L1 / shared-memory split every kernel of the library shares).
bool kernel_attrs(const void* kernel, size_t smem);

// Largest grid of a persistent kernel: sm_count() * min(occupancy, cap).
int persistent_grid(const void* kernel, int threads, size_t smem, int cap);

}  // namespace gn
