// tiled_aux.cu - the memory-bound step of the TiledLinear backward next to its tensor-core
// products (Helios kernels article, section "内核三 TiledLinear": per chunk of tokens, recompute
// the pre-activation, then dx = dz W and dW += dz^T x, db += sum dz): gn_colsum_bf16, the column
// sums of a bf16 matrix into fp32 (db), in a fixed order.
#include "gn_common.cuh"
#include "gn_host.h"

namespace gn {
namespace {

constexpr int kColsumSlices = 64;

// Stage 1: slice s of the rows (rows s*R .. (s+1)*R - 1, R = ceil(rows / slices)) summed per
// column into ws[s][c]: block = 64 columns x 8 warps; lane l owns columns 2l, 2l+1 of the block,
// warp w the rows w, w + 8, ... of the slice; the 8 warps' sums combined in warp order.
__global__ void __launch_bounds__(256) colsum_bf16_slices(const __nv_bfloat16* __restrict__ src, float* __restrict__ ws,
                                                          int64_t rows, int64_t cols, int64_t ld) {
  __shared__ float2 part[8][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t c = (int64_t)blockIdx.x * 64 + 2 * lane;
  const int64_t per = (rows + gridDim.y - 1) / gridDim.y;
  const int64_t rb = (int64_t)blockIdx.y * per, re = rb + per < rows ? rb + per : rows;
  float2 acc = make_float2(0.0f, 0.0f);
  if (c < cols)
    for (int64_t r = rb + warp; r < re; r += 8) {
      const uint32_t v = *reinterpret_cast<const uint32_t*>(src + r * ld + c);  // two bf16, c even
      acc.x += __uint_as_float(v << 16);
      acc.y += __uint_as_float(v & 0xffff0000u);
    }
  part[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && c < cols) {
    float2 s = part[0][lane];
#pragma unroll
    for (int w = 1; w < 8; ++w) s.x += part[w][lane].x, s.y += part[w][lane].y;
    ws[(int64_t)blockIdx.y * cols + c] = s.x;
    ws[(int64_t)blockIdx.y * cols + c + 1] = s.y;
  }
}

// Stage 2: out[c] (+)= sum over the slices in slice order.
__global__ void __launch_bounds__(256) colsum_bf16_final(const float* __restrict__ ws, float* __restrict__ out,
                                                         int64_t cols, int slices, int accumulate) {
  const int64_t c = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (c >= cols) return;
  float t = 0.0f;
  for (int s = 0; s < slices; ++s) t += ws[(int64_t)s * cols + c];
  out[c] = accumulate ? out[c] + t : t;
}

}  // namespace
}  // namespace gn

using namespace gn;

extern "C" size_t gn_colsum_bf16_workspace(int64_t cols) {
  return cols > 0 ? (size_t)kColsumSlices * (size_t)cols * sizeof(float) : 0;
}

extern "C" gn_status gn_colsum_bf16(const void* src, float* out, void* ws, size_t ws_bytes, int64_t rows, int64_t cols,
                                    int64_t ld, int accumulate, gn_dtype dt, void* stream) {
  if (dt != GN_BF16) return dt_ok(dt) ? GN_ERR_UNSUPPORTED : GN_ERR_DTYPE;
  if (rows < 0 || cols <= 0 || ld < cols || cols % 2 || ld % 2) return GN_ERR_SHAPE;
  cudaStream_t s = (cudaStream_t)stream;
  if (!out) return GN_ERR_NULL;
  if (rows == 0) {
    if (!accumulate && cudaMemsetAsync(out, 0, (size_t)cols * sizeof(float), s) != cudaSuccess) return GN_ERR_CUDA;
    return GN_OK;
  }
  if (!src) return GN_ERR_NULL;
  if (!ws) return GN_ERR_WORKSPACE;
  if (ws_bytes < gn_colsum_bf16_workspace(cols)) return GN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(src) & 3u) || !aligned16(ws)) return GN_ERR_ALIGN;
  if (!kernel_attrs((const void*)colsum_bf16_slices, 0) || !kernel_attrs((const void*)colsum_bf16_final, 0))
    return GN_ERR_CUDA;
  const dim3 g1((unsigned)((cols + 63) / 64), kColsumSlices);
  colsum_bf16_slices<<<g1, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(src), static_cast<float*>(ws), rows, cols,
                                       ld);
  colsum_bf16_final<<<(unsigned)((cols + 255) / 256), 256, 0, s>>>(static_cast<const float*>(ws), out, cols,
                                                                    kColsumSlices, accumulate);
  count_launches(2);
  return launch_status();
}
