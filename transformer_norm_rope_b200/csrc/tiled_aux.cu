// tiled_aux.cu - the memory-bound steps of the TiledLinear backward around its tensor-core
// products (Helios kernels article, section "内核三 TiledLinear": per chunk of tokens, recompute
// the pre-activation, then dx = dz W and dW += dz^T x, db += sum dz):
//   * gn_transpose: a bf16 matrix transposed (the weight gradient contracts over the tokens, so
//     its two operands are fed to the K-major tensor-core kernel as dz^T and x^T);
//   * gn_colsum_bf16: column sums of a bf16 matrix into fp32 (db), in a fixed order.
#include "gn_common.cuh"
#include "gn_host.h"

namespace gn {
namespace {

// 64 x 64 tile per CTA of 256 threads. Loads: thread t reads 16 elements (two 16-byte vectors)
// of row t / 4 of the tile, four threads per 128-byte row segment. The tile sits in shared memory
// as 32-bit words (two elements of a row), rows padded to 33 words. Stores: thread t writes 16
// elements of output row t / 4 (= input column), gathered from 16 input rows, as two 16-byte
// vectors. Columns are a multiple of 8 (whole vectors); a row count that is not is padded: the
// output rows are written up to the next multiple of 8 columns, with zeros past the input rows.
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const __nv_bfloat16* __restrict__ src,
                                                             __nv_bfloat16* __restrict__ dst, int64_t rows,
                                                             int64_t cols, int64_t lds, int64_t ldd) {
  __shared__ uint32_t tile[64][33];
  const int t = threadIdx.x;
  const int64_t r0 = (int64_t)blockIdx.y * 64, c0 = (int64_t)blockIdx.x * 64;
  {
    const int r = t >> 2, c = (t & 3) * 16;
    uint4 v[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
    if (r0 + r < rows) {
      const __nv_bfloat16* p = src + (r0 + r) * lds + c0 + c;
      if (c0 + c < cols) v[0] = ld_stream(p);
      if (c0 + c + 8 < cols) v[1] = ld_stream(p + 8);
    }
    const uint32_t w[8] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w};
#pragma unroll
    for (int i = 0; i < 8; ++i) tile[r][c / 2 + i] = w[i];
  }
  __syncthreads();
  const int oc = t >> 2, seg = (t & 3) * 16;  // output row oc (input column c0 + oc), input rows seg..
  if (c0 + oc >= cols) return;
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t a = tile[seg + 2 * i][oc >> 1], b = tile[seg + 2 * i + 1][oc >> 1];
    const uint32_t lo = (oc & 1) ? (a >> 16) : (a & 0xffffu);
    const uint32_t hi = (oc & 1) ? (b & 0xffff0000u) : (b << 16);
    w[i] = lo | hi;
  }
  __nv_bfloat16* q = dst + (c0 + oc) * ldd + r0 + seg;
  if (r0 + seg < rows) st_stream(q, make_uint4(w[0], w[1], w[2], w[3]));
  if (r0 + seg + 8 < rows) st_stream(q + 8, make_uint4(w[4], w[5], w[6], w[7]));  // zeros past rows
}

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

extern "C" gn_status gn_transpose(const void* src, void* dst, int64_t rows, int64_t cols, int64_t ld_src,
                                  int64_t ld_dst, gn_dtype dt, void* stream) {
  if (dt != GN_BF16) return dt_ok(dt) ? GN_ERR_UNSUPPORTED : GN_ERR_DTYPE;
  if (rows < 0 || cols < 0 || ld_src < cols || ld_dst < (rows + 7) / 8 * 8 || cols % 8 || ld_src % 8 || ld_dst % 8)
    return GN_ERR_SHAPE;
  if (rows == 0 || cols == 0) return GN_OK;
  if (!src || !dst) return GN_ERR_NULL;
  if (!aligned16(src) || !aligned16(dst)) return GN_ERR_ALIGN;
  if ((rows + 63) / 64 > 65535) return GN_ERR_SHAPE;
  if (!kernel_attrs((const void*)transpose_bf16_kernel, 0)) return GN_ERR_CUDA;
  const dim3 grid((unsigned)((cols + 63) / 64), (unsigned)((rows + 63) / 64));
  transpose_bf16_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(static_cast<const __nv_bfloat16*>(src),
                                                                static_cast<__nv_bfloat16*>(dst), rows, cols, ld_src,
                                                                ld_dst);
  count_launches(1);
  return launch_status();
}

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
