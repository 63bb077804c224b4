// act.cu - the epilogue activation and its gradient, elementwise: y = act(z), dz = dy * act'(z).
//
// The backward of a linear layer with an activation (y = act(z), z = x W^T + b) needs dz before
// its two gradient products; gn_act_grad is that step for a caller that holds z (the token-chunked
// layer of the Helios kernels article, section "内核三 TiledLinear", never stores z: its
// recompute applies the same derivative in the tensor-core epilogue). gn_act_fwd applies the
// activation to a stored pre-activation, for the training form of the fused norm + linear layer
// that keeps z for its backward instead of recomputing it (Janus-Pro-7B article, section 4.1:
// SiLU after the first projection; "LLM层的优化算子", section "编写定制融合算子": tanh-GeLU). Both
// use the functions of the normalization kernels' epilogues (epi_fwd, epi_grad: the tanh-GeLU
// with the same constants, SiLU). 16-byte vectors per thread, grid-stride; a ragged tail of fewer
// than one vector is handled element by element.
#include "gn_common.cuh"
#include "gn_host.h"

namespace gn {
namespace {

// dz may alias z or dy (each element is read before it is written, by the same thread)
template <typename T, int EPI>
__global__ void __launch_bounds__(256) act_grad_kernel(const T* z, const T* dy, T* dz, int64_t n) {
  constexpr int E = Vec<T>::N;
  constexpr bool FAST = fast_math_for<T>();
  const int64_t nvec = n / E;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec; v += stride) {
    float fz[E], fg[E];
    Vec<T>::unpack(ld_stream(z + v * E), fz);
    Vec<T>::unpack(ld_stream(dy + v * E), fg);
#pragma unroll
    for (int e = 0; e < E; ++e) fg[e] *= epi_grad<EPI, FAST>(fz[e]);
    st_stream(dz + v * E, Vec<T>::pack(fg));
  }
  // the ragged tail, by the first threads of the grid
  const int64_t t = nvec * E + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t < n) Vec<T>::store1(dz + t, Vec<T>::load1(dy + t) * epi_grad<EPI, FAST>(Vec<T>::load1(z + t)));
}

// y may alias z (each element is read before it is written, by the same thread)
template <typename T, int EPI>
__global__ void __launch_bounds__(256) act_fwd_kernel(const T* z, T* y, int64_t n) {
  constexpr int E = Vec<T>::N;
  constexpr bool FAST = fast_math_for<T>();
  const int64_t nvec = n / E;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec; v += stride) {
    float f[E];
    Vec<T>::unpack(ld_stream(z + v * E), f);
#pragma unroll
    for (int e = 0; e < E; ++e) f[e] = epi_fwd<EPI, FAST>(f[e]);
    st_stream(y + v * E, Vec<T>::pack(f));
  }
  const int64_t t = nvec * E + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t < n) Vec<T>::store1(y + t, epi_fwd<EPI, FAST>(Vec<T>::load1(z + t)));
}

template <typename T>
void* pick_fwd(int epi) {
  if (epi == GN_EPI_GELU_TANH) return (void*)act_fwd_kernel<T, EPI_GELU_TANH>;
  if (epi == GN_EPI_SILU) return (void*)act_fwd_kernel<T, EPI_SILU>;
  return (void*)act_fwd_kernel<T, EPI_NONE>;
}

// blocks of 256 threads for n elements of dt: one 16-byte vector per thread, at most 8 blocks per SM
int64_t act_blocks(int64_t n, gn_dtype dt) {
  const int64_t nvec = n / (int64_t)(16 / dt_size(dt));
  int64_t blocks = (nvec + 255) / 256;
  const int64_t cap = (int64_t)(sm_count() > 0 ? sm_count() : 148) * 8;
  if (blocks > cap) blocks = cap;
  return blocks < 1 ? 1 : blocks;
}

template <typename T>
void* pick(int epi) {
  if (epi == GN_EPI_GELU_TANH) return (void*)act_grad_kernel<T, EPI_GELU_TANH>;
  if (epi == GN_EPI_SILU) return (void*)act_grad_kernel<T, EPI_SILU>;
  return (void*)act_grad_kernel<T, EPI_NONE>;
}

}  // namespace
}  // namespace gn

using namespace gn;

extern "C" gn_status gn_act_grad(const void* z, const void* dy, void* dz, int64_t n, gn_epilogue epi, gn_dtype dt,
                                 void* stream) {
  if (!dt_ok(dt) || !epi_ok(epi)) return GN_ERR_DTYPE;
  if (n < 0) return GN_ERR_SHAPE;
  if (n == 0) return GN_OK;
  if (!z || !dy || !dz) return GN_ERR_NULL;
  if (!aligned16(z) || !aligned16(dy) || !aligned16(dz)) return GN_ERR_ALIGN;
  void* kern = dt == GN_BF16 ? pick<__nv_bfloat16>(epi) : pick<float>(epi);
  const int64_t blocks = act_blocks(n, dt);
  void* args[] = {&z, &dy, &dz, &n};
  if (cudaLaunchKernel(kern, dim3((unsigned)blocks), dim3(256), args, 0, (cudaStream_t)stream) != cudaSuccess)
    return GN_ERR_CUDA;
  count_launches(1);
  return launch_status();
}

extern "C" gn_status gn_act_fwd(const void* z, void* y, int64_t n, gn_epilogue epi, gn_dtype dt, void* stream) {
  if (!dt_ok(dt) || !epi_ok(epi)) return GN_ERR_DTYPE;
  if (n < 0) return GN_ERR_SHAPE;
  if (n == 0) return GN_OK;
  if (!z || !y) return GN_ERR_NULL;
  if (!aligned16(z) || !aligned16(y)) return GN_ERR_ALIGN;
  void* kern = dt == GN_BF16 ? pick_fwd<__nv_bfloat16>(epi) : pick_fwd<float>(epi);
  const int64_t blocks = act_blocks(n, dt);
  void* args[] = {&z, &y, &n};
  if (cudaLaunchKernel(kern, dim3((unsigned)blocks), dim3(256), args, 0, (cudaStream_t)stream) != cudaSuccess)
    return GN_ERR_CUDA;
  count_launches(1);
  return launch_status();
}
