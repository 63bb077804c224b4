// api.cu - runtime pieces of libgn shared by all entry points: status strings, the launch
// counter, the device error word, device property caches, the tuning knobs and the
// deterministic column reduction that finishes every weight gradient.
#include <atomic>
#include <cstring>
#include <mutex>

#include "gn_common.cuh"
#include "gn_host.h"

namespace gn {

Tuning g_tune = {0, 0, 0, 0, 0, 0, 0};

static std::atomic<uint64_t> g_launches{0};

void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

// One error word per device. Kernels receive its address as an argument.
__device__ unsigned g_device_error_word;

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned* g_err_ptr[kMaxDevices];
int g_sms[kMaxDevices];
size_t g_smem[kMaxDevices];

int current_device() {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
  return d;
}
}  // namespace

unsigned* device_err_word() {
  const int d = current_device();
  if (d < 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[d] = static_cast<unsigned*>(p);
  }
  return g_err_ptr[d];
}

int sm_count() {
  const int d = current_device();
  if (d < 0) return 0;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sms[d]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d) != cudaSuccess) return 0;
    g_sms[d] = v;
  }
  return g_sms[d];
}

size_t smem_optin() {
  const int d = current_device();
  if (d < 0) return 0;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_smem[d]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, d) != cudaSuccess) return 0;
    g_smem[d] = (size_t)v;
  }
  return g_smem[d];
}

gn_status launch_status() { return cudaGetLastError() == cudaSuccess ? GN_OK : GN_ERR_CUDA; }

// Every kernel of the library asks for the same L1 / shared-memory split (the most shared
// memory): an SM whose split differs from the next kernel's must be reconfigured between the two
// kernels, which costs the next launch several microseconds.
#ifndef GN_CARVEOUT
#define GN_CARVEOUT 100
#endif

bool kernel_attrs(const void* kernel, size_t smem) {
  const int d = current_device();
  if (d < 0) return false;
  struct Seen {
    const void* k;
    int d;
    size_t smem;
  };
  static std::mutex mu;
  static Seen seen[512];
  static int nseen = 0;
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < nseen; ++i)
    if (seen[i].k == kernel && seen[i].d == d && seen[i].smem >= smem) return true;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return false;
  if (GN_CARVEOUT >= 0 &&
      cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, GN_CARVEOUT) != cudaSuccess)
    return false;
  for (int i = 0; i < nseen; ++i)
    if (seen[i].k == kernel && seen[i].d == d) {
      seen[i].smem = smem;
      return true;
    }
  if (nseen < 512) seen[nseen++] = Seen{kernel, d, smem};
  return true;
}

int persistent_grid(const void* kernel, int threads, size_t smem, int cap) {
  const int sms = sm_count();
  if (sms <= 0) return 0;
  if (!kernel_attrs(kernel, smem)) return 0;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess) return 0;
  if (per_sm <= 0) return 0;
  if (cap > 0 && per_sm > cap) per_sm = cap;
  return per_sm * sms;
}

// ---------------------------------------------------------------- column reduction
// Block = 32 columns x 32 slices of the partial rows (1024 threads: a whole SM's worth of loads in
// flight, the partial rows being L2-resident right after the backward wrote them). Slice k sums
// rows g = k, k+32, ... in order, then the first warp adds the 32 slice sums in order: a fixed
// order for a given G, so the result is the same on every run.
constexpr int kColsumSlices = 32;

__global__ void __launch_bounds__(32 * kColsumSlices) colsum_kernel(const float* __restrict__ ws, int64_t G,
                                                                    int64_t ncols, int64_t split,
                                                                    float* __restrict__ out0,
                                                                    float* __restrict__ out1) {
  __shared__ float part[kColsumSlices][33];
  pdl_wait();  // the partial rows are complete: the backward grid before this one has finished
  const int cl = threadIdx.x & 31, sl = threadIdx.x >> 5;
  const int64_t c = (int64_t)blockIdx.x * 32 + cl;
  float acc = 0.f;
  if (c < ncols) {
#pragma unroll 4
    for (int64_t g = sl; g < G; g += kColsumSlices) acc += ws[g * ncols + c];
  }
  part[sl][cl] = acc;
  __syncthreads();
  if (sl == 0 && c < ncols) {
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < kColsumSlices; ++k) t += part[k][cl];
    if (c < split) {
      if (out0) out0[c] = t;
    } else if (out1) {
      out1[c - split] = t;
    }
  }
}

// Self-test of the bounded wait: one thread waits for a phase of an mbarrier that nothing
// will complete, gives up after limit_ns and records the timeout in the error word.
__global__ void wait_timeout_selftest_kernel(unsigned* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  mbar_fence_init();
  (void)mbar_wait(&bar, 0, err, limit_ns);  // phase 0 never completes: no arrival comes
}

gn_status launch_colsum(const float* ws, int64_t G, int64_t ncols, int64_t split, float* out0,
                        float* out1, cudaStream_t s) {
  if (!out0 && !out1) return GN_OK;
  const int64_t blocks = (ncols + 31) / 32;
  if (!kernel_attrs((const void*)colsum_kernel, 0)) return GN_ERR_CUDA;
  // launched with programmatic stream serialization: its launch overlaps the tail of the
  // backward grid before it, which it waits for on the device (pdl_wait)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(32 * kColsumSlices);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = GN_PDL;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, colsum_kernel, ws, G, ncols, split, out0, out1) != cudaSuccess) return GN_ERR_CUDA;
  count_launches(1);
  return launch_status();
}

}  // namespace gn

using namespace gn;

extern "C" const char* gn_status_string(gn_status s) {
  switch (s) {
    case GN_OK: return "GN_OK";
    case GN_ERR_NULL: return "GN_ERR_NULL: a required pointer is NULL";
    case GN_ERR_SHAPE: return "GN_ERR_SHAPE: invalid size, stride or sign";
    case GN_ERR_ALIGN: return "GN_ERR_ALIGN: pointer or row stride not 16-byte aligned";
    case GN_ERR_DTYPE: return "GN_ERR_DTYPE: unknown dtype or epilogue";
    case GN_ERR_WORKSPACE: return "GN_ERR_WORKSPACE: workspace missing or too small";
    case GN_ERR_UNSUPPORTED: return "GN_ERR_UNSUPPORTED: row does not fit the kernel";
    case GN_ERR_CUDA: return "GN_ERR_CUDA: CUDA runtime error";
  }
  return "unknown gn_status";
}

extern "C" uint64_t gn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

extern "C" gn_status gn_device_error(unsigned* word, int clear) {
  if (!word) return GN_ERR_NULL;
  unsigned* p = device_err_word();
  if (!p) return GN_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return GN_ERR_CUDA;
  if (cudaMemcpy(word, p, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess) return GN_ERR_CUDA;
  if (clear && cudaMemset(p, 0, sizeof(unsigned)) != cudaSuccess) return GN_ERR_CUDA;
  if (clear && cudaDeviceSynchronize() != cudaSuccess) return GN_ERR_CUDA;
  return GN_OK;
}

extern "C" gn_status gn_selftest_wait_timeout(uint32_t limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 1000000) return GN_ERR_SHAPE;
  unsigned* err = device_err_word();
  if (!err) return GN_ERR_CUDA;
  wait_timeout_selftest_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(err, (uint64_t)limit_us * 1000u);
  count_launches(1);
  return launch_status();
}

extern "C" gn_status gn_tune(const char* key, int value) {
  if (!key || value < 0) return GN_ERR_SHAPE;
  if (!strcmp(key, "stages")) {
    if (value > 16) return GN_ERR_SHAPE;
    g_tune.stages = value;
  } else if (!strcmp(key, "ctas_per_sm")) {
    g_tune.ctas_per_sm = value;
  } else if (!strcmp(key, "vpt")) {
    if (value != 0 && value != 1 && value != 2 && value != 4 && value != 8) return GN_ERR_SHAPE;
    g_tune.vpt = value;
  } else if (!strcmp(key, "unit_bytes")) {
    g_tune.unit_bytes = value;
  } else if (!strcmp(key, "group_rows")) {
    g_tune.group_rows = value;
  } else if (!strcmp(key, "fwd_warps")) {
    if (value > 20) return GN_ERR_SHAPE;
    g_tune.fwd_warps = value;
  } else if (!strcmp(key, "fwd_path")) {
    if (value > 3) return GN_ERR_SHAPE;
    g_tune.fwd_path = value;

  } else {
    return GN_ERR_SHAPE;
  }
  return GN_OK;
}
