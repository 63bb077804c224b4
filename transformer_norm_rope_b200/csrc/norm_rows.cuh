// norm_rows.cuh - row I/O helpers of the one-CTA-per-row normalization kernels.
//
// A consumer thread of the row pipeline (row_pipe.cuh) owns whole 16-byte vectors of a row.
// Whole vectors come from the TMA stage in shared memory; the ragged tail of a row whose byte
// length is not a multiple of 16 is read and written element by element in global memory.
#pragma once

#include "gn_common.cuh"

namespace gn {

// per-column parameters (weight, bias) copied once into shared memory, padded with zeros
// (times `scale`, a power of two, so the stored values stay exact)
template <typename T>
__device__ __forceinline__ void stage_param(uint8_t* dst, const T* src, int N, int nvec, float dflt, int ct, int nct,
                                            float scale = 1.0f) {
  T* d = reinterpret_cast<T*>(dst);
  const int n = nvec * Vec<T>::N;
  for (int i = ct; i < n; i += nct) Vec<T>::store1(d + i, i < N ? scale * ld_param(src, i, dflt) : 0.0f);
}

// the parameters of vector v as element pairs
template <typename T>
__device__ __forceinline__ void param_pairs(const uint8_t* p, int v, float2 (&f)[Vec<T>::N / 2]) {
  unpack2<T>(*reinterpret_cast<const uint4*>(p + (size_t)v * 16), f);
}

template <typename T>
__device__ __forceinline__ void load_pairs(const uint8_t* st, const T* row, int v, int nfull, int N, bool ok,
                                           float2 (&f)[Vec<T>::N / 2]) {
  constexpr int E = Vec<T>::N;
  if (ok && v < nfull) {
    unpack2<T>(*reinterpret_cast<const uint4*>(st + (size_t)v * 16), f);
  } else {
#pragma unroll
    for (int h = 0; h < E / 2; ++h) {
      const int col = v * E + 2 * h;
      f[h].x = (ok && col < N) ? Vec<T>::load1(row + col) : 0.0f;
      f[h].y = (ok && col + 1 < N) ? Vec<T>::load1(row + col + 1) : 0.0f;
    }
  }
}

template <typename T>
__device__ __forceinline__ void store_pairs(T* row, int v, int nfull, int N, const float2 (&f)[Vec<T>::N / 2]) {
  constexpr int E = Vec<T>::N;
  if (v < nfull) {
    st_stream(row + (size_t)v * E, pack2<T>(f));
  } else {
#pragma unroll
    for (int h = 0; h < E / 2; ++h) {
      const int col = v * E + 2 * h;
      if (col < N) Vec<T>::store1(row + col, f[h].x);
      if (col + 1 < N) Vec<T>::store1(row + col + 1, f[h].y);
    }
  }
}

// vector v of a row as its 16 raw bytes: whole vectors straight from the stage, the ragged
// tail (and vectors past the row) packed from global memory, zero beyond the row
template <typename T>
__device__ __forceinline__ uint4 load_raw(const uint8_t* st, const T* row, int v, int nfull, int N, bool ok) {
  if (ok && v < nfull) return *reinterpret_cast<const uint4*>(st + (size_t)v * 16);
  float2 f[Vec<T>::N / 2];
  load_pairs<T>(st, row, v, nfull, N, ok, f);  // takes its element-wise branch here
  return pack2<T>(f);  // exact: the values came from T
}

}  // namespace gn
