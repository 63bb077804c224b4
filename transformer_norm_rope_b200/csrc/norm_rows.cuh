// norm_rows.cuh - row I/O helpers of the one-CTA-per-row normalization kernels.
//
// A consumer thread of the row pipeline (row_pipe.cuh) owns whole 16-byte vectors of a row.
// Whole vectors come from the TMA stage in shared memory; the ragged tail of a row whose byte
// length is not a multiple of 16 is read and written element by element in global memory.
#pragma once

#include "gn_common.cuh"

namespace gn {

// Per-column parameters (weight, bias) copied once into shared memory, padded with zeros,
// times `scale` (a power of two, so the stored values stay exact); `dflt` stands for a null
// src. Consumer thread ct writes vectors ct + j * nct (j < VPT), which covers the row. The
// whole 16-byte vectors of an aligned src are fetched with one load each, all of a thread's
// loads issued before the first is used: an element-strided loop paid one L2 round trip per
// element at the start of every CTA. A ragged tail or an unaligned src goes element by element.
template <typename T, int VPT>
__device__ __forceinline__ void stage_param(uint8_t* dst, const T* src, int N, int nvec, float dflt, int ct, int nct,
                                            float scale = 1.0f) {
  constexpr int E = Vec<T>::N;
  const int nfull = (src && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) ? N / E : 0;
  uint4 raw[VPT];
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int v = ct + j * nct;
    raw[j] = v < nfull ? __ldg(reinterpret_cast<const uint4*>(src) + v) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int v = ct + j * nct;
    if (v < nvec) {
      float f[E];
      if (v < nfull) {
        Vec<T>::unpack(raw[j], f);
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) f[e] = v * E + e < N ? ld_param(src, v * E + e, dflt) : 0.0f;
      }
#pragma unroll
      for (int e = 0; e < E; ++e) f[e] *= scale;
      *reinterpret_cast<uint4*>(dst + (size_t)v * 16) = Vec<T>::pack(f);
    }
  }
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
