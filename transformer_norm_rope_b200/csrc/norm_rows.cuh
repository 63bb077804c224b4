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

// fp32 parameter vectors in shared memory are stored in planes of 16-byte chunks: chunk c
// (elements 4c .. 4c+3) of row vector v sits at float4 index c * nvec + v. Lanes that read
// consecutive vectors then read consecutive 16-byte words (no bank conflict), where a plain
// row-major copy of a bf16 row's 32-byte fp32 vectors would put lanes 32 bytes apart.

// the H element pairs of vector v of such a parameter vector
template <int H>
__device__ __forceinline__ void prm_pairs(const float* p, int v, int nvec, float2 (&f)[H]) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < H / 2; ++i) {
    const float4 t = q[i * nvec + v];
    f[2 * i] = make_float2(t.x, t.y);
    f[2 * i + 1] = make_float2(t.z, t.w);
  }
}

// dst[i] = (src[i] + add) * scale for i < N (src == null: dflt for src[i]), 0 for N <= i < nvec * E,
// in the chunk-plane layout above.
// All threads of the CTA take part. An aligned src is read one 16-byte vector at a time with four
// loads in flight per thread (an element-strided copy pays one L2 round trip per element); a
// ragged tail or an unaligned src goes element by element.
template <typename T>
__device__ __forceinline__ void stage_fp32(float* dst, const T* src, int N, int nvec, float add, float scale,
                                           float dflt) {
  using V = Vec<T>;
  constexpr int E = V::N;
  const int nfull = (src && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) ? N / E : 0;
  const int nt = (int)blockDim.x;
  for (int v0 = (int)threadIdx.x; v0 < nvec; v0 += 4 * nt) {
    uint4 raw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int v = v0 + j * nt;
      raw[j] = v < nfull ? __ldg(reinterpret_cast<const uint4*>(src) + v) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int v = v0 + j * nt;
      if (v >= nvec) break;
      float f[E];
      if (v < nfull) {
        V::unpack(raw[j], f);
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) f[e] = v * E + e < N ? ld_param(src, v * E + e, dflt) : 0.0f;
      }
#pragma unroll
      for (int e = 0; e < E; e += 4) {
        float4 o;
        o.x = v * E + e < N ? (f[e] + add) * scale : 0.0f;
        o.y = v * E + e + 1 < N ? (f[e + 1] + add) * scale : 0.0f;
        o.z = v * E + e + 2 < N ? (f[e + 2] + add) * scale : 0.0f;
        o.w = v * E + e + 3 < N ? (f[e + 3] + add) * scale : 0.0f;
        reinterpret_cast<float4*>(dst)[(e / 4) * nvec + v] = o;
      }
    }
  }
}

// Per-column parameters copied once into shared memory as fp32 in the chunk-plane layout above,
// (src + add) * scale per element (src == null: dflt), zero past N. Consumer thread ct writes vectors ct + j * nct (j < VPT), the
// vectors it reads back; the 16-byte loads of an aligned src are all issued before the first is
// used; a ragged tail or an unaligned src goes element by element.
template <typename T, int VPT>
__device__ __forceinline__ void stage_param_f32(float* dst, const T* src, int N, int nvec, float add, float scale,
                                                float dflt, int ct, int nct) {
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
      for (int e = 0; e < E; e += 4) {
        float4 o;
        o.x = v * E + e < N ? (f[e] + add) * scale : 0.0f;
        o.y = v * E + e + 1 < N ? (f[e + 1] + add) * scale : 0.0f;
        o.z = v * E + e + 2 < N ? (f[e + 2] + add) * scale : 0.0f;
        o.w = v * E + e + 3 < N ? (f[e + 3] + add) * scale : 0.0f;
        reinterpret_cast<float4*>(dst)[(e / 4) * nvec + v] = o;
      }
    }
  }
}

// dst vector v (16 bytes, the row type) = src vector v * scale (a power of two: exact), src == null
// giving dflt, zero past N. All threads of the CTA take part, one 16-byte load each per vector of
// an aligned src (element by element for a ragged tail or an unaligned src).
template <typename T>
__device__ __forceinline__ void stage_rowtype(uint8_t* dst, const T* src, int N, int nvec, float scale, float dflt) {
  using V = Vec<T>;
  constexpr int E = V::N;
  const int nfull = (src && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) ? N / E : 0;
  for (int v = (int)threadIdx.x; v < nvec; v += (int)blockDim.x) {
    float f[E];
    if (v < nfull) {
      V::unpack(__ldg(reinterpret_cast<const uint4*>(src) + v), f);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) f[e] = v * E + e < N ? ld_param(src, v * E + e, dflt) : 0.0f;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) f[e] *= scale;
    *reinterpret_cast<uint4*>(dst + (size_t)v * 16) = V::pack(f);
  }
}

// the parameters of vector v as element pairs// the parameters of vector v as element pairs
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
