// Row I/O helpers shared by the scan kernels: E consecutive io elements of one row held as
// 32-bit words, loaded with streaming 128-bit (or 64-bit) loads when aligned, stored back with
// round-to-nearest-even bf16 packing.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ssm_device.cuh"

namespace ssm {

// E consecutive elements of one row, held as 32-bit words.
template <typename IO, int E>
struct Row {
  static constexpr int kWords = E * (int)sizeof(IO) / 4;
  uint32_t w[kWords];
  __device__ __forceinline__ float get(int k) const {
    if (sizeof(IO) == 4) return __uint_as_float(w[k]);
    const uint32_t x = w[k >> 1];
    return (k & 1) ? bf16_hi(x) : bf16_lo(x);
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < kWords; ++i) w[i] = 0u;
  }
};

// Load E consecutive elements at p; elements at or beyond nvalid read as zero.  VEC: p is aligned
// to E*sizeof(IO) bytes (8, 16 or 32) and all E elements are in bounds.
template <typename IO, int E, bool VEC>
__device__ __forceinline__ void load_row(Row<IO, E>& r, const IO* p, int nvalid) {
  constexpr int B = E * (int)sizeof(IO);
  if (VEC) {
    if constexpr (B == 8) {
      const uint2 v = __ldcs(reinterpret_cast<const uint2*>(p));
      r.w[0] = v.x;
      r.w[1] = v.y;
    } else {
#pragma unroll
      for (int i = 0; i < B / 16; ++i) {
        const uint4 v = __ldcs(reinterpret_cast<const uint4*>(p) + i);
        r.w[4 * i] = v.x; r.w[4 * i + 1] = v.y; r.w[4 * i + 2] = v.z; r.w[4 * i + 3] = v.w;
      }
    }
  } else {
    r.zero();
    if (sizeof(IO) == 4) {
      const uint32_t* s = reinterpret_cast<const uint32_t*>(p);
#pragma unroll
      for (int e = 0; e < E; ++e)
        if (e < nvalid) r.w[e] = __ldcs(s + e);
    } else {
      const unsigned short* s = reinterpret_cast<const unsigned short*>(p);
#pragma unroll
      for (int e = 0; e < E; ++e)
        if (e < nvalid) r.w[e >> 1] |= ((uint32_t)__ldcs(s + e)) << (16 * (e & 1));
    }
  }
}

template <typename IO, int E, bool VEC>
__device__ __forceinline__ void store_row(IO* p, const float (&o)[E], int nvalid) {
  constexpr int B = E * (int)sizeof(IO);
  uint32_t w[B / 4];
  if (sizeof(IO) == 2) {
#pragma unroll
    for (int i = 0; i < E / 2; ++i) w[i] = pack_bf16x2(o[2 * i], o[2 * i + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < E; ++i) w[i] = __float_as_uint(o[i]);
  }
  if (VEC) {
    if constexpr (B == 8) {
      __stcs(reinterpret_cast<uint2*>(p), make_uint2(w[0], w[1]));
    } else {
#pragma unroll
      for (int i = 0; i < B / 16; ++i)
        __stcs(reinterpret_cast<uint4*>(p) + i, make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]));
    }
  } else if (sizeof(IO) == 2) {
    unsigned short* s = reinterpret_cast<unsigned short*>(p);
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (e < nvalid) s[e] = (unsigned short)(w[e >> 1] >> (16 * (e & 1)));
  } else {
    float* s = reinterpret_cast<float*>(p);
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (e < nvalid) s[e] = o[e];
  }
}

}  // namespace ssm
