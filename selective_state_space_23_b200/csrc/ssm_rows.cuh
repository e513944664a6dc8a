// Row I/O helpers shared by the scan kernels: E consecutive io elements of one row held as
// 32-bit words, loaded with streaming 128-bit (or 64-bit) loads when aligned, stored back with
// round-to-nearest-even bf16 packing; the load_steps / store_steps forms address the row in scan
// order, which is the row's own order or (reverse scan) its mirror image.
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

// Element order of a row reversed in place (row k <- row E-1-k).
template <typename IO, int E>
__device__ __forceinline__ void reverse_row(Row<IO, E>& r) {
  constexpr int W = Row<IO, E>::kWords;
  uint32_t t[W];
#pragma unroll
  for (int i = 0; i < W; ++i) t[i] = r.w[W - 1 - i];
#pragma unroll
  for (int i = 0; i < W; ++i) r.w[i] = sizeof(IO) == 2 ? __byte_perm(t[i], 0u, 0x1032) : t[i];
}

// E consecutive steps [tau, tau + E) of one time row in scan order.  In reverse order (rev) the
// scan's step tau is stored at row index L-1-tau, so the E steps are the row's elements
// [L-tau-E, L-tau) read backwards.  Steps at or beyond nvalid read as zero.  VEC: the row
// segment is aligned as load_row requires and all E steps are valid.  REORDER = false leaves a
// reversed segment in row order (reverse_row later puts it in scan order), so that a prefetch
// does not wait for its data at the load.
// ts: the row's element stride (1 for rows along L; the channel count for a [batch][L][dim]
// layout); only the element paths (VEC = false) take a stride other than 1.
template <typename IO, int E, bool VEC, bool REORDER = true>
__device__ __forceinline__ void load_steps(Row<IO, E>& r, const IO* row, int L, int tau, int nvalid,
                                           bool rev, long long ts = 1) {
  if (VEC || ts == 1) {
    if (!rev) {
      load_row<IO, E, VEC>(r, row + tau, nvalid);
      return;
    }
    if (VEC) {
      load_row<IO, E, true>(r, row + ((long long)L - tau - E), E);
      if (REORDER) reverse_row(r);
      return;
    }
  }
  // element accesses: step tau + e (scan order) lives at row index i(e)
  r.zero();
#pragma unroll
  for (int e = 0; e < E; ++e) {
    // a mirrored segment kept in row order (REORDER = false) places scan step E-1-e in slot e
    const int sstep = (rev && !REORDER) ? E - 1 - e : e;
    if (sstep < nvalid) {
      const long long i = (rev ? (long long)L - 1 - tau - sstep : (long long)tau + sstep) * ts;
      if (sizeof(IO) == 4)
        r.w[e] = __ldcs(reinterpret_cast<const uint32_t*>(row) + i);
      else
        r.w[e >> 1] |= ((uint32_t)__ldcs(reinterpret_cast<const unsigned short*>(row) + i))
                       << (16 * (e & 1));
    }
  }
}

// Store E values of steps [tau, tau + E) (only the first nvalid) to a time row in scan order.
template <typename IO, int E, bool VEC>
__device__ __forceinline__ void store_steps(IO* row, const float (&o)[E], int L, int tau, int nvalid,
                                            bool rev, long long ts = 1) {
  if constexpr (VEC) {
    if (!rev) {
      store_row<IO, E, true>(row + tau, o, nvalid);
    } else {
      float rv[E];
#pragma unroll
      for (int e = 0; e < E; ++e) rv[e] = o[E - 1 - e];
      store_row<IO, E, true>(row + ((long long)L - tau - E), rv, E);
    }
  } else {
    if (!rev && ts == 1) {
      store_row<IO, E, false>(row + tau, o, nvalid);
      return;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if (e < nvalid) {
        const long long i = (rev ? (long long)L - 1 - tau - e : (long long)tau + e) * ts;
        if (sizeof(IO) == 4) reinterpret_cast<float*>(row)[i] = o[e];
        else reinterpret_cast<uint16_t*>(row)[i] = f32_to_bf16(o[e]);
      }
    }
  }
}

}  // namespace ssm
