// Streaming helpers shared by the kernels that read whole logit rows: the
// balanced split of a flattened (row, 16-byte vector) space over persistent
// warps, non-allocating 128-bit loads, element access on raw vectors (bf16
// and f32), and the warp-uniform running maximum.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "kld_common.cuh"

namespace kld {

// First flattened vector of warp w when `total` vectors are split evenly
// over `nwarps` warps.
__host__ __device__ __forceinline__ int64_t warp_begin(int64_t w, int64_t total, int nwarps) {
  return (total * w) / nwarps;
}

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Element access on raw 16-byte vectors.  bf16: a 32-bit word holds
// elements (2k, 2k+1) in its low and high halves, so a pair widens to f32
// with one shift and one mask.  f32: the vector is four elements.
template <bool kBF16>
struct Elems;

template <>
struct Elems<true> {
  static constexpr int E = 8;
  __device__ __forceinline__ static float2 pair(const uint4& v, int k) {
    const uint32_t w = k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
  __device__ __forceinline__ static float vmax(const uint4& v) {
    uint32_t a, b, m;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(a) : "r"(v.x), "r"(v.y));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(b) : "r"(v.z), "r"(v.w));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(a), "r"(b));
    return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u));
  }
  // Largest of the 16 elements of two vectors (NaN only if all are NaN,
  // as for vmax).
  __device__ __forceinline__ static float vmax2(const uint4& v, const uint4& w) {
    uint32_t a, b, c, d, e, f, m;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(a) : "r"(v.x), "r"(v.y));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(b) : "r"(v.z), "r"(v.w));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(c) : "r"(w.x), "r"(w.y));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(w.z), "r"(w.w));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(e) : "r"(a), "r"(b));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(f) : "r"(c), "r"(d));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(e), "r"(f));
    return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u));
  }
  __device__ __forceinline__ static float load1(const void* base, int64_t i) {
    const unsigned short b = reinterpret_cast<const unsigned short*>(base)[i];
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
  }
};

template <>
struct Elems<false> {
  static constexpr int E = 4;
  __device__ __forceinline__ static float2 pair(const uint4& v, int k) {
    return k == 0 ? make_float2(__uint_as_float(v.x), __uint_as_float(v.y))
                  : make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
  }
  __device__ __forceinline__ static float vmax(const uint4& v) {
    return fmaxf(fmaxf(__uint_as_float(v.x), __uint_as_float(v.y)),
                 fmaxf(__uint_as_float(v.z), __uint_as_float(v.w)));
  }
  __device__ __forceinline__ static float vmax2(const uint4& v, const uint4& w) {
    return fmaxf(vmax(v), vmax(w));
  }
  __device__ __forceinline__ static float load1(const void* base, int64_t i) {
    return reinterpret_cast<const float*>(base)[i];
  }
};

// Warp that owns flattened vector g (inverse of warp_begin).
__device__ __forceinline__ int warp_of(int64_t g, int64_t total, int nwarps) {
  int w = (int)((g * nwarps) / total);
  while (w + 1 < nwarps && warp_begin(w + 1, total, nwarps) <= g) ++w;
  while (w > 0 && warp_begin(w, total, nwarps) > g) --w;
  return w;
}

// Order-preserving map between floats and signed ints, so that a warp-wide
// float maximum is one redux.sync.max.s32.  A lane maximum is NaN only when
// all its elements are NaN; that row is invalid whatever maximum wins.
__device__ __forceinline__ int ordered_key(float f) {
  const int i = __float_as_int(f);
  return i ^ ((i >> 31) & 0x7fffffff);
}
__device__ __forceinline__ float key_value(int k) { return __int_as_float(k ^ ((k >> 31) & 0x7fffffff)); }

__device__ __forceinline__ float warp_max(float v) {
  return key_value(__reduce_max_sync(0xffffffffu, ordered_key(v)));
}

// Warp-uniform side state: the maximum m and its index a are the same in
// every lane; each lane keeps its own share r of sum_{i != a} exp(z_i - m).
struct WarpSide {
  float m;
  int a;
  float r;
};

// The exponent offset of a side: c = -m log2(e) rounded to f32 (0 before a
// finite value), so a weight is 2^(z log2(e) + c) from one fused
// multiply-add; c misses -m log2(e) by rho = -m log2(e) - c (exact, from a
// second fused multiply-add), so those weights are exp(z - m) 2^-rho, and
// sums formed with c are multiplied by fix = 2^rho when they join the row's.
// |rho| is at most half a unit in the last place of c, so the form needs a
// small |c|: below |m| = 2^20 it is under 1/16 and t = z log2(e) + c is as
// accurate as (z - m) log2(e); from 2^20 on it grows with |m| (2^-rho leaves
// the f32 range near |m| = 2^31, and z log2(e) overflows near 2^127).  A side
// with |m| >= 2^20 is therefore marked exact, and its weights are formed as
// (z - m) log2(e) in two operations (c = -m, fix = 1).
struct Offset {
  float c, fix;
  bool exact;
};

__device__ __forceinline__ Offset offset_of(const WarpSide& s) {
  if (s.a < 0) return Offset{0.f, 1.f, false};
  if (!(fabsf(s.m) < 0x1p20f)) return Offset{-s.m, 1.f, true};
  const float c = __fmul_rn(-s.m, kLog2e);
  const float rho = fmaf(-s.m, kLog2e, -c);
  return Offset{c, ex2(rho), false};
}

// The offsets of two sides, both in the exact form when either needs it.
__device__ __forceinline__ void offsets_of(const WarpSide& x, const WarpSide& y, Offset& ox, Offset& oy) {
  ox = offset_of(x);
  oy = offset_of(y);
  if (ox.exact || oy.exact) {
    ox = Offset{x.a < 0 ? 0.f : -x.m, 1.f, true};
    oy = Offset{y.a < 0 ? 0.f : -y.m, 1.f, true};
  }
}

}  // namespace kld
