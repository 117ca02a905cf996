// pa_common.cuh -- device helpers shared by the libpa kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pa.h"

namespace pa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------------------
// Element types.  Cache rows are moved as 16-byte vectors; each vector holds
// kPerVec elements and is widened to fp32 in registers.
// ---------------------------------------------------------------------------
template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int kBytes = 4;
  static constexpr int kPerVec = 4;
  __device__ __forceinline__ static void widen(const uint4 &v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static float load1(const void *p, int64_t i) {
    return static_cast<const float *>(p)[i];
  }
  __device__ __forceinline__ static void store1(void *p, int64_t i, float x) {
    static_cast<float *>(p)[i] = x;
  }
  // Elements i and i + 1 (i even, base 16-byte aligned).
  __device__ __forceinline__ static void store2(void *p, int64_t i, float a, float b) {
    *reinterpret_cast<float2 *>(static_cast<float *>(p) + i) = make_float2(a, b);
  }
  // Elements i .. i + 3 (i a multiple of 4, base 16-byte aligned).
  __device__ __forceinline__ static void store4(void *p, int64_t i, float4 v) {
    *reinterpret_cast<float4 *>(static_cast<float *>(p) + i) = v;
  }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kBytes = 2;
  static constexpr int kPerVec = 8;
  // bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits.
  __device__ __forceinline__ static void widen(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ static float load1(const void *p, int64_t i) {
    return __uint_as_float(
        static_cast<uint32_t>(static_cast<const uint16_t *>(p)[i]) << 16);
  }
  __device__ __forceinline__ static void store1(void *p, int64_t i, float x) {
    static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
  }
  // Elements i and i + 1 (i even, base 16-byte aligned), each rounded to
  // nearest even.
  __device__ __forceinline__ static void store2(void *p, int64_t i, float a, float b) {
    *reinterpret_cast<__nv_bfloat162 *>(static_cast<__nv_bfloat16 *>(p) + i) =
        __floats2bfloat162_rn(a, b);
  }
  // Elements i .. i + 3 (i a multiple of 4, base 16-byte aligned), rounded to
  // nearest even.
  __device__ __forceinline__ static void store4(void *p, int64_t i, float4 v) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t *>(&lo);
    u.y = *reinterpret_cast<const uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p) + i) = u;
  }
};

// Streaming 16-byte read of data that no kernel writes while it runs.
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void set_error(int32_t *err_word, int32_t bit) {
  if (err_word != nullptr) atomicOr(err_word, bit);
}

// ---------------------------------------------------------------------------
// Transposed butterfly reduction across the L lanes of an aligned lane group.
//
// Every lane holds N partial sums v[0..N).  After the call, with j the lane's
// index inside its group:
//   N >= L : v[0 .. N/L) hold the group-wide sums of indices
//            j*(N/L) .. j*(N/L) + N/L - 1;
//   N <  L : v[0] holds the group-wide sum of index j >> log2(L/N) (lanes
//            that differ only in their low log2(L/N) bits hold the same sum).
// Each stage halves the number of live values, so the whole reduction costs
// N - 1 shuffles per lane when N >= L instead of N * log2(L).
// ---------------------------------------------------------------------------
template <int N, int MASK>
struct Butterfly {
  __device__ __forceinline__ static void run(float *v, int lane) {
    if constexpr (MASK > 0) {
      if constexpr (N >= 2) {
        constexpr int H = N / 2;
        const bool upper = (lane & MASK) != 0;
#pragma unroll
        for (int i = 0; i < H; ++i) {
          const float send = upper ? v[i] : v[i + H];
          const float keep = upper ? v[i + H] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, MASK);
        }
        Butterfly<H, MASK / 2>::run(v, lane);
      } else {
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], MASK);
        Butterfly<1, MASK / 2>::run(v, lane);
      }
    }
  }
};

template <int X>
struct Log2 {
  static constexpr int value = 1 + Log2<X / 2>::value;
};
template <>
struct Log2<1> {
  static constexpr int value = 0;
};

// ---------------------------------------------------------------------------
// FP8 pages (E4M3, OCP "fn" form: bias 7, subnormals at exponent 0, no
// infinities, S.1111.111 NaN, largest finite 448).
// ---------------------------------------------------------------------------
// Quantise: the codes nearest to lo and hi (ties to the even mantissa,
// magnitudes at or above 448 saturating to 448, NaN stays NaN); lo's code in
// the low byte.
__device__ __forceinline__ uint32_t e4m3x2_nearest(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Sixteen bf16 elements (a: 0..7, b: 8..15) divided by `scale` (IEEE single
// precision division) and quantised to sixteen codes, element 0 lowest.
__device__ __forceinline__ uint4 bf16x16_to_e4m3(const uint4 &a, const uint4 &b, float scale) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float f0 = __fdiv_rn(__uint_as_float(w[2 * i] << 16), scale);
    const float f1 = __fdiv_rn(__uint_as_float(w[2 * i] & 0xffff0000u), scale);
    const float f2 = __fdiv_rn(__uint_as_float(w[2 * i + 1] << 16), scale);
    const float f3 = __fdiv_rn(__uint_as_float(w[2 * i + 1] & 0xffff0000u), scale);
    c[i] = e4m3x2_nearest(f0, f1) | (e4m3x2_nearest(f2, f3) << 16);
  }
  return make_uint4(c[0], c[1], c[2], c[3]);
}

}  // namespace pa
