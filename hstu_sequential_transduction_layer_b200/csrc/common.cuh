// Shared device-side helpers of libhstu_b200: the device status word, dtype traits, vector I/O.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "hstu.h"

namespace hstu {

// First device-side error wins; hstu_get_device_status() reads and clears it.  (The library is a
// single translation unit, so the definition lives here.)
__device__ int g_device_status = 0;

__device__ __forceinline__ void report(int code) { atomicCAS(&g_device_status, 0, code); }

// Host-side count of kernel launches issued by the library (hstu_launch_count()).
inline std::atomic<uint64_t> g_launches{0};
inline void count_launch(uint64_t n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

using bf16 = __nv_bfloat16;

template <typename T> struct io;
template <> struct io<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
};
template <> struct io<bf16> {
  static __device__ __forceinline__ float load(const bf16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void store(bf16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// Round-to-nearest-even pack of two floats into bf16x2 (low half = a).
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// SiLU(x) = x * sigmoid(x).  Accurate form for the fp32 path.
__device__ __forceinline__ float silu_accurate(float x) { return x / (1.0f + expf(-x)); }
// Fast form for bf16 outputs: exp via ex2.approx, divide via the approximate reciprocal.
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

__device__ __forceinline__ int64_t clamp64(int64_t v, int64_t lo, int64_t hi) {
  return v < lo ? lo : (v > hi ? hi : v);
}

}  // namespace hstu
