// Shared device helpers of the paged KV library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pagedkv.h"

namespace pkv {

constexpr float kLog2e = 1.4426950408889634f;

// ---- element loads widened to fp32 ------------------------------------------

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f32(float x) { return x; }
};
template <> struct Elem<__half> {
  static __device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
};
template <> struct Elem<__nv_fp8_storage_t> {
  static __device__ __forceinline__ float to_f32(__nv_fp8_storage_t x) {
    __half_raw h = __nv_cvt_fp8_to_halfraw(x, __NV_E4M3);
    return __half2float(__half(h));
  }
};

// Round-to-nearest-even store of an fp32 value into the output dtype.
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Load N consecutive elements (4, 8 or a multiple of 16 bytes, aligned) as fp32.
template <typename T, int N>
__device__ __forceinline__ void load_row(const T* __restrict__ p, float (&v)[N]) {
  constexpr int kBytes = N * (int)sizeof(T);
  static_assert(kBytes == 4 || kBytes == 8 || kBytes % 16 == 0, "unsupported row chunk");
  if constexpr (kBytes == 4) {
    uint32_t raw = __ldg(reinterpret_cast<const unsigned int*>(p));
    const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
    for (int j = 0; j < N; ++j) v[j] = Elem<T>::to_f32(e[j]);
  } else if constexpr (kBytes % 16 == 0) {
    constexpr int kVec = kBytes / 16;
    constexpr int kPer = 16 / (int)sizeof(T);
#pragma unroll
    for (int k = 0; k < kVec; ++k) {
      uint4 raw = __ldg(reinterpret_cast<const uint4*>(p) + k);
      const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int j = 0; j < kPer; ++j) v[k * kPer + j] = Elem<T>::to_f32(e[j]);
    }
  } else {
    uint2 raw = __ldg(reinterpret_cast<const uint2*>(p));
    const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
    for (int j = 0; j < N; ++j) v[j] = Elem<T>::to_f32(e[j]);
  }
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float fast_log2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__host__ __device__ __forceinline__ int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace pkv
