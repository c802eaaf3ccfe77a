// Shared device helpers: the per-device error word and element conversions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pagedkv.h"

namespace pagedkv {

// Per-device error word (PA_DEVERR_* bits). Kernels OR bits in when they skip
// an out-of-range index; pa_get_device_error reads and clears it.
__device__ unsigned int g_error_word;

__device__ __forceinline__ void raise_device_error(unsigned int bits) {
  atomicOr(&g_error_word, bits);
}

constexpr float kLog2e = 1.4426950408889634f;

// Element <-> fp32. bf16 widening is exact (the bf16 pattern is the upper half
// of a binary32); narrowing rounds to nearest even.
template <typename T> struct Elem;
template <> struct Elem<float> {
  __device__ __forceinline__ static float to_f32(float x) { return x; }
  __device__ __forceinline__ static float from_f32(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  __device__ __forceinline__ static float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ __forceinline__ static __nv_bfloat16 from_f32(float x) { return __float2bfloat16_rn(x); }
};

// Bit views of vectors of N elements of T, loaded/stored as one access.
template <typename T, int N> struct alignas(sizeof(T) * N) Vec {
  T v[N];
};

template <typename T, int N>
__device__ __forceinline__ void load_f32(const T* __restrict__ p, float (&out)[N]) {
  Vec<T, N> x = *reinterpret_cast<const Vec<T, N>*>(p);
#pragma unroll
  for (int i = 0; i < N; ++i) out[i] = Elem<T>::to_f32(x.v[i]);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

}  // namespace pagedkv
