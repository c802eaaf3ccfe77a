// Shared device helpers: the per-device error word and element conversions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "pagedkv.h"

namespace pagedkv {

// ---- host: per-device one-time set-up --------------------------------------
// A value computed once per device ordinal (a kernel attribute set, an
// occupancy, an attribute read) the first time a call runs with that device
// current; thread-safe. get() returns the cached value for the current device.
constexpr int kMaxDevices = 64;

template <typename T>
struct PerDevice {
  std::mutex mu;
  bool ready[kMaxDevices] = {};
  T value[kMaxDevices] = {};

  template <typename Init>
  cudaError_t get(T* out, Init init) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!ready[dev]) {
      e = init(&value[dev]);
      if (e != cudaSuccess) return e;
      ready[dev] = true;
    }
    *out = value[dev];
    return cudaSuccess;
  }
};

// SM count of the current device; 148 (a B200) when no device can be queried,
// e.g. workspace sizing on a host without a GPU.
inline int32_t device_sm_count() {
  static PerDevice<int32_t> cache;
  int32_t n = 0;
  cudaError_t e = cache.get(&n, [](int32_t* v) {
    int dev = 0;
    cudaError_t r = cudaGetDevice(&dev);
    if (r == cudaSuccess) r = cudaDeviceGetAttribute(v, cudaDevAttrMultiProcessorCount, dev);
    return r;
  });
  if (e != cudaSuccess || n <= 0) {
    cudaGetLastError();  // clear the sticky-free error of a failed query
    return 148;
  }
  return n;
}

// Raises the dynamic shared-memory limit of `kernel` to `bytes` once per device.
template <typename Kernel>
inline cudaError_t set_smem_once(PerDevice<int32_t>& cache, Kernel kernel, int32_t bytes) {
  int32_t done = 0;
  return cache.get(&done, [&](int32_t* v) {
    *v = 1;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  });
}

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
