// Generic split-KV paged decode on CUDA cores: any supported dtype, head_dim
// and head group. Used for fp32 pools and shapes the staged bf16 kernels do
// not cover.
//
// One CTA = (partition, KV head g, sequence b), 4 warps. The warps take the
// partition's tokens round-robin; per token each lane holds D/32 contiguous
// elements of K and V (one vector load each), forms its part of the G dot
// products, and a 5-step warp-shuffle sum gives the scores. Every warp keeps
// its own online-softmax state per query head; the four states are merged in
// shared memory at the end. The token's block comes from the block table
// ("大模型推理性能优化：PagedAttention与Continuous Batching原理与实践" §2.2, gather
// through the page table).
#pragma once

#include "decode_common.cuh"

namespace pagedkv {

// Up to 8 query heads per KV head the per-head state fits in 128 registers, so
// the kernel is compiled for 4 resident CTAs per SM (which also lets the
// compiler keep the smallest instances out of local memory); 16 heads need
// more registers per thread.
template <typename T, int D, int GMAX>
__global__ void __launch_bounds__(128, GMAX <= 8 ? 4 : 1) decode_generic_kernel(DecodeParams p) {
  constexpr int NW = 4;
  constexpr int PER = D / 32;
  const int32_t part = blockIdx.x;
  const int32_t g = blockIdx.y;
  const int32_t b = blockIdx.z;
  const int32_t warp = threadIdx.x >> 5;
  const int32_t lane = threadIdx.x & 31;
  const int32_t G = p.group;
  const int32_t H = p.num_heads;
  T* out = reinterpret_cast<T*>(p.out);

  const int32_t L = checked_len(p, b, part == 0 && g == 0 && threadIdx.x == 0);
  const int32_t S = p.partition_tokens;
  const int32_t nparts = (L + S - 1) / S;
  if (L == 0) {
    if (part == 0)
      for (int32_t i = threadIdx.x; i < G * D; i += blockDim.x)
        out[((size_t)b * H + (size_t)g * G) * D + i] = Elem<T>::from_f32(0.f);
    return;
  }
  if (part >= nparts) return;
  const int32_t t0 = part * S;
  const int32_t t1 = min(t0 + S, L);

  __shared__ float q_s[GMAX][D];
  __shared__ float red_m[NW][GMAX];
  __shared__ float red_l[NW][GMAX];
  __shared__ float red_acc[NW][GMAX][D];

  const T* q = reinterpret_cast<const T*>(p.q) + ((size_t)b * H + (size_t)g * G) * D;
  for (int32_t i = threadIdx.x; i < G * D; i += blockDim.x)
    q_s[i / D][i % D] = Elem<T>::to_f32(q[i]) * p.scale_log2;
  __syncthreads();

  float qr[GMAX][PER];
  float m[GMAX], l[GMAX], acc[GMAX][PER];
#pragma unroll
  for (int h = 0; h < GMAX; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      acc[h][i] = 0.f;
      qr[h][i] = (h < G) ? q_s[h][lane * PER + i] : 0.f;
    }
  }

  const int32_t* table = p.block_tables + (size_t)b * p.max_blocks;
  const T* pool = reinterpret_cast<const T*>(p.pool);
  const size_t kv_stride = (size_t)p.num_kv_heads * 16 * D;  // K tile -> V tile
  for (int32_t t = t0 + warp; t < t1; t += NW) {
    const int32_t blk = __ldg(table + (t >> 4));
    float kf[PER], vf[PER];
    if (blk < 0 || blk >= p.num_blocks) {
      if (lane == 0) raise_device_error(PA_DEVERR_BLOCK);
#pragma unroll
      for (int i = 0; i < PER; ++i) kf[i] = vf[i] = 0.f;
    } else {
      const T* base = pool + ((size_t)blk * 2 * p.num_kv_heads + g) * 16 * D + (t & 15) * D + lane * PER;
      load_f32<T, PER>(base, kf);
      load_f32<T, PER>(base + kv_stride, vf);
    }
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
      if (h < G) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) s = fmaf(kf[i], qr[h][i], s);
        s = warp_sum(s);
        const float mn = fmaxf(m[h], s);
        const float a = exp2f(m[h] - mn);
        const float e = exp2f(s - mn);
        l[h] = l[h] * a + e;
#pragma unroll
        for (int i = 0; i < PER; ++i) acc[h][i] = fmaf(e, vf[i], acc[h][i] * a);
        m[h] = mn;
      }
    }
  }

#pragma unroll
  for (int h = 0; h < GMAX; ++h) {
    if (h < G) {
      if (lane == 0) {
        red_m[warp][h] = m[h];
        red_l[warp][h] = l[h];
      }
#pragma unroll
      for (int i = 0; i < PER; ++i) red_acc[warp][h][lane * PER + i] = acc[h][i];
    }
  }
  __syncthreads();

  for (int32_t i = threadIdx.x; i < G * D; i += blockDim.x) {
    const int32_t h = i / D;
    const int32_t d = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, red_m[w][h]);
    float Ls = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float e = exp2f(red_m[w][h] - M);  // 0 for a warp with no token
      Ls = fmaf(red_l[w][h], e, Ls);
      A = fmaf(red_acc[w][h][d], e, A);
    }
    const size_t bh = (size_t)b * H + (size_t)g * G + h;
    if (nparts == 1) {
      out[bh * D + d] = Elem<T>::from_f32(A / Ls);
    } else {
      p.ws_acc[(bh * p.max_partitions + part) * D + d] = A;
      if (d == 0) {
        p.ws_ml[(bh * p.max_partitions + part) * 2] = M;
        p.ws_ml[(bh * p.max_partitions + part) * 2 + 1] = Ls;
      }
    }
  }
}

}  // namespace pagedkv
