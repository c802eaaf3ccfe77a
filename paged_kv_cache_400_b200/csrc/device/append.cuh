// Cache append ("scatter" of each new token's K/V into its slot) and whole-block
// copy for copy-on-write.
//
// "大模型推理性能优化：PagedAttention与Continuous Batching原理与实践" §2.2 names the
// scatter of new K/V into scattered pages as one of the two memory operations
// PagedAttention kernels must do well; "vLLM 原理" / 工作原理 §2 gives the
// position -> (page, row) mapping. The kernels are plain 16-byte copies: every
// thread moves one 16-byte chunk, consecutive threads take consecutive chunks
// of one (token, K|V, head) row, so each row is one coalesced run on both sides.
#pragma once

#include "common.cuh"

namespace pagedkv {

// One thread per 16-byte chunk. CTA (x, h, kv) covers 256 consecutive chunks
// of the rows (token t, K|V kv, KV head h) in token order, kChunks chunks per
// row (a compile-time count, so the index arithmetic is a shift and a mask;
// the head and K|V come from the grid, not from a division).
template <int kChunks>
__global__ void __launch_bounds__(256)
append_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ pool,
              const int64_t* __restrict__ slots, int32_t num_tokens, int32_t num_kv_heads, int64_t num_slots) {
  const int32_t h = blockIdx.y;
  const int32_t kv = blockIdx.z;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t t = e / kChunks;
  const int32_t c = (int32_t)(e % kChunks);
  if (t >= num_tokens) return;
  const int64_t s = __ldg(slots + t);
  if (s < 0) return;  // padding
  if (s >= num_slots) {
    if (c == 0 && h == 0 && kv == 0) raise_device_error(PA_DEVERR_SLOT);
    return;
  }
  const int64_t blk = s >> 4;
  const int32_t row = (int32_t)(s & 15);
  const uint4* src = (kv ? v : k) + (t * num_kv_heads + h) * kChunks + c;
  uint4* dst = pool + (((blk * 2 + kv) * num_kv_heads + h) * 16 + row) * kChunks + c;
  *dst = __ldg(src);
}

// One CTA per pair; the CTA copies the whole block as 16-byte chunks.
__global__ void __launch_bounds__(256)
copy_blocks_kernel(uint4* __restrict__ pool, const int32_t* __restrict__ src,
                   const int32_t* __restrict__ dst, int32_t num_blocks, int64_t chunks_per_block) {
  const int32_t s = src[blockIdx.x];
  const int32_t d = dst[blockIdx.x];
  if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) {
    if (threadIdx.x == 0) raise_device_error(PA_DEVERR_BLOCK);
    return;
  }
  const uint4* from = pool + (int64_t)s * chunks_per_block;
  uint4* to = pool + (int64_t)d * chunks_per_block;
  for (int64_t i = threadIdx.x; i < chunks_per_block; i += blockDim.x) to[i] = from[i];
}

// Whole-block copy between two pools of the same block shape (device <->
// pinned host for swapping, or device <-> device): pair i copies block src[i]
// of `from` to block dst[i] of `to`. Each block is split across `split` CTAs
// so that even a few pairs keep many 16-byte transfers in flight (a PCIe or
// C2C link needs that to reach its bandwidth).
__global__ void __launch_bounds__(256)
copy_blocks_between_kernel(uint4* __restrict__ to, int32_t to_blocks, const uint4* __restrict__ from,
                           int32_t from_blocks, const int32_t* __restrict__ src, const int32_t* __restrict__ dst,
                           int64_t chunks_per_block, int32_t split) {
  const int32_t pair = blockIdx.x / split;
  const int32_t part = blockIdx.x % split;
  const int32_t s = src[pair];
  const int32_t d = dst[pair];
  if (s < 0 || s >= from_blocks || d < 0 || d >= to_blocks) {
    if (threadIdx.x == 0 && part == 0) raise_device_error(PA_DEVERR_BLOCK);
    return;
  }
  const int64_t per = chunks_per_block / split;
  const uint4* a = from + (int64_t)s * chunks_per_block + part * per;
  uint4* b = to + (int64_t)d * chunks_per_block + part * per;
  for (int64_t i = threadIdx.x; i < per; i += blockDim.x) b[i] = a[i];
}

}  // namespace pagedkv
