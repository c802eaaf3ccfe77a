// C-ABI device entry points of libpagedkv.so: argument checks, kernel choice,
// launches. All kernels live in this one translation unit so they share the
// per-device error word without relocatable device code.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "../host/errors.hpp"
#include "append.cuh"
#include "common.cuh"
#include "decode_common.cuh"
#include "decode_generic.cuh"
#include "decode_staged.cuh"
#include "prefill_tc.cuh"
#ifdef PA_PREFILL_MMA_SYNC
#include "prefill.cuh"  // comparison build only: the mma.sync prefill kernel
#endif

using pagedkv::fail;

namespace {

// From this many partitions per sequence the staged decode runs as a
// persistent grid over a work list (largest partitions first) instead of one
// CTA per (partition, head, sequence): most grid CTAs of short sequences would
// be empty, and a few long sequences would finish last. Below it the plain
// grid is faster (no plan launch, no per-item latency).
#ifndef PA_WORKLIST_PARTITIONS
#define PA_WORKLIST_PARTITIONS 4
#endif
constexpr int32_t kWorkListPartitions = PA_WORKLIST_PARTITIONS;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(int32_t dtype) { return dtype == PA_BF16 ? 2 : 4; }

pa_status check_pool(const pa_pool_desc& pool, const char* fn) {
  if (pool.block_size != PA_BLOCK_SIZE)
    return fail(PA_ERR_UNSUPPORTED, "%s: block_size %d (only 16)", fn, pool.block_size);
  if (pool.dtype != PA_F32 && pool.dtype != PA_BF16)
    return fail(PA_ERR_UNSUPPORTED, "%s: dtype %d", fn, pool.dtype);
  if (pool.head_dim != 64 && pool.head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "%s: head_dim %d (64 or 128)", fn, pool.head_dim);
  if (pool.num_blocks <= 0 || pool.num_kv_heads <= 0)
    return fail(PA_ERR_INVALID_ARG, "%s: num_blocks %d, num_kv_heads %d", fn, pool.num_blocks,
                pool.num_kv_heads);
  return PA_OK;
}

pa_status launch_status(const char* fn) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
  return PA_OK;
}

#ifndef PA_PARTITION_TOKENS
#define PA_PARTITION_TOKENS 2048
#endif
static_assert(PA_PARTITION_TOKENS % 16 == 0 && PA_PARTITION_TOKENS / 16 <= pagedkv::kMaxPartitionBlocks,
              "partition of whole blocks, at most 2048 tokens (a warp holds at most 32 block ids)");

int32_t partition_tokens_for(int32_t num_seqs, const pa_pool_desc& pool, int32_t max_seq_len) {
  // PA_PARTITION_TOKENS-token partitions (2048 unless built otherwise: large
  // partitions keep the partial states and their merge small); halve while
  // the grid would not give every SM of the current device a few CTAs, down
  // to 128.
  int32_t S = PA_PARTITION_TOKENS;
  const int64_t pairs = (int64_t)num_seqs * pool.num_kv_heads;
  const int64_t want = 4 * (int64_t)pagedkv::device_sm_count();
  while (S > 128 && pairs * (((int64_t)max_seq_len + S - 1) / S) < want) S /= 2;
  return S;
}

// The persistent decode's work items hold the partition index in 16 bits.
constexpr int64_t kMaxPartitions = 65535;

// Host-side checks shared by pa_decode, pa_append_decode and
// pa_decode_noalloc, in this order: pool, sizes, head group, table width,
// scale, then (for a non-empty batch) the partition count, pointers and
// alignment. The workspace is checked by the caller afterwards.
pa_status check_decode_args(const char* fn, const void* out, const void* q, const void* kv_pool,
                            const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                            int32_t num_seqs, int32_t num_heads, float scale, const pa_pool_desc& pool,
                            int32_t max_seq_len) {
  pa_status s = check_pool(pool, fn);
  if (s != PA_OK) return s;
  if (num_seqs < 0 || num_heads <= 0 || max_blocks_per_seq <= 0 || max_seq_len < 0)
    return fail(PA_ERR_INVALID_ARG, "%s: num_seqs %d, num_heads %d, max_blocks %d, max_seq_len %d", fn, num_seqs,
                num_heads, max_blocks_per_seq, max_seq_len);
  if (num_heads % pool.num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "%s: num_heads %d not a multiple of num_kv_heads %d", fn, num_heads,
                pool.num_kv_heads);
  const int32_t G = num_heads / pool.num_kv_heads;
  if (G > 16) return fail(PA_ERR_UNSUPPORTED, "%s: head group %d > 16", fn, G);
  if (num_seqs > 65535) return fail(PA_ERR_UNSUPPORTED, "%s: num_seqs %d > 65535", fn, num_seqs);
  if ((int64_t)max_seq_len > (int64_t)max_blocks_per_seq * PA_BLOCK_SIZE)
    return fail(PA_ERR_INVALID_ARG, "%s: max_seq_len %d > max_blocks_per_seq * 16", fn, max_seq_len);
  if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "%s: scale is not finite", fn);
  if (num_seqs == 0) return PA_OK;
  const int32_t S = partition_tokens_for(num_seqs, pool, max_seq_len > 0 ? max_seq_len : 1);
  if (((int64_t)max_seq_len + S - 1) / S > kMaxPartitions)
    return fail(PA_ERR_UNSUPPORTED, "%s: max_seq_len %d needs more than %lld partitions of %d tokens", fn,
                max_seq_len, (long long)kMaxPartitions, S);
  if (!out || !q || !kv_pool || !block_tables || !seq_lens) return fail(PA_ERR_INVALID_ARG, "%s: NULL pointer", fn);
  if (!aligned16(out) || !aligned16(q) || !aligned16(kv_pool))
    return fail(PA_ERR_INVALID_ARG, "%s: out, q and kv_pool must be 16-byte aligned", fn);
  return PA_OK;
}

struct WorkspaceLayout {
  size_t acc_bytes, ml_offset, items_offset, header_offset, total;
  int32_t partitions;
};

WorkspaceLayout workspace_layout(int32_t num_seqs, int32_t num_heads, const pa_pool_desc& pool,
                                 int32_t max_seq_len) {
  WorkspaceLayout w{0, 0, 0, 0, 0, 0};
  const int32_t S = partition_tokens_for(num_seqs, pool, max_seq_len);
  w.partitions = (int32_t)(((int64_t)max_seq_len + S - 1) / S);
  if (w.partitions <= 1) return w;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t units = (size_t)num_seqs * num_heads * w.partitions;
  w.acc_bytes = units * pool.head_dim * sizeof(float);
  w.ml_offset = up(w.acc_bytes);
  // work list of the persistent decode: one int per (sequence, partition)
  w.items_offset = up(w.ml_offset + units * 2 * sizeof(float));
  w.header_offset = up(w.items_offset + (size_t)num_seqs * w.partitions * sizeof(int32_t));
  w.total = w.header_offset + 2 * sizeof(int32_t);
  return w;
}

template <typename T, int D>
pa_status launch_generic(const pagedkv::DecodeParams& p, cudaStream_t st) {
  dim3 grid(p.max_partitions, p.num_kv_heads, p.num_seqs);
  const int G = p.group;
  if (G <= 1) pagedkv::decode_generic_kernel<T, D, 1><<<grid, 128, 0, st>>>(p);
  else if (G <= 2) pagedkv::decode_generic_kernel<T, D, 2><<<grid, 128, 0, st>>>(p);
  else if (G <= 4) pagedkv::decode_generic_kernel<T, D, 4><<<grid, 128, 0, st>>>(p);
  else if (G <= 8) pagedkv::decode_generic_kernel<T, D, 8><<<grid, 128, 0, st>>>(p);
  else pagedkv::decode_generic_kernel<T, D, 16><<<grid, 128, 0, st>>>(p);
  pa_status s = launch_status("pa_decode");
  if (s != PA_OK || p.max_partitions <= 1) return s;
  cudaError_t e = pagedkv::launch_partition_merge<T, D>(p, st);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_decode (merge): launch failed: %s", cudaGetErrorString(e));
  return PA_OK;
}

}  // namespace

extern "C" {

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported configuration";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_NO_BLOCKS: return "no free blocks";
    case PA_ERR_UNKNOWN_SEQ: return "unknown sequence";
    case PA_ERR_DEVICE_BOUNDS: return "device index out of bounds";
    case PA_ERR_SEQ_EXISTS: return "sequence exists";
    case PA_ERR_CAPACITY: return "capacity exceeded";
    case PA_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

const char* pa_last_error(void) { return pagedkv::last_error_slot().c_str(); }

pa_status pa_reshape_and_cache(const void* k, const void* v, void* kv_pool,
                               const int64_t* slot_mapping, int32_t num_tokens,
                               pa_pool_desc pool, void* stream) {
  pa_status s = check_pool(pool, "pa_reshape_and_cache");
  if (s != PA_OK) return s;
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "pa_reshape_and_cache: num_tokens %d", num_tokens);
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !kv_pool || !slot_mapping)
    return fail(PA_ERR_INVALID_ARG, "pa_reshape_and_cache: NULL pointer");
  if (!aligned16(k) || !aligned16(v) || !aligned16(kv_pool))
    return fail(PA_ERR_INVALID_ARG, "pa_reshape_and_cache: k, v and kv_pool must be 16-byte aligned");
  const int32_t chunks = (int32_t)(pool.head_dim * elem_size(pool.dtype) / 16);  // 8, 16 or 32
  const int64_t per_rows = (int64_t)num_tokens * chunks;  // chunks of one (K|V, head) across the tokens
  const dim3 grid((unsigned)((per_rows + 255) / 256), (unsigned)pool.num_kv_heads, 2);
  const uint4* k4 = reinterpret_cast<const uint4*>(k);
  const uint4* v4 = reinterpret_cast<const uint4*>(v);
  uint4* p4 = reinterpret_cast<uint4*>(kv_pool);
  const int64_t num_slots = (int64_t)pool.num_blocks * PA_BLOCK_SIZE;
  cudaStream_t st = (cudaStream_t)stream;
  if (chunks == 8)
    pagedkv::append_kernel<8><<<grid, 256, 0, st>>>(k4, v4, p4, slot_mapping, num_tokens, pool.num_kv_heads, num_slots);
  else if (chunks == 16)
    pagedkv::append_kernel<16><<<grid, 256, 0, st>>>(k4, v4, p4, slot_mapping, num_tokens, pool.num_kv_heads, num_slots);
  else
    pagedkv::append_kernel<32><<<grid, 256, 0, st>>>(k4, v4, p4, slot_mapping, num_tokens, pool.num_kv_heads, num_slots);
  return launch_status("pa_reshape_and_cache");
}

int32_t pa_decode_partition_tokens(int32_t num_seqs, int32_t num_heads, pa_pool_desc pool,
                                   int32_t max_seq_len) {
  (void)num_heads;
  if (num_seqs < 0 || max_seq_len < 0 || pool.num_kv_heads <= 0) return 0;
  return partition_tokens_for(num_seqs, pool, max_seq_len);
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads, pa_pool_desc pool,
                                int32_t max_seq_len) {
  if (num_seqs <= 0 || num_heads <= 0 || max_seq_len <= 0 || pool.num_kv_heads <= 0 ||
      pool.head_dim <= 0)
    return 0;
  return workspace_layout(num_seqs, num_heads, pool, max_seq_len).total;
}

pa_status pa_decode(void* out, const void* q, const void* kv_pool, const int32_t* block_tables,
                    int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t num_seqs,
                    int32_t num_heads, float scale, pa_pool_desc pool, void* workspace,
                    size_t workspace_bytes, int32_t max_seq_len, void* stream) {
  pa_status s = check_decode_args("pa_decode", out, q, kv_pool, block_tables, max_blocks_per_seq, seq_lens,
                                  num_seqs, num_heads, scale, pool, max_seq_len);
  if (s != PA_OK || num_seqs == 0) return s;
  const int32_t G = num_heads / pool.num_kv_heads;
  const WorkspaceLayout w = workspace_layout(num_seqs, num_heads, pool, max_seq_len > 0 ? max_seq_len : 1);
  if (w.total > 0 && (!workspace || workspace_bytes < w.total))
    return fail(PA_ERR_WORKSPACE, "pa_decode: workspace %zu bytes at %p, need %zu", workspace_bytes,
                workspace, w.total);
  if (w.total > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(PA_ERR_INVALID_ARG, "pa_decode: workspace must be 256-byte aligned");

  pagedkv::DecodeParams p;
  p.out = out;
  p.q = q;
  p.pool = kv_pool;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.ws_acc = reinterpret_cast<float*>(workspace);
  p.ws_ml = w.total ? reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + w.ml_offset) : nullptr;
  p.k_new = nullptr;
  p.v_new = nullptr;
  p.slot_mapping = nullptr;
  const bool use_list = w.total && w.partitions >= kWorkListPartitions;
  p.work_items = use_list ? reinterpret_cast<int32_t*>(reinterpret_cast<char*>(workspace) + w.items_offset) : nullptr;
  p.work_header =
      use_list ? reinterpret_cast<int32_t*>(reinterpret_cast<char*>(workspace) + w.header_offset) : nullptr;
  p.max_blocks = max_blocks_per_seq;
  p.num_seqs = num_seqs;
  p.num_heads = num_heads;
  p.num_kv_heads = pool.num_kv_heads;
  p.group = G;
  p.num_blocks = pool.num_blocks;
  p.max_seq_len = max_seq_len;
  p.partition_tokens = partition_tokens_for(num_seqs, pool, max_seq_len > 0 ? max_seq_len : 1);
  p.max_partitions = w.partitions > 0 ? w.partitions : 1;
  p.scale_log2 = scale * pagedkv::kLog2e;
  cudaStream_t st = (cudaStream_t)stream;

  if (pool.dtype == PA_BF16 && pool.head_dim == 128) {
    pa_status r = pagedkv::launch_staged_bf16_d128(p, st);
    if (r != PA_ERR_UNSUPPORTED) return r;
  }
  if (pool.dtype == PA_BF16) {
    return pool.head_dim == 128 ? launch_generic<__nv_bfloat16, 128>(p, st)
                                : launch_generic<__nv_bfloat16, 64>(p, st);
  }
  return pool.head_dim == 128 ? launch_generic<float, 128>(p, st) : launch_generic<float, 64>(p, st);
}

pa_status pa_append_decode(void* out, const void* q, const void* k_new, const void* v_new, void* kv_pool,
                           const int64_t* slot_mapping, const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* seq_lens, int32_t num_seqs, int32_t num_heads, float scale,
                           pa_pool_desc pool, void* workspace, size_t workspace_bytes, int32_t max_seq_len,
                           void* stream) {
  if (num_seqs > 0 && (!k_new || !v_new || !slot_mapping))
    return fail(PA_ERR_INVALID_ARG, "pa_append_decode: NULL k_new, v_new or slot_mapping");
  if (num_seqs > 0 && (!aligned16(k_new) || !aligned16(v_new)))
    return fail(PA_ERR_INVALID_ARG, "pa_append_decode: k_new and v_new must be 16-byte aligned");
  const bool staged = pool.dtype == PA_BF16 && pool.head_dim == 128 && pool.block_size == PA_BLOCK_SIZE;
  if (!staged) {
    // other shapes: the two calls in sequence (same results)
    pa_status s = pa_reshape_and_cache(k_new, v_new, kv_pool, slot_mapping, num_seqs, pool, stream);
    if (s != PA_OK) return s;
    return pa_decode(out, q, kv_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_heads, scale, pool,
                     workspace, workspace_bytes, max_seq_len, stream);
  }
  // Validate exactly as pa_decode does, then launch the decode kernel with the
  // append folded in.
  pa_status s = check_decode_args("pa_append_decode", out, q, kv_pool, block_tables, max_blocks_per_seq, seq_lens,
                                  num_seqs, num_heads, scale, pool, max_seq_len);
  if (s != PA_OK || num_seqs == 0) return s;
  const int32_t G = num_heads / pool.num_kv_heads;
  const WorkspaceLayout w = workspace_layout(num_seqs, num_heads, pool, max_seq_len > 0 ? max_seq_len : 1);
  if (w.total > 0 && (!workspace || workspace_bytes < w.total))
    return fail(PA_ERR_WORKSPACE, "pa_append_decode: workspace %zu bytes at %p, need %zu", workspace_bytes,
                workspace, w.total);
  if (w.total > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(PA_ERR_INVALID_ARG, "pa_append_decode: workspace must be 256-byte aligned");
  pagedkv::DecodeParams p;
  p.out = out;
  p.q = q;
  p.pool = kv_pool;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.ws_acc = reinterpret_cast<float*>(workspace);
  p.ws_ml = w.total ? reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + w.ml_offset) : nullptr;
  p.k_new = k_new;
  p.v_new = v_new;
  p.slot_mapping = slot_mapping;
  const bool use_list = w.total && w.partitions >= kWorkListPartitions;
  p.work_items = use_list ? reinterpret_cast<int32_t*>(reinterpret_cast<char*>(workspace) + w.items_offset) : nullptr;
  p.work_header =
      use_list ? reinterpret_cast<int32_t*>(reinterpret_cast<char*>(workspace) + w.header_offset) : nullptr;
  p.max_blocks = max_blocks_per_seq;
  p.num_seqs = num_seqs;
  p.num_heads = num_heads;
  p.num_kv_heads = pool.num_kv_heads;
  p.group = G;
  p.num_blocks = pool.num_blocks;
  p.max_seq_len = max_seq_len;
  p.partition_tokens = partition_tokens_for(num_seqs, pool, max_seq_len > 0 ? max_seq_len : 1);
  p.max_partitions = w.partitions > 0 ? w.partitions : 1;
  p.scale_log2 = scale * pagedkv::kLog2e;
  return pagedkv::launch_staged_bf16_d128(p, (cudaStream_t)stream);
}

pa_status pa_prefill(void* out, const void* q, const void* kv_pool, const int32_t* block_tables,
                     int32_t max_blocks_per_seq, const int32_t* seq_lens, const int32_t* query_start,
                     int32_t num_seqs, int32_t num_tokens, int32_t num_heads, float scale, pa_pool_desc pool,
                     int32_t max_query_len, void* stream) {
  pa_status s = check_pool(pool, "pa_prefill");
  if (s != PA_OK) return s;
  if (pool.dtype != PA_BF16 || pool.head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "pa_prefill: only bf16 pools with head_dim 128");
  if (num_seqs < 0 || num_tokens < 0 || num_heads <= 0 || max_blocks_per_seq <= 0 || max_query_len < 0)
    return fail(PA_ERR_INVALID_ARG,
                "pa_prefill: num_seqs %d, num_tokens %d, num_heads %d, max_blocks %d, max_query_len %d", num_seqs,
                num_tokens, num_heads, max_blocks_per_seq, max_query_len);
  if (max_query_len > num_tokens)
    return fail(PA_ERR_INVALID_ARG, "pa_prefill: max_query_len %d > num_tokens %d", max_query_len, num_tokens);
  if (num_heads % pool.num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "pa_prefill: num_heads %d not a multiple of num_kv_heads %d", num_heads,
                pool.num_kv_heads);
  const int32_t G = num_heads / pool.num_kv_heads;
  if (G > 16 || (G & (G - 1)) != 0)
    return fail(PA_ERR_UNSUPPORTED, "pa_prefill: head group %d (1, 2, 4, 8 or 16)", G);
  if (num_seqs > 65535 || pool.num_kv_heads > 65535)
    return fail(PA_ERR_UNSUPPORTED, "pa_prefill: num_seqs %d or num_kv_heads %d > 65535", num_seqs,
                pool.num_kv_heads);
  if ((int64_t)max_query_len > (int64_t)max_blocks_per_seq * PA_BLOCK_SIZE)
    return fail(PA_ERR_INVALID_ARG, "pa_prefill: max_query_len %d > max_blocks_per_seq * 16", max_query_len);
  if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "pa_prefill: scale is not finite");
  if (num_seqs == 0 || max_query_len == 0) return PA_OK;
  if (!out || !q || !kv_pool || !block_tables || !seq_lens || !query_start)
    return fail(PA_ERR_INVALID_ARG, "pa_prefill: NULL pointer");
  if (!aligned16(out) || !aligned16(q) || !aligned16(kv_pool))
    return fail(PA_ERR_INVALID_ARG, "pa_prefill: out, q and kv_pool must be 16-byte aligned");
  pagedkv::PrefillParams p;
  p.out = out;
  p.q = q;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.query_start = query_start;
  p.max_blocks = max_blocks_per_seq;
  p.num_heads = num_heads;
  p.num_kv_heads = pool.num_kv_heads;
  p.group = G;
  p.num_blocks = pool.num_blocks;
  p.tile_tokens = 64 / G;
  p.max_query_len = max_query_len;
  p.num_tokens = num_tokens;
  p.scale_log2 = scale * pagedkv::kLog2e;
#ifdef PA_PREFILL_MMA_SYNC
  // comparison build: the mma.sync kernel (same results within rounding)
  p.tile_tokens = 64 / G;
  return pagedkv::launch_prefill_bf16_d128(kv_pool, pool.num_blocks, p, num_seqs, (cudaStream_t)stream);
#else
  p.tile_tokens = 128 / G;
  return pagedkv::launch_prefill_tc(kv_pool, pool.num_blocks, p, num_seqs, (cudaStream_t)stream);
#endif
}

pa_status pa_copy_blocks(void* kv_pool, const int32_t* src, const int32_t* dst, int32_t n,
                         pa_pool_desc pool, void* stream) {
  pa_status s = check_pool(pool, "pa_copy_blocks");
  if (s != PA_OK) return s;
  if (n < 0) return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: n %d", n);
  if (n == 0) return PA_OK;
  if (!kv_pool || !src || !dst) return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: NULL pointer");
  if (!aligned16(kv_pool)) return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: kv_pool must be 16-byte aligned");
  const int64_t chunks = (int64_t)2 * pool.num_kv_heads * PA_BLOCK_SIZE * pool.head_dim *
                         (int64_t)elem_size(pool.dtype) / 16;
  pagedkv::copy_blocks_kernel<<<n, 256, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<uint4*>(kv_pool), src, dst, pool.num_blocks, chunks);
  return launch_status("pa_copy_blocks");
}

namespace {

// A pool the GPU can address: device memory, or pinned host memory mapped
// into the device's address space (checked at both ends of the range).
pa_status check_addressable(const void* p, size_t bytes, const char* fn, const char* name) {
  for (const char* q : {static_cast<const char*>(p), static_cast<const char*>(p) + bytes - 1}) {
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, q);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(PA_ERR_INVALID_ARG, "%s: %s is not memory the GPU can address (%s)", fn, name,
                  cudaGetErrorString(e));
    }
    const bool ok = (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged ||
                     (a.type == cudaMemoryTypeHost && a.devicePointer == q));
    if (!ok)
      return fail(PA_ERR_INVALID_ARG, "%s: %s must be device memory or mapped pinned host memory", fn, name);
  }
  return PA_OK;
}

}  // namespace

pa_status pa_copy_blocks_between(void* dst_pool, int32_t dst_num_blocks, const void* src_pool,
                                 int32_t src_num_blocks, const int32_t* src, const int32_t* dst, int32_t n,
                                 pa_pool_desc pool, void* stream) {
  pa_pool_desc d = pool;
  d.num_blocks = 1;
  pa_status s = check_pool(d, "pa_copy_blocks_between");
  if (s != PA_OK) return s;
  if (n < 0 || dst_num_blocks <= 0 || src_num_blocks <= 0)
    return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks_between: n %d, blocks %d / %d", n, dst_num_blocks,
                src_num_blocks);
  if (n == 0) return PA_OK;
  if (!dst_pool || !src_pool || !src || !dst)
    return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks_between: NULL pointer");
  if (!aligned16(dst_pool) || !aligned16(src_pool))
    return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks_between: pools must be 16-byte aligned");
  const size_t block_bytes =
      (size_t)2 * pool.num_kv_heads * PA_BLOCK_SIZE * pool.head_dim * elem_size(pool.dtype);
  if ((s = check_addressable(dst_pool, block_bytes * dst_num_blocks, "pa_copy_blocks_between", "dst_pool")) != PA_OK)
    return s;
  if ((s = check_addressable(src_pool, block_bytes * src_num_blocks, "pa_copy_blocks_between", "src_pool")) != PA_OK)
    return s;
  if ((s = check_addressable(src, sizeof(int32_t) * n, "pa_copy_blocks_between", "src")) != PA_OK) return s;
  if ((s = check_addressable(dst, sizeof(int32_t) * n, "pa_copy_blocks_between", "dst")) != PA_OK) return s;
  const int64_t chunks = (int64_t)(block_bytes / 16);
  int32_t split = 1;
  while (split < 16 && (chunks % (split * 2)) == 0 && chunks / (split * 2) >= 256) split *= 2;
  pagedkv::copy_blocks_between_kernel<<<(unsigned)(n * split), 256, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<uint4*>(dst_pool), dst_num_blocks, reinterpret_cast<const uint4*>(src_pool),
      src_num_blocks, src, dst, chunks, split);
  return launch_status("pa_copy_blocks_between");
}

namespace pagedkv {
// One thread waits on a barrier nothing arrives at; the bounded wait gives up
// after limit_ns and the error bit is raised as the kernels raise it.
__global__ void selftest_timeout_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  if (!mbar_wait_bounded(&bar, 0, limit_ns)) raise_device_error(PA_DEVERR_TIMEOUT);
}
}  // namespace pagedkv

pa_status pa_selftest_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1 || limit_ns > 1000000000ull)
    return fail(PA_ERR_INVALID_ARG, "pa_selftest_timeout: limit %llu ns outside 1 .. 1e9",
                (unsigned long long)limit_ns);
  pagedkv::selftest_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_ns);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_selftest_timeout: %s", cudaGetErrorString(e));
  return PA_OK;
}

pa_status pa_get_device_error(uint32_t* flags, void* stream) {
  if (!flags) return fail(PA_ERR_INVALID_ARG, "pa_get_device_error: flags is NULL");
  void* addr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&addr, pagedkv::g_error_word);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_get_device_error: %s", cudaGetErrorString(e));
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t v = 0;
  e = cudaMemcpyAsync(&v, addr, sizeof(v), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(addr, 0, sizeof(uint32_t), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_get_device_error: %s", cudaGetErrorString(e));
  *flags = v;
  return v ? PA_ERR_DEVICE_BOUNDS : PA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// pa_decode_noalloc: decode for callers that cannot allocate device memory.
// The split-KV partial results go to one fixed array in this file instead of
// a caller-provided workspace.
// ---------------------------------------------------------------------------
namespace {

// Scratch of pa_decode_noalloc. One per device, created when the module is
// loaded on that device and kept until exit; shared by every call.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device. In host code the
// array's name is only a stand-in, never a device address: the address comes
// from cudaGetSymbolAddress, once per device, with that device current.
pa_status noalloc_scratch(void** ptr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_decode_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return fail(PA_ERR_UNSUPPORTED, "pa_decode_noalloc: device ordinal %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(PA_ERR_CUDA, "pa_decode_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_noalloc(void* out, const void* q, const void* kv_pool,
                                       const int32_t* block_tables, int32_t max_blocks_per_seq,
                                       const int32_t* seq_lens, int32_t num_seqs, int32_t num_heads,
                                       float scale, pa_pool_desc pool, int32_t max_seq_len,
                                       void* stream) {
  // pa_decode's own argument errors come first, then the scratch limit
  pa_status s = check_decode_args("pa_decode_noalloc", out, q, kv_pool, block_tables, max_blocks_per_seq, seq_lens,
                                  num_seqs, num_heads, scale, pool, max_seq_len);
  if (s != PA_OK || num_seqs == 0) return s;
  const size_t need = pa_decode_workspace_size(num_seqs, num_heads, pool, max_seq_len);
  if (need > PA_DECODE_NOALLOC_SCRATCH_BYTES)
    return fail(PA_ERR_WORKSPACE,
                "pa_decode_noalloc: this shape needs %zu bytes of split-KV scratch, the fixed array holds %u; "
                "use pa_decode with a workspace",
                need, (unsigned)PA_DECODE_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != PA_OK) return s;
  return pa_decode(out, q, kv_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_heads, scale,
                   pool, scratch, PA_DECODE_NOALLOC_SCRATCH_BYTES, max_seq_len, stream);
}
