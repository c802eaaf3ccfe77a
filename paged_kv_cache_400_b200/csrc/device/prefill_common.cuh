// Arguments of the paged prefill kernels (tcgen05 and the mma.sync comparison
// build): sequence b holds seq_lens[b] tokens of KV, its newest
// query_start[b+1] - query_start[b] tokens are the queries.
#pragma once

#include "common.cuh"

namespace pagedkv {

struct PrefillParams {
  void* out;                    // [T][H][128] bf16
  const void* q;                // [T][H][128] bf16
  const int32_t* block_tables;  // [B][max_blocks]
  const int32_t* seq_lens;      // [B] KV length, new tokens included
  const int32_t* query_start;   // [B+1] first q row of each sequence
  int32_t max_blocks;
  int32_t num_heads;
  int32_t num_kv_heads;
  int32_t group;                // G = H / Hkv, a power of two <= 16
  int32_t num_blocks;
  int32_t tile_tokens;          // 64 / G
  int32_t max_query_len;
  int32_t num_tokens;           // rows of q / out
  float scale_log2;
};

}  // namespace pagedkv
