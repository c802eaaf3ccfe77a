// Parameters and the partition-reduce kernel shared by every decode variant.
//
// Split-KV decode: a sequence of length L is cut into ceil(L / S) partitions of
// S tokens. Each partition produces the online-softmax state of its tokens
// (running max m, sum l of exp(s - m), and acc = sum exp(s - m) V); a sequence
// with one partition is finished in place. The reduce merges the states by
// log-sum-exp. Scores are kept in the log2 domain (s * scale * log2 e), so every
// exponential is exp2.
#pragma once

#include "common.cuh"

namespace pagedkv {

struct DecodeParams {
  void* out;                    // [B][H][D] pool dtype
  const void* q;                // [B][H][D] pool dtype
  const void* pool;             // [N][2][Hkv][16][D]
  const int32_t* block_tables;  // [B][max_blocks]
  const int32_t* seq_lens;      // [B]
  float* ws_acc;                // [B][H][P][D] partial acc (fp32)
  float* ws_ml;                 // [B][H][P][2] partial (m, l)
  int32_t max_blocks;
  int32_t num_seqs;
  int32_t num_heads;
  int32_t num_kv_heads;
  int32_t group;                // H / Hkv
  int32_t num_blocks;           // N
  int32_t max_seq_len;
  int32_t partition_tokens;     // S, multiple of 16
  int32_t max_partitions;       // P = ceil(max_seq_len / S)
  float scale_log2;             // scale * log2(e)
};

// Effective length: an out-of-range length counts as 0 (its output is zeros);
// `report` raises PA_DEVERR_SEQLEN once for it.
__device__ __forceinline__ int32_t checked_len(const DecodeParams& p, int32_t b, bool report) {
  const int32_t L = __ldg(p.seq_lens + b);
  const bool ok = L >= 0 && L <= p.max_seq_len && (int64_t)L <= (int64_t)p.max_blocks * 16;
  if (!ok) {
    if (report) raise_device_error(PA_DEVERR_SEQLEN);
    return 0;
  }
  return L;
}

// Merge of the partition states of (b, h): grid (H, B), blockDim = D.
template <typename T, int D>
__global__ void __launch_bounds__(128) partition_reduce_kernel(DecodeParams p) {
  const int32_t h = blockIdx.x;
  const int32_t b = blockIdx.y;
  const int32_t L = checked_len(p, b, false);
  const int32_t nparts = (L + p.partition_tokens - 1) / p.partition_tokens;
  if (nparts <= 1) return;  // finished by the partition kernel
  const size_t bh = (size_t)b * p.num_heads + h;
  const float* ml = p.ws_ml + bh * p.max_partitions * 2;
  const float* acc = p.ws_acc + bh * p.max_partitions * D;
  float M = -INFINITY;
  for (int32_t i = 0; i < nparts; ++i) M = fmaxf(M, ml[2 * i]);
  float Lsum = 0.f;
  for (int32_t i = 0; i < nparts; ++i) Lsum += ml[2 * i + 1] * exp2f(ml[2 * i] - M);
  const float inv = 1.f / Lsum;
  for (int32_t d = threadIdx.x; d < D; d += blockDim.x) {
    float a = 0.f;
    for (int32_t i = 0; i < nparts; ++i) a += acc[(size_t)i * D + d] * exp2f(ml[2 * i] - M);
    reinterpret_cast<T*>(p.out)[bh * D + d] = Elem<T>::from_f32(a * inv);
  }
}

}  // namespace pagedkv
