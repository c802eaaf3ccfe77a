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
  const void* k_new;            // fused append: [B][Hkv][D] new token K (or null)
  const void* v_new;            // fused append: [B][Hkv][D] new token V
  const int64_t* slot_mapping;  // fused append: [B] slot of each new token
  int32_t* work_items;          // persistent decode: (b << 16 | part) items, or null
  int32_t* work_header;         // [0] item count, [1] next-item counter
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

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Merge of the partition states of one (sequence b, KV head g): its G query
// heads, grid (Hkv, B), 128 threads. All (m, l) pairs are read at once into
// shared memory, each head's weights exp2(m_p - M) / L are formed once, and
// each output element then sums its partial accumulators with every load of a
// round in flight together (a few L2 round trips per CTA, not one per
// partition). Launched as a programmatic dependent of the partition kernel:
// everything before griddepcontrol.wait may overlap that kernel's tail.
constexpr int kMergeThreads = 128;
constexpr int kMergeMaxParts = 64;

template <typename T, int D>
__global__ void __launch_bounds__(kMergeThreads) partition_merge_kernel(DecodeParams p) {
  constexpr int kOut = 4;     // output elements per thread per round
  constexpr int kChunk = 16;  // partitions summed per round
  __shared__ float w[16][kMergeMaxParts];
  __shared__ float wl[16][kMergeMaxParts];
  const int32_t g = blockIdx.x;
  const int32_t b = blockIdx.y;
  const int32_t G = p.group;
  const int32_t L = checked_len(p, b, false);
  const int32_t nparts = (L + p.partition_tokens - 1) / p.partition_tokens;
  if (nparts <= 1) return;  // finished by the partition kernel
  grid_dependency_wait();   // the partition kernel's states are complete and visible
  const size_t bh0 = (size_t)b * p.num_heads + (size_t)g * G;
  if (nparts <= kMergeMaxParts) {
    for (int32_t i = threadIdx.x; i < G * nparts; i += blockDim.x) {
      const int32_t h = i / nparts;
      const int32_t q = i % nparts;
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.ws_ml) + (bh0 + h) * p.max_partitions + q);
      w[h][q] = ml.x;
      wl[h][q] = ml.y;
    }
    __syncthreads();
    if (threadIdx.x < G) {
      const int32_t h = threadIdx.x;
      float M = -INFINITY;
      for (int32_t q = 0; q < nparts; ++q) M = fmaxf(M, w[h][q]);
      float Ls = 0.f;
      for (int32_t q = 0; q < nparts; ++q) {
        const float e = exp2f(w[h][q] - M);
        Ls = fmaf(wl[h][q], e, Ls);
        w[h][q] = e;
      }
      const float inv = 1.f / Ls;
      for (int32_t q = 0; q < nparts; ++q) w[h][q] *= inv;
    }
    __syncthreads();
    for (int32_t i0 = threadIdx.x; i0 < G * D; i0 += kOut * blockDim.x) {
      float sum[kOut];
#pragma unroll
      for (int o = 0; o < kOut; ++o) sum[o] = 0.f;
      for (int32_t q0 = 0; q0 < nparts; q0 += kChunk) {
        float a[kOut][kChunk];
#pragma unroll
        for (int o = 0; o < kOut; ++o) {
          const int32_t i = i0 + o * blockDim.x;
          const float* acc = p.ws_acc + (bh0 + i / D) * p.max_partitions * D + (i % D);
#pragma unroll
          for (int j = 0; j < kChunk; ++j)
            a[o][j] = (i < G * D && q0 + j < nparts) ? __ldcg(acc + (size_t)(q0 + j) * D) : 0.f;
        }
#pragma unroll
        for (int o = 0; o < kOut; ++o) {
          const int32_t h = (i0 + o * blockDim.x) / D;
#pragma unroll
          for (int j = 0; j < kChunk; ++j)
            if (q0 + j < nparts && h < G) sum[o] = fmaf(a[o][j], w[h][q0 + j], sum[o]);
        }
      }
#pragma unroll
      for (int o = 0; o < kOut; ++o) {
        const int32_t i = i0 + o * blockDim.x;
        if (i < G * D) reinterpret_cast<T*>(p.out)[(bh0 + i / D) * D + (i % D)] = Elem<T>::from_f32(sum[o]);
      }
    }
    return;
  }
  // more than kMergeMaxParts partitions: plain per-element merge
  for (int32_t i = threadIdx.x; i < G * D; i += blockDim.x) {
    const int32_t h = i / D;
    const int32_t d = i % D;
    const float* ml = p.ws_ml + (bh0 + h) * p.max_partitions * 2;
    const float* acc = p.ws_acc + (bh0 + h) * p.max_partitions * D + d;
    float M = -INFINITY;
    for (int32_t q = 0; q < nparts; ++q) M = fmaxf(M, __ldcg(ml + 2 * q));
    float Ls = 0.f, A = 0.f;
    for (int32_t q = 0; q < nparts; ++q) {
      const float e = exp2f(__ldcg(ml + 2 * q) - M);
      Ls = fmaf(__ldcg(ml + 2 * q + 1), e, Ls);
      A = fmaf(__ldcg(acc + (size_t)q * D), e, A);
    }
    reinterpret_cast<T*>(p.out)[(bh0 + h) * D + d] = Elem<T>::from_f32(A / Ls);
  }
}

// Launches partition_merge_kernel as a programmatic dependent of the kernel
// just launched on `st` (which calls griddepcontrol.launch_dependents).
template <typename T, int D>
inline cudaError_t launch_partition_merge(const DecodeParams& p, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.num_kv_heads, p.num_seqs);
  cfg.blockDim = dim3(kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, partition_merge_kernel<T, D>, p);
}

}  // namespace pagedkv
