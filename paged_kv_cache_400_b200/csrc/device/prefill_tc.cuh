// Paged prefill / chunked-prefill attention on the 5th-generation tensor core
// (tcgen05 MMA, accumulators in tensor memory), bf16 pools with head_dim 128.
//
// Same operation as prefill_kernel: sequence b holds L tokens of KV, its n
// newest are queries at positions L-n .. L-1, the query at position P attends
// causally to positions 0..P through the block table ("大模型推理性能优化：
// PagedAttention与Continuous Batching原理与实践" §2: prefill runs the whole prompt;
// §2.2: KV is gathered from fixed 16-token pages through the page table).
//
// CTA = (128-row query tile, KV head g, sequence b); a row is (query token,
// query head of g's group): 128/G tokens x G heads, so one staged KV tile
// serves every head of the group. 192 threads in four roles:
//   warps 0-3  softmax: thread t owns row t = tensor-memory lane t;
//   warp 4     producer: Q tile by TMA once, then KV tiles of 64 keys (four
//              16-token blocks gathered through the table, one TMA box per
//              block and K|V and head-dim half) into a 2-stage ring;
//   warp 5     MMA issuer (one thread): S = Q K^T into tensor memory, then
//              O += P V with P read back from tensor memory.
// Tensor memory (256 columns): O [0,128) fp32; two S buffers [128,192) and
// [192,256) fp32, each overwritten in place by its P as packed bf16 pairs.
// Issue order S_0, S_1, PV_0, S_2, PV_1, ... lets the softmax of tile j run
// while S_{j+1} is computed. The running max is only raised when a tile's max
// exceeds it by more than 2^8 (log2 domain), so O in tensor memory is rescaled
// rarely; O and the row sum l always share the same reference max, so the
// final O / l is exact up to rounding.
// Shared memory: Q 32 KB + 2 x 32 KB KV stages (K and V halves 8 KB each,
// 128-byte swizzle, the canonical K-major / MN-major UMMA layouts), so two
// CTAs fit on an SM and their MMA and softmax phases interleave.
// Every wait gives up after 2 s (PA_DEVERR_TIMEOUT); the CTA still frees its
// tensor memory before it exits. Phase tracking: every mbarrier is waited on at
// most one completion ahead of the last one its waiter consumed (S and P
// buffers alternate, PV completions alternate between two barriers), so a
// parity wait is never ambiguous.
#pragma once

#include "decode_staged.cuh"
#include "tcgen05.cuh"

namespace pagedkv {

constexpr int kTcKeys = 64;                       // keys per KV tile
constexpr int kTcBlocksPerTile = kTcKeys / 16;
constexpr int kTcStages = 2;
constexpr int kTcHalfBytes = kTcKeys * 128;       // 64 keys x 64 dims x bf16
constexpr int kTcStageBytes = 4 * kTcHalfBytes;   // K lo, K hi, V lo, V hi
constexpr int kTcQBytes = 128 * 256;              // 128 rows x 128 dims x bf16
constexpr int kTcSmem = kTcQBytes + kTcStages * kTcStageBytes + 1024;
constexpr int kTcThreads = 192;
constexpr uint32_t kTcTmemCols = 256;
constexpr float kTcRescaleLog2 = 8.0f;            // raise the reference max past this growth

struct PrefillTcShared {
  uint64_t q_full;
  uint64_t kv_full[kTcStages];
  uint64_t kv_empty[kTcStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];  // PV_j completes pv_done[j & 1]
  uint32_t tmem_base;
};

// Region offsets inside a stage.
__device__ __forceinline__ uint32_t tc_region(int kv, int half) { return (uint32_t)((kv * 2 + half) * kTcHalfBytes); }

__global__ void __launch_bounds__(kTcThreads) prefill_tc_kernel(const __grid_constant__ CUtensorMap pool_map,
                                                                const __grid_constant__ CUtensorMap q_map,
                                                                PrefillParams p, const uint4* __restrict__ pool) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ PrefillTcShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = smem;
  uint8_t* kv_smem = smem + kTcQBytes;

  const int32_t G = p.group;
  const int32_t QT = 128 / G;
  const int32_t tile = gridDim.x - 1 - blockIdx.x;  // the longest (last) tiles start first
  const int32_t g = blockIdx.y;
  const int32_t b = blockIdx.z;
  const int32_t warp = threadIdx.x >> 5;
  const int32_t lane = threadIdx.x & 31;

  const int32_t q0 = __ldg(p.query_start + b);
  const int32_t n = __ldg(p.query_start + b + 1) - q0;
  const int32_t L = __ldg(p.seq_lens + b);
  const bool bad = q0 < 0 || n < 0 || n > p.max_query_len || q0 + n > p.num_tokens || L < n ||
                   (int64_t)L > (int64_t)p.max_blocks * 16;
  if (bad) {
    if (tile == 0 && g == 0 && threadIdx.x == 0) raise_device_error(PA_DEVERR_SEQLEN);
    return;
  }
  const int32_t tok_begin = tile * QT;
  if (tok_begin >= n) return;
  // after a timed-out wait anywhere in the grid, CTAs that start later skip
  // their work (the error stays set until the host reads it)
  if (*reinterpret_cast<volatile unsigned int*>(&g_error_word) & PA_DEVERR_TIMEOUT) return;
  const int32_t tok_end = min(n, tok_begin + QT);
  const int32_t ctx = L - n;
  const int32_t last_pos = ctx + tok_end - 1;
  const int32_t nblocks = last_pos / 16 + 1;
  const int32_t ntiles = (nblocks + kTcBlocksPerTile - 1) / kTcBlocksPerTile;
  const int32_t* table = p.block_tables + (size_t)b * p.max_blocks;

  if (threadIdx.x == 0) {
    mbar_init(&sh.q_full, 1);
#pragma unroll
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&sh.kv_full[s], 1);
      mbar_init(&sh.kv_empty[s], 1);
    }
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sh.s_full[s], 1);
      mbar_init(&sh.p_full[s], 128);
    }
    mbar_init(&sh.pv_done[0], 1);
    mbar_init(&sh.pv_done[1], 1);
    fence_barrier_init();
    prefetch_tensormap(&pool_map);
    prefetch_tensormap(&q_map);
  }
  if (warp == 5) {
    tmem_alloc(&sh.tmem_base, kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 4) {
    // ---- producer ---------------------------------------------------------------
    if (lane == 0) {
      mbar_arrive_expect_tx(&sh.q_full, kTcQBytes);
      tma_load_3d(q_smem, &q_map, &sh.q_full, 0, g * G, q0 + tok_begin);
      tma_load_3d(q_smem + kTcQBytes / 2, &q_map, &sh.q_full, 64, g * G, q0 + tok_begin);
    }
    for (int32_t j = 0; j < ntiles; ++j) {
      const int32_t s = j % kTcStages;
      if (j >= kTcStages) {
        const bool ok = mbar_wait_bounded(&sh.kv_empty[s], (uint32_t)(j / kTcStages - 1) & 1u, kWaitLimitNs);
        if (__any_sync(0xffffffffu, !ok)) {
          if (lane == 0) raise_device_error(PA_DEVERR_TIMEOUT);
          break;
        }
      }
      uint8_t* st = kv_smem + s * kTcStageBytes;
      // Which slots TMA fills (whole blocks inside the sequence); the rest are
      // written here: the sequence's partial last block row by row (rows past
      // L zeroed) and slots past the tile's last block or with a bad id as zeros.
      uint32_t tma_mask = 0;
      for (int32_t i = 0; i < kTcBlocksPerTile; ++i) {
        const int32_t bi = j * kTcBlocksPerTile + i;
        int32_t blk = -1;
        if (bi < nblocks) {
          blk = __ldg(table + bi);
          if (blk < 0 || blk >= p.num_blocks) {
            if (lane == 0) raise_device_error(PA_DEVERR_BLOCK);
            blk = -1;
          }
        }
        const int32_t rows = blk < 0 ? 0 : min(16, L - bi * 16);
        if (rows == 16) {
          tma_mask |= 1u << i;
          continue;
        }
        // 16 rows x 16 chunks of 16 bytes, K and V: 512 chunks over the warp
        for (int32_t e = lane; e < 512; e += 32) {
          const int32_t kv = e >> 8;
          const int32_t row = (e >> 4) & 15;
          const int32_t c = e & 15;  // 16-byte chunk of the 256-byte row
          uint4 val = make_uint4(0, 0, 0, 0);
          if (row < rows)
            val = __ldg(pool + ((((size_t)blk * 2 + kv) * p.num_kv_heads + g) * 16 + row) * 16 + c);
          const int32_t key = i * 16 + row;
          *reinterpret_cast<uint4*>(st + tc_region(kv, c >> 3) + key * 128 + (((c & 7) ^ (key & 7)) << 4)) = val;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const uint32_t bytes = (uint32_t)__popc(tma_mask) * 4u * 2048u;
        if (bytes) mbar_arrive_expect_tx(&sh.kv_full[s], bytes);
        else mbar_arrive(&sh.kv_full[s]);
        for (int32_t i = 0; i < kTcBlocksPerTile; ++i) {
          if (!((tma_mask >> i) & 1u)) continue;
          const int32_t blk = __ldg(table + j * kTcBlocksPerTile + i);
#pragma unroll
          for (int kv = 0; kv < 2; ++kv)
#pragma unroll
            for (int half = 0; half < 2; ++half)
              tma_load_5d(st + tc_region(kv, half) + i * 2048, &pool_map, &sh.kv_full[s], 64 * half, 0, g, kv,
                          blk);
        }
      }
    }
  } else if (warp == 5) {
    // ---- MMA issuer ----------------------------------------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc_idesc_bf16(128, kTcKeys, false);
      constexpr uint32_t idesc_pv = tc_idesc_bf16(128, 128, true);
      const uint32_t q_addr = smem_addr(q_smem);
      const uint32_t kv_addr = smem_addr(kv_smem);
      bool ok = mbar_wait_bounded(&sh.q_full, 0, kWaitLimitNs);
      // S_j = Q K_j^T: eight k-steps of 16 dims (32 bytes inside the swizzled
      // 128-byte rows; dims 64..127 in the second half region).
      auto issue_s = [&](int32_t j) {
        const int32_t s = j % kTcStages;
        ok = ok && mbar_wait_bounded(&sh.kv_full[s], (uint32_t)(j / kTcStages) & 1u, kWaitLimitNs);
        if (!ok) return;
        tc_fence_after_sync();
        const uint32_t kaddr = kv_addr + s * kTcStageBytes;
        const uint32_t d = tmem + 128 + 64 * (j & 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * (kTcQBytes / 2) + (kk & 3) * 32;
          const uint32_t koff = (kk >> 2) * kTcHalfBytes + (kk & 3) * 32;
          tc_mma_ss(d, tc_desc_sw128(q_addr + off, 16, 1024), tc_desc_sw128(kaddr + koff, 16, 1024), idesc_s,
                    kk > 0);
        }
        tc_commit(&sh.s_full[j & 1]);
      };
      if (ok) issue_s(0);
      for (int32_t j = 0; j < ntiles && ok; ++j) {
        if (j + 1 < ntiles) issue_s(j + 1);
        ok = ok && mbar_wait_bounded(&sh.p_full[j & 1], (uint32_t)(j >> 1) & 1u, kWaitLimitNs);
        if (!ok) break;
        tc_fence_after_sync();
        // O += P_j V_j: four k-steps of 16 keys; V is MN-major (dims contiguous),
        // its two 64-dim halves one leading offset apart, 8-key groups 1024 B apart.
        const int32_t s = j % kTcStages;
        const uint32_t vaddr = kv_addr + s * kTcStageBytes + tc_region(1, 0);
        const uint32_t pa = tmem + 128 + 64 * (j & 1);
#pragma unroll
        for (int kk = 0; kk < kTcKeys / 16; ++kk)
          tc_mma_ts(tmem, pa + 8 * kk, tc_desc_sw128(vaddr + kk * 2048, kTcHalfBytes, 1024), idesc_pv,
                    (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&sh.pv_done[j & 1]);
        if (j + kTcStages < ntiles) tc_commit(&sh.kv_empty[s]);
      }
      if (!ok) raise_device_error(PA_DEVERR_TIMEOUT);
    }
  } else {
    // ---- softmax: thread t owns row t -------------------------------------------------
    const int32_t r = threadIdx.x;
    const int32_t tok = tok_begin + r / G;
    const int32_t h = r % G;
    const bool valid = tok < tok_end;
    const int32_t P = valid ? ctx + tok : last_pos;  // padding rows: any finite row
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int32_t j = 0; j < ntiles; ++j) {
      const bool arrived = mbar_wait_bounded(&sh.s_full[j & 1], (uint32_t)(j >> 1) & 1u, kWaitLimitNs);
      if (__any_sync(0xffffffffu, !arrived)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t sbuf = lane_base + 128 + 64 * (j & 1);
      uint32_t sr[2][32];
      tmem_ld32_wait(sbuf, sr[0]);
      tmem_ld32_wait(sbuf + 32, sr[1]);
      const int32_t key0 = j * kTcKeys;
      float x[64];
      float mt = -INFINITY;
      if (key0 + kTcKeys - 1 > P) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          x[c] = key0 + c <= P ? __uint_as_float(sr[c >> 5][c & 31]) * p.scale_log2 : -INFINITY;
          mt = fmaxf(mt, x[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          x[c] = __uint_as_float(sr[c >> 5][c & 31]) * p.scale_log2;
          mt = fmaxf(mt, x[c]);
        }
      }
      if (j == 0) {
        m_ref = mt;  // key 0 is never masked: finite
      } else {
        const bool need = mt > m_ref + kTcRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          // O holds PV_0 .. PV_{j-1}: wait for the last of them, then rescale
          const bool done =
              mbar_wait_bounded(&sh.pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, kWaitLimitNs);
          if (__any_sync(0xffffffffu, !done)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const float alpha = need ? exp2f(m_ref - mt) : 1.f;
          if (need) m_ref = mt;
          l *= alpha;
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t o[32];
            tmem_ld32_wait(lane_base + 32 * cc, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(lane_base + 32 * cc, o);
          }
        }
      }
      uint32_t pw[32];
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = exp2f(x[2 * c] - m_ref);
        const float p1 = exp2f(x[2 * c + 1] - m_ref);
        sum += p0 + p1;
        pw[c] = pack_bf16x2(p0, p1);
      }
      l += sum;
      tmem_st32(sbuf, pw);
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(&sh.p_full[j & 1]);
    }
    if (ok) {
      const bool done =
          mbar_wait_bounded(&sh.pv_done[(ntiles - 1) & 1], (uint32_t)((ntiles - 1) >> 1) & 1u, kWaitLimitNs);
      ok = !__any_sync(0xffffffffu, !done);
    }
    if (ok) {
      tc_fence_after_sync();
      const float inv = 1.f / l;
      uint4* orow = reinterpret_cast<uint4*>(p.out) + ((size_t)(q0 + tok) * p.num_heads + (size_t)g * G + h) * 16;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        tmem_ld32_wait(lane_base + 32 * cc, o);
        if (valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
            orow[4 * cc + v] = w;
          }
        }
      }
    } else if (lane == 0) {
      raise_device_error(PA_DEVERR_TIMEOUT);
    }
    tc_fence_before_sync();
  }

  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTcTmemCols);
  }
}

// Tensor map of q / out rows: (d 128, head H, token T), box (64, G, 128 / G),
// 128-byte swizzle, zero fill past the last token.
inline pa_status encode_q_map(const void* q, int32_t num_heads, int32_t num_tokens, int32_t group,
                              CUtensorMap* map) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[3] = {128, (cuuint64_t)num_heads, (cuuint64_t)num_tokens};
  const cuuint64_t strides[2] = {256, (cuuint64_t)num_heads * 256};
  const cuuint32_t box[3] = {64, (cuuint32_t)group, (cuuint32_t)(128 / group)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled (q) failed (%d)", (int)r);
  return PA_OK;
}

inline pa_status launch_prefill_tc(const void* pool, int32_t num_blocks, const PrefillParams& p, int32_t num_seqs,
                                   cudaStream_t st) {
  CUtensorMap pool_map, q_map;
  pa_status s = encode_pool_map(pool, p.num_kv_heads, num_blocks, &pool_map, 1);
  if (s != PA_OK) return s;
  s = encode_q_map(p.q, p.num_heads, p.num_tokens, p.group, &q_map);
  if (s != PA_OK) return s;
  static cudaError_t attr =
      cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem);
  if (attr != cudaSuccess) return fail(PA_ERR_CUDA, "pa_prefill: %s", cudaGetErrorString(attr));
  const int32_t qt = 128 / p.group;
  dim3 grid((p.max_query_len + qt - 1) / qt, p.num_kv_heads, num_seqs);
  prefill_tc_kernel<<<grid, kTcThreads, kTcSmem, st>>>(pool_map, q_map, p, reinterpret_cast<const uint4*>(pool));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_prefill: launch failed: %s", cudaGetErrorString(e));
  return PA_OK;
}

}  // namespace pagedkv
