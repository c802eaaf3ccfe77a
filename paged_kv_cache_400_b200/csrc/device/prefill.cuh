// Paged prefill / chunked-prefill attention for bf16 pools with head_dim 128.
//
// Prefill processes a request's whole prompt, decode one token per step
// ("大模型推理性能优化：PagedAttention与Continuous Batching原理与实践" §2); a prompt may
// also arrive in chunks after earlier KV is cached. Sequence b holds L tokens
// of KV; its n newest tokens are queries at positions L-n .. L-1, and the
// query at position P attends to positions 0..P through the block table.
//
// CTA = (query tile, KV head g, sequence b): a tile is 64 rows of
// (query token, query head of g's group), 64/G tokens x G heads. Unlike decode,
// every warp needs every KV block, so one producer warp stages blocks (the same
// TMA boxes and 128-byte swizzle as the decode kernel) into a 4-deep ring with
// a full and an empty mbarrier per stage, and four consumer warps, 16 rows
// each, run S = Q K^T and O += P V on mma.sync m16n8k16 with an online softmax
// in registers (log2 domain, fp32). Blocks past the tile's last query position
// are never loaded; the diagonal blocks are masked per element. Each warp owns
// its rows end to end, so the output is written straight from registers. All
// waits give up after 2 s and raise PA_DEVERR_TIMEOUT.
#pragma once

#include "decode_staged.cuh"
#include "prefill_common.cuh"

namespace pagedkv {

constexpr int kPrefillConsumers = 4;
constexpr int kPrefillStages = 4;
constexpr int kPrefillThreads = (kPrefillConsumers + 1) * 32;
constexpr int kPrefillSmem = kPrefillStages * kStageBytes + 1024;

__global__ void __launch_bounds__(kPrefillThreads) prefill_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                  PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kPrefillStages];
  __shared__ __align__(8) uint64_t empty[kPrefillStages];
  __shared__ int32_t stage_ok[kPrefillStages];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int32_t tile = gridDim.x - 1 - blockIdx.x;  // the longest (last) tiles start first
  const int32_t g = blockIdx.y;
  const int32_t b = blockIdx.z;
  const int32_t warp = threadIdx.x >> 5;
  const int32_t lane = threadIdx.x & 31;
  const int32_t G = p.group;
  const int32_t H = p.num_heads;
  const int32_t QT = p.tile_tokens;

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
  const int32_t tok_end = min(n, tok_begin + QT);
  const int32_t ctx = L - n;                    // cached tokens before the new ones
  const int32_t last_pos = ctx + tok_end - 1;   // the tile's last query position
  const int32_t nblocks = last_pos / 16 + 1;
  const int32_t* table = p.block_tables + (size_t)b * p.max_blocks;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < kPrefillStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kPrefillConsumers);
    }
    fence_barrier_init();
    prefetch_tensormap(&tmap);
  }
  __syncthreads();

  // ---- producer warp: stage blocks 0 .. nblocks-1 ------------------------------
  if (warp == kPrefillConsumers) {
    if (lane == 0) {
      for (int32_t j = 0; j < nblocks; ++j) {
        const int32_t s = j % kPrefillStages;
        if (j >= kPrefillStages &&
            !mbar_wait_bounded(&empty[s], (uint32_t)(j / kPrefillStages - 1) & 1u, kWaitLimitNs)) {
          raise_device_error(PA_DEVERR_TIMEOUT);
          break;
        }
        const int32_t blk = __ldg(table + j);
        if (blk >= 0 && blk < p.num_blocks) {
          stage_ok[s] = 1;
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          tma_load_5d(smem + s * kStageBytes, &tmap, &full[s], 0, 0, g, 0, blk);
          tma_load_5d(smem + s * kStageBytes + 4096, &tmap, &full[s], 64, 0, g, 0, blk);
        } else {
          raise_device_error(PA_DEVERR_BLOCK);
          stage_ok[s] = 0;
          mbar_arrive(&full[s]);
        }
      }
    }
    return;
  }

  // ---- consumer warps: 16 rows each -----------------------------------------
  const int32_t gid = lane >> 2;
  const int32_t tig = lane & 3;
  const int32_t r0 = 16 * warp + gid, r1 = r0 + 8;
  const int32_t tok0 = tok_begin + r0 / G, tok1 = tok_begin + r1 / G;
  const int32_t h0 = r0 % G, h1 = r1 % G;
  const bool v0 = tok0 < tok_end, v1 = tok1 < tok_end;
  // a padding row attends to position 0 only (finite) and is not written
  const int32_t P0 = v0 ? ctx + tok0 : 0;
  const int32_t P1 = v1 ? ctx + tok1 : 0;
  const int32_t pmin = min(v0 ? P0 : last_pos, v1 ? P1 : last_pos);

  uint32_t qa[8][4];
  {
    const uint32_t* qw = reinterpret_cast<const uint32_t*>(p.q);
    const size_t row0 = ((size_t)(q0 + tok0) * H + (size_t)g * G + h0) * 64;
    const size_t row1 = ((size_t)(q0 + tok1) * H + (size_t)g * G + h1) * 64;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int32_t lo = (16 * kk + 2 * tig) >> 1;
      qa[kk][0] = v0 ? __ldg(qw + row0 + lo) : 0u;
      qa[kk][1] = v1 ? __ldg(qw + row1 + lo) : 0u;
      qa[kk][2] = v0 ? __ldg(qw + row0 + lo + 4) : 0u;
      qa[kk][3] = v1 ? __ldg(qw + row1 + lo + 4) : 0u;
    }
  }
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const uint32_t base = smem_addr(smem);

  for (int32_t j = 0; j < nblocks; ++j) {
    const int32_t s = j % kPrefillStages;
    const bool arrived = mbar_wait_bounded(&full[s], (uint32_t)(j / kPrefillStages) & 1u, kWaitLimitNs);
    if (__any_sync(0xffffffffu, !arrived)) {
      if (lane == 0) raise_device_error(PA_DEVERR_TIMEOUT);
      break;  // the output of this tile is then undefined
    }
    const bool ok = stage_ok[s] != 0;
    const uint32_t st = base + s * kStageBytes;
    const int32_t kv0 = 16 * j;
    if (ok && kv0 + 16 > L) {
      // V rows past the sequence end (last block only): zeroed before use
      for (int32_t e = lane; e < (kv0 + 16 - L) * 16; e += 32) {
        const int32_t row = (L - kv0) + (e >> 4);
        *reinterpret_cast<uint4*>(smem + s * kStageBytes + tile_chunk(1, row, e & 15)) = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    if (ok) {
      const int32_t tok = (lane & 7) + ((lane >> 4) << 3);
      const int32_t half = (lane >> 3) & 1;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(st + tile_chunk(0, tok, 2 * kk + half), a0, a1, a2, a3);
        mma_bf16_16816(sc[0], qa[kk], a0, a1);
        mma_bf16_16816(sc[1], qa[kk], a2, a3);
      }
    }
    const bool diag = kv0 + 15 > pmin;  // some element of this warp is causally masked
    float bm0 = -INFINITY, bm1 = -INFINITY;
#pragma unroll
    for (int nn = 0; nn < 2; ++nn) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int32_t t = kv0 + 8 * nn + 2 * tig + (e & 1);
        float x = sc[nn][e] * p.scale_log2;
        if (diag) x = t <= (e < 2 ? P0 : P1) ? x : -INFINITY;
        sc[nn][e] = x;
        if (e < 2) bm0 = fmaxf(bm0, x);
        else bm1 = fmaxf(bm1, x);
      }
    }
    bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, 1));
    bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, 2));
    bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, 1));
    bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, 2));
    // a row whose every key in this block is masked keeps its state
    const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
    const float a0 = mn0 == -INFINITY ? 1.f : exp2f(m0 - mn0);
    const float a1 = mn1 == -INFINITY ? 1.f : exp2f(m1 - mn1);
    float pr[2][4];
#pragma unroll
    for (int nn = 0; nn < 2; ++nn) {
      pr[nn][0] = mn0 == -INFINITY ? 0.f : exp2f(sc[nn][0] - mn0);
      pr[nn][1] = mn0 == -INFINITY ? 0.f : exp2f(sc[nn][1] - mn0);
      pr[nn][2] = mn1 == -INFINITY ? 0.f : exp2f(sc[nn][2] - mn1);
      pr[nn][3] = mn1 == -INFINITY ? 0.f : exp2f(sc[nn][3] - mn1);
    }
    m0 = mn0;
    m1 = mn1;
    l0 = l0 * a0 + ((pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]));
    l1 = l1 * a1 + ((pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]));
    if (__any_sync(0xffffffffu, a0 != 1.f || a1 != 1.f)) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        o[i][0] *= a0;
        o[i][1] *= a0;
        o[i][2] *= a1;
        o[i][3] *= a1;
      }
    }
    if (ok) {
      const uint32_t pa[4] = {pack_bf16x2(pr[0][0], pr[0][1]), pack_bf16x2(pr[0][2], pr[0][3]),
                              pack_bf16x2(pr[1][0], pr[1][1]), pack_bf16x2(pr[1][2], pr[1][3])};
      const int32_t tok = (lane & 7) + (((lane >> 3) & 1) << 3);
      const int32_t half = lane >> 4;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(st + tile_chunk(1, tok, 2 * jj + half), b0, b1, b2, b3);
        mma_bf16_16816(o[2 * jj], pa, b0, b1);
        mma_bf16_16816(o[2 * jj + 1], pa, b2, b3);
      }
    }
    // the zeroed rows were written by the generic proxy; order them before the
    // next TMA write of this stage
    if (ok && kv0 + 16 > L) fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = 1.f / l0, inv1 = 1.f / l1;
  uint32_t* ow = reinterpret_cast<uint32_t*>(p.out);
  const size_t orow0 = ((size_t)(q0 + tok0) * H + (size_t)g * G + h0) * 64;
  const size_t orow1 = ((size_t)(q0 + tok1) * H + (size_t)g * G + h1) * 64;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int32_t w = (8 * i + 2 * tig) >> 1;
    if (v0) ow[orow0 + w] = pack_bf16x2(o[i][0] * inv0, o[i][1] * inv0);
    if (v1) ow[orow1 + w] = pack_bf16x2(o[i][2] * inv1, o[i][3] * inv1);
  }
}

inline pa_status launch_prefill_bf16_d128(const void* pool, int32_t num_blocks, const PrefillParams& p,
                                          int32_t num_seqs, cudaStream_t st) {
  CUtensorMap map;
  pa_status s = encode_pool_map(pool, p.num_kv_heads, num_blocks, &map);
  if (s != PA_OK) return s;
  static PerDevice<int32_t> smem_set;
  cudaError_t attr = set_smem_once(smem_set, prefill_kernel, kPrefillSmem);
  if (attr != cudaSuccess) return fail(PA_ERR_CUDA, "pa_prefill: %s", cudaGetErrorString(attr));
  dim3 grid((p.max_query_len + p.tile_tokens - 1) / p.tile_tokens, p.num_kv_heads, num_seqs);
  prefill_kernel<<<grid, kPrefillThreads, kPrefillSmem, st>>>(map, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_prefill: launch failed: %s", cudaGetErrorString(e));
  return PA_OK;
}

}  // namespace pagedkv
