// Paged prefill / chunked-prefill attention on the 5th-generation tensor core
// (tcgen05 MMA, accumulators in tensor memory), bf16 pools with head_dim 128.
//
// Same operation as prefill_kernel: sequence b holds L tokens of KV, its n
// newest are queries at positions L-n .. L-1, the query at position P attends
// causally to positions 0..P through the block table ("大模型推理性能优化：
// PagedAttention与Continuous Batching原理与实践" §2: prefill runs the whole prompt;
// §2.2: KV is gathered from fixed 16-token pages through the page table).
//
// CTA = (unit of two 128-row query tiles, KV head g, sequence b); a row is
// (query token, query head of g's group): each tile is 128/G tokens x G heads,
// so one staged KV tile serves every head of the group and both tiles (twice
// the MMA work per staged byte). 384 threads in four roles:
//   warps 0-3, 4-7  softmax, one warp group per query tile: thread r owns row
//              r of its tile = tensor-memory lane r;
//   warps 8-9  producers: both Q tiles by TMA once (warp 8), then KV tiles of
//              64 keys (four 16-token blocks gathered through the table, one
//              TMA box per block and K|V and head-dim half) into a 4-stage
//              ring; each warp stages two of the four blocks, its 8 boxes
//              issued by 8 lanes at once (two warps issue boxes about 1.5x as
//              fast as one);
//   warps 10-11 MMA issuers (one thread each), one per query tile: S = Q K^T
//              into tensor memory, then O += P V with P read back from tensor
//              memory; the two tiles' MMA chains overlap on the tensor core.
// Tensor memory (512 columns, so one CTA per SM): per tile t at 256 t, O
// [0,128) fp32 and two S buffers [128,192), [192,256) fp32, each overwritten in
// place by its P as packed bf16 pairs. Issue order per tile S_0, S_1, PV_0,
// S_2, PV_1, ... (S_{j+1} after PV_j instead when its K/V tile is not in yet),
// the two tiles interleaved, so the tensor core works on one tile while the
// other's softmax runs. The running max is only raised when a
// tile's max exceeds it by more than 2^8 (log2 domain), so O in tensor memory
// is rescaled rarely; O and the row sum l always share the same reference max,
// so the final O / l is exact up to rounding.
// Shared memory: Q 2 x 32 KB + 4 x 32 KB KV stages (K and V halves 8 KB each,
// 128-byte swizzle, the canonical K-major / MN-major UMMA layouts).
// A one-tile variant (192 threads, 2-stage ring, two CTAs per SM) is kept for
// comparison; it is compiled only into a comparison build (PA_PREFILL_QTILES=1).
// Every wait gives up after 2 s (PA_DEVERR_TIMEOUT); the CTA still frees its
// tensor memory before it exits. Phase tracking: every mbarrier is waited on at
// most one completion ahead of the last one its waiter consumed (S and P
// buffers alternate, PV completions alternate between two barriers), so a
// parity wait is never ambiguous.
#pragma once

#include "decode_staged.cuh"
#include "prefill_common.cuh"
#include "tcgen05.cuh"

namespace pagedkv {

constexpr int kTcKeys = 64;                       // keys per KV tile
constexpr int kTcBlocksPerTile = kTcKeys / 16;
constexpr int kTcHalfBytes = kTcKeys * 128;       // 64 keys x 64 dims x bf16
constexpr int kTcStageBytes = 4 * kTcHalfBytes;   // K lo, K hi, V lo, V hi
constexpr int kTcQBytes = 128 * 256;              // one 128-row query tile x 128 dims x bf16
constexpr float kTcRescaleLog2 = 8.0f;            // raise the reference max past this growth

// kQTiles query tiles of 128 rows share every staged KV tile. Two tiles: one
// CTA per SM (all 512 tensor-memory columns, 193 KB of shared memory), a
// 4-deep KV ring; one tile: two CTAs per SM, a 2-deep ring.
#ifndef PA_PREFILL_QTILES
#define PA_PREFILL_QTILES 2
#endif
static_assert(PA_PREFILL_QTILES == 1 || PA_PREFILL_QTILES == 2, "one or two query tiles per CTA");

template <int kQTiles>
struct TcConfig {
  static constexpr int kStages = kQTiles == 2 ? 4 : 2;
  static constexpr int kProducers = 2;              // producer warps, each stages half of every KV tile
  static constexpr int kThreads = kQTiles * 128 + kProducers * 32 + kQTiles * 32;
  static constexpr int kProducerWarp = kQTiles * 4;  // first producer warp
  static constexpr int kMmaWarp = kQTiles * 4 + kProducers;  // first of kQTiles issuer warps, one per tile
  static constexpr uint32_t kTmemCols = kQTiles * 256;
  static constexpr int kSmem = kQTiles * kTcQBytes + kStages * kTcStageBytes + 1024;
};

template <int kQTiles, int kStages>
struct PrefillTcShared {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[kQTiles][2];   // S_j of tile t ready: s_full[t][j & 1]
  uint64_t p_full[kQTiles][2];   // P_j of tile t written (one arrival per softmax warp)
  uint64_t pv_done[kQTiles][2];  // PV_j of tile t complete: pv_done[t][j & 1]
  uint32_t tmem_base;
};

// 2^x on the special-function unit (approximate, flushes results below 2^-126
// to zero).
__device__ __forceinline__ float ex2_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Region offsets inside a stage.
__device__ __forceinline__ uint32_t tc_region(int kv, int half) { return (uint32_t)((kv * 2 + half) * kTcHalfBytes); }

template <int kQTiles>
__global__ void __launch_bounds__(TcConfig<kQTiles>::kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap pool_map, const __grid_constant__ CUtensorMap q_map,
                      PrefillParams p, const uint4* __restrict__ pool) {
  using Cfg = TcConfig<kQTiles>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ PrefillTcShared<kQTiles, S> sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = smem;
  uint8_t* kv_smem = smem + kQTiles * kTcQBytes;

  const int32_t G = p.group;
  const int32_t QT = 128 / G;                       // tokens per 128-row tile
  const int32_t unit = gridDim.x - 1 - blockIdx.x;  // the longest (last) units start first
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
    if (unit == 0 && g == 0 && threadIdx.x == 0) raise_device_error(PA_DEVERR_SEQLEN);
    return;
  }
  const int32_t tok_begin = unit * kQTiles * QT;
  if (tok_begin >= n) return;
  // after a timed-out wait anywhere in the grid, CTAs that start later skip
  // their work (the error stays set until the host reads it)
  if (*reinterpret_cast<volatile unsigned int*>(&g_error_word) & PA_DEVERR_TIMEOUT) return;
  const int32_t ctx = L - n;
  // KV tiles each query tile needs (0 for a tile past the sequence's new tokens)
  int32_t nt[kQTiles];
#pragma unroll
  for (int t = 0; t < kQTiles; ++t) {
    const int32_t tb = tok_begin + t * QT;
    nt[t] = tb < n ? ((ctx + min(n, tb + QT) - 1) / 16 + kTcBlocksPerTile) / kTcBlocksPerTile : 0;
  }
  const int32_t nblocks = (ctx + min(n, tok_begin + kQTiles * QT) - 1) / 16 + 1;
  const int32_t nt_max = (nblocks + kTcBlocksPerTile - 1) / kTcBlocksPerTile;
  const int32_t* table = p.block_tables + (size_t)b * p.max_blocks;

  // The producer warp sets up the mbarriers and starts loading at once; the
  // other warps wait on named barrier 1 (which the producer only arrives at)
  // and the MMA warp allocates tensor memory meanwhile.
  if (warp == Cfg::kProducerWarp && lane == 0) {
    mbar_init(&sh.q_full, 1);
#pragma unroll
    for (int s = 0; s < S; ++s) {
      mbar_init(&sh.kv_full[s], Cfg::kProducers);  // one arrival (with its bytes) per producer warp
      mbar_init(&sh.kv_empty[s], kQTiles);         // one release per issuer
    }
#pragma unroll
    for (int t = 0; t < kQTiles; ++t)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        mbar_init(&sh.s_full[t][i], 1);
        mbar_init(&sh.p_full[t][i], 4);  // one arrival per softmax warp
        mbar_init(&sh.pv_done[t][i], 1);
      }
    fence_barrier_init();
    prefetch_tensormap(&pool_map);
    prefetch_tensormap(&q_map);
  }
  if (warp == Cfg::kMmaWarp) {
    tmem_alloc(&sh.tmem_base, Cfg::kTmemCols);
    tmem_relinquish();
  }
  if (warp == Cfg::kProducerWarp) {
    // the first producer warp initialised the barriers: it only arrives (the
    // second producer warp waits here like the rest)
    __syncwarp();
    named_barrier_arrive(1, Cfg::kThreads);
  } else {
    tc_fence_before_sync();
    named_barrier_sync(1, Cfg::kThreads);
    tc_fence_after_sync();
  }
  const uint32_t tmem = sh.tmem_base;  // read by the MMA and softmax warps only

  if (warp >= Cfg::kProducerWarp && warp < Cfg::kMmaWarp) {
    // ---- producers: warp pw stages blocks 2 pw, 2 pw + 1 of every 64-key tile --------
    const int32_t pw = warp - Cfg::kProducerWarp;
    if (pw == 0 && lane == 0) {
      mbar_arrive_expect_tx(&sh.q_full, kQTiles * kTcQBytes);
#pragma unroll
      for (int t = 0; t < kQTiles; ++t) {
        tma_load_3d(q_smem + t * kTcQBytes, &q_map, &sh.q_full, 0, g * G, q0 + tok_begin + t * QT);
        tma_load_3d(q_smem + t * kTcQBytes + kTcQBytes / 2, &q_map, &sh.q_full, 64, g * G, q0 + tok_begin + t * QT);
      }
    }
    // block ids in batches of 32 (8 KV tiles), lane l holding entry l of its
    // batch; the next batch is in flight while the current one is staged
    constexpr int32_t kTilesPerBatch = 32 / kTcBlocksPerTile;
    auto load_batch = [&](int32_t k) -> int32_t {
      const int32_t bi = k * 32 + lane;
      return bi < nblocks ? __ldg(table + bi) : -1;
    };
    int32_t ids = load_batch(0);
    int32_t ids_next = load_batch(1);
    for (int32_t j = 0; j < nt_max; ++j) {
      if (j > 0 && j % kTilesPerBatch == 0) {
        ids = ids_next;
        ids_next = load_batch(j / kTilesPerBatch + 1);
      }
      const int32_t first = (j % kTilesPerBatch) * kTcBlocksPerTile;  // this tile's entries in the batch
      const int32_t s = j % S;
      if (j >= S) {
        const bool ok = mbar_wait_bounded(&sh.kv_empty[s], (uint32_t)(j / S - 1) & 1u, kWaitLimitNs);
        if (__any_sync(0xffffffffu, !ok)) {
          if (lane == 0) raise_device_error(PA_DEVERR_TIMEOUT);
          break;
        }
      }
      uint8_t* st = kv_smem + s * kTcStageBytes;
      // TMA fills whole blocks inside the sequence; the warp writes the
      // sequence's partial last block row by row (rows past L zeroed) and zeros
      // for slots past the last block or with a bad id.
      constexpr int32_t kMine = kTcBlocksPerTile / Cfg::kProducers;  // block slots of this warp
      int32_t blk[kMine];
      uint32_t tma_mask = 0;
#pragma unroll
      for (int32_t m = 0; m < kMine; ++m) {
        const int32_t i = pw * kMine + m;  // block slot in the tile
        const int32_t bi = j * kTcBlocksPerTile + i;
        blk[m] = __shfl_sync(0xffffffffu, ids, first + i);
        if (bi < nblocks && (blk[m] < 0 || blk[m] >= p.num_blocks)) {
          if (lane == 0) raise_device_error(PA_DEVERR_BLOCK);
          blk[m] = -1;
        }
        const int32_t rows = (bi < nblocks && blk[m] >= 0) ? min(16, L - bi * 16) : 0;
        if (rows == 16) {
          tma_mask |= 1u << m;
          continue;
        }
        // 16 rows x 16 chunks of 16 bytes, K and V: 512 chunks over the warp
        for (int32_t e = lane; e < 512; e += 32) {
          const int32_t kv = e >> 8;
          const int32_t row = (e >> 4) & 15;
          const int32_t c = e & 15;  // 16-byte chunk of the 256-byte row
          uint4 val = make_uint4(0, 0, 0, 0);
          if (row < rows)
            val = __ldg(pool + ((((size_t)blk[m] * 2 + kv) * p.num_kv_heads + g) * 16 + row) * 16 + c);
          const int32_t key = i * 16 + row;
          *reinterpret_cast<uint4*>(st + tc_region(kv, c >> 3) + key * 128 + (((c & 7) ^ (key & 7)) << 4)) = val;
        }
      }
      if (tma_mask != (1u << kMine) - 1) fence_proxy_async_smem();  // the warp wrote slots
      __syncwarp();
      if (lane == 0) {
        const uint32_t bytes = (uint32_t)__popc(tma_mask) * 4u * 2048u;
        if (bytes) mbar_arrive_expect_tx(&sh.kv_full[s], bytes);
        else mbar_arrive(&sh.kv_full[s]);
      }
      __syncwarp();
      // one TMA box per lane: lane = 4 x (this warp's block m) + 2 x (K|V) + head-dim half
      const int32_t slot = pw * kMine + ((lane >> 2) & (kMine - 1));
      const int32_t my_blk = __shfl_sync(0xffffffffu, ids, first + slot);
      if (lane < 4 * kMine && ((tma_mask >> (lane >> 2)) & 1u)) {
        const int kv = (lane >> 1) & 1;
        const int half = lane & 1;
        tma_load_5d(st + tc_region(kv, half) + slot * 2048, &pool_map, &sh.kv_full[s], 64 * half, 0, g, kv,
                    my_blk);
      }
    }
  } else if (warp >= Cfg::kMmaWarp) {
    // ---- MMA issuers: warp kMmaWarp + t, one thread, drives query tile t -------------
    const int t = warp - Cfg::kMmaWarp;
    const int32_t ntt = (kQTiles == 1 || t == 0) ? nt[0] : nt[kQTiles - 1];
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc_idesc_bf16(128, kTcKeys, false);
      constexpr uint32_t idesc_pv = tc_idesc_bf16(128, 128, true);
      const uint32_t qa = smem_addr(q_smem) + t * kTcQBytes;
      const uint32_t kv_addr = smem_addr(kv_smem);
      const uint32_t tm = tmem + t * 256;
      bool ok = mbar_wait_bounded(&sh.q_full, 0, kWaitLimitNs);
      int32_t kv_ready = -1;  // KV tiles 0 .. kv_ready have been waited for, in order
      auto ensure_kv = [&](int32_t j) {
        for (int32_t i = kv_ready + 1; i <= j && ok; ++i)
          ok = mbar_wait_bounded(&sh.kv_full[i % S], (uint32_t)(i / S) & 1u, kWaitLimitNs);
        kv_ready = j;
      };
      // S_j = Q_t K_j^T: eight k-steps of 16 dims (32 bytes inside the swizzled
      // 128-byte rows; dims 64..127 in the second half region).
      auto issue_s = [&](int32_t j) {
        ensure_kv(j);
        if (!ok) return;
        tc_fence_after_sync();
        const uint32_t kaddr = kv_addr + (j % S) * kTcStageBytes;
        const uint32_t d = tm + 128 + 64 * (j & 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * (kTcQBytes / 2) + (kk & 3) * 32;
          const uint32_t koff = (kk >> 2) * kTcHalfBytes + (kk & 3) * 32;
          tc_mma_ss(d, tc_desc_sw128(qa + off, 16, 1024), tc_desc_sw128(kaddr + koff, 16, 1024), idesc_s,
                    kk > 0);
        }
        tc_commit(&sh.s_full[t][j & 1]);
      };
      if (ok && ntt > 0) issue_s(0);
      for (int32_t j = 0; j < nt_max && ok; ++j) {
        if (j < ntt) {
          // S_{j+1} goes ahead of PV_j when its K/V tile is already in;
          // otherwise PV_j is issued as soon as P_j is written and S_{j+1}
          // follows it, so a late K/V tile does not hold PV_j back
          bool s_next = false;
          if (j + 1 < ntt &&
              (kv_ready >= j + 1 || mbar_test_wait(&sh.kv_full[(j + 1) % S], (uint32_t)((j + 1) / S) & 1u))) {
            if (kv_ready < j + 1) kv_ready = j + 1;
            issue_s(j + 1);
            s_next = true;
          }
          ok = ok && mbar_wait_bounded(&sh.p_full[t][j & 1], (uint32_t)(j >> 1) & 1u, kWaitLimitNs);
          if (!ok) break;
          tc_fence_after_sync();
          // O_t += P_j V_j: four k-steps of 16 keys; V is MN-major (dims
          // contiguous), its two 64-dim halves one leading offset apart, 8-key
          // groups 1024 B apart.
          const uint32_t vaddr = kv_addr + (j % S) * kTcStageBytes + tc_region(1, 0);
          const uint32_t pa = tm + 128 + 64 * (j & 1);
#pragma unroll
          for (int kk = 0; kk < kTcKeys / 16; ++kk)
            tc_mma_ts(tm, pa + 8 * kk, tc_desc_sw128(vaddr + kk * 2048, kTcHalfBytes, 1024), idesc_pv,
                      (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&sh.pv_done[t][j & 1]);
          if (j + S < nt_max) tc_commit(&sh.kv_empty[j % S]);
          if (j + 1 < ntt && !s_next) issue_s(j + 1);
        } else if (j + S < nt_max) {
          // this tile never reads KV tile j; release it in order, after its load
          ensure_kv(j);
          if (ok) mbar_arrive(&sh.kv_empty[j % S]);
        }
      }
      if (!ok) raise_device_error(PA_DEVERR_TIMEOUT);
    }
  } else {
    // ---- softmax: warp group t, thread r owns row r of query tile t ----------------
    const int32_t t = warp >> 2;
    const int32_t r = threadIdx.x - 128 * t;
    const int32_t ntt = (kQTiles == 1 || t == 0) ? nt[0] : nt[kQTiles - 1];
    const int32_t tb = tok_begin + t * QT;
    const int32_t tok = tb + r / G;
    const int32_t h = r % G;
    const int32_t te = min(n, tb + QT);
    const bool valid = tok < te;
    const int32_t P = valid ? ctx + tok : ctx + te - 1;  // padding rows: any finite row
    const uint32_t lane_base = tmem + t * 256 + ((uint32_t)((warp & 3) * 32) << 16);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int32_t j = 0; j < ntt; ++j) {
      const bool arrived = mbar_wait_bounded(&sh.s_full[t][j & 1], (uint32_t)(j >> 1) & 1u, kWaitLimitNs);
      if (__any_sync(0xffffffffu, !arrived)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t sbuf = lane_base + 128 + 64 * (j & 1);
      uint32_t sr[64];
      tmem_ld64_wait(sbuf, sr);
      const int32_t key0 = j * kTcKeys;
      const bool diag = key0 + kTcKeys - 1 > P;
      if (diag) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (key0 + c > P) sr[c] = __float_as_uint(-INFINITY);
      }
      // tile max of the raw scores: three-input max, four independent chains
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < 32; ++c)
        m4[c & 3] = max3(m4[c & 3], __uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1]));
      float mt = max3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
      mt *= p.scale_log2;
      if (j == 0) {
        m_ref = mt;  // key 0 is never masked: finite
      } else {
        const bool need = mt > m_ref + kTcRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          // O holds PV_0 .. PV_{j-1}: wait for the last of them, then rescale
          const bool done =
              mbar_wait_bounded(&sh.pv_done[t][(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, kWaitLimitNs);
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
      // p = 2^(s * scale - m) on the special-function unit; the exponent
      // arguments and the row sum two columns per instruction
      const float2 scale2 = make_float2(p.scale_log2, p.scale_log2);
      const float2 neg_m2 = make_float2(-m_ref, -m_ref);
      uint32_t pw[32];
      float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float2 x =
            fma2(make_float2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), scale2, neg_m2);
        float p0 = ex2_sfu(x.x);
        float p1 = ex2_sfu(x.y);
        if (diag) {  // masked keys contribute exactly 0
          p0 = key0 + 2 * c <= P ? p0 : 0.f;
          p1 = key0 + 2 * c + 1 <= P ? p1 : 0.f;
        }
        sum2[c & 1] = add2(sum2[c & 1], make_float2(p0, p1));
        pw[c] = pack_bf16x2(p0, p1);
      }
      l += (sum2[0].x + sum2[1].x) + (sum2[0].y + sum2[1].y);
      tmem_st32(sbuf, pw);
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.p_full[t][j & 1]);
    }
    if (ok && ntt > 0) {
      const bool done =
          mbar_wait_bounded(&sh.pv_done[t][(ntt - 1) & 1], (uint32_t)((ntt - 1) >> 1) & 1u, kWaitLimitNs);
      ok = !__any_sync(0xffffffffu, !done);
      if (ok) {
        tc_fence_after_sync();
        const float inv = 1.f / l;
        uint4* orow =
            reinterpret_cast<uint4*>(p.out) + ((size_t)(q0 + tok) * p.num_heads + (size_t)g * G + h) * 16;
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
      }
    }
    if (!ok && lane == 0) raise_device_error(PA_DEVERR_TIMEOUT);
    tc_fence_before_sync();
  }

  __syncthreads();
  if (warp == Cfg::kMmaWarp) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, Cfg::kTmemCols);
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

template <int kQTiles>
inline pa_status launch_prefill_tc_variant(const CUtensorMap& pool_map, const CUtensorMap& q_map,
                                           const PrefillParams& p, const uint4* pool, int32_t num_seqs,
                                           cudaStream_t st) {
  using Cfg = TcConfig<kQTiles>;
  static PerDevice<int32_t> smem_set;
  cudaError_t attr = set_smem_once(smem_set, prefill_tc_kernel<kQTiles>, Cfg::kSmem);
  if (attr != cudaSuccess) return fail(PA_ERR_CUDA, "pa_prefill: %s", cudaGetErrorString(attr));
  const int32_t unit_tokens = kQTiles * (128 / p.group);
  dim3 grid((p.max_query_len + unit_tokens - 1) / unit_tokens, p.num_kv_heads, num_seqs);
  prefill_tc_kernel<kQTiles><<<grid, Cfg::kThreads, Cfg::kSmem, st>>>(pool_map, q_map, p, pool);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_prefill: launch failed: %s", cudaGetErrorString(e));
  return PA_OK;
}

inline pa_status launch_prefill_tc(const void* pool, int32_t num_blocks, const PrefillParams& p, int32_t num_seqs,
                                   cudaStream_t st) {
  CUtensorMap pool_map, q_map;
  pa_status s = encode_pool_map(pool, p.num_kv_heads, num_blocks, &pool_map, 1);
  if (s != PA_OK) return s;
  s = encode_q_map(p.q, p.num_heads, p.num_tokens, p.group, &q_map);
  if (s != PA_OK) return s;
  const uint4* pool4 = reinterpret_cast<const uint4*>(pool);
  return launch_prefill_tc_variant<PA_PREFILL_QTILES>(pool_map, q_map, p, pool4, num_seqs, st);
}

}  // namespace pagedkv
