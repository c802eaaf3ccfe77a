// Split-KV paged decode for bf16 pools with head_dim 128, blocks staged in
// shared memory by TMA.
//
// Gather ("大模型推理性能优化：PagedAttention与Continuous Batching原理与实践" §2.2: the
// page table locates the scattered 16-token pages at attention time): each
// (block, KV head) is two contiguous 4 KB tiles (K and V) in the pool. The pool
// is described to the TMA unit as a 5-D tensor
//     (d: 128, row: 16, kv_head: Hkv, k|v: 2, block: N)
// and one box of (64, 16, 1, 2, 1) brings K and V of half the head dims for all
// 16 rows (4 KB); two boxes fill a stage with the whole block (8 KB). The box
// rows are 128 bytes and use the 128-byte swizzle, so 8 consecutive tokens of
// one 16-byte column fall in 8 different bank groups: ldmatrix and 16-byte
// shared loads run without bank conflicts.
//
// Work unit = (partition, KV head g, sequence b), one CTA of 4 warps at a
// time. Without split partitions the grid has one CTA per unit; with them, a
// one-CTA plan kernel lists the non-empty units (full partitions first, then
// the sequences' last partitions by decreasing size) and a grid of resident
// CTAs takes units from that list through an atomic counter, so empty
// partitions cost nothing and the smallest units finish last. Warp w owns the
// partition's blocks w, w+4, w+8, ...; it runs its own ring of 2 stages with
// one mbarrier each, issuing the TMA for its next block as soon as a stage is
// consumed, so each warp keeps up to 16 KB in flight and a CTA 64 KB. Every
// warp keeps an online-softmax state (running max m, partial sum l, output
// accumulator) in the log2 domain; the four states are merged through shared
// memory at the end and either written out (one partition) or stored as a
// partition state for the merge kernel (partition_merge_kernel, launched as a
// programmatic dependent so its launch overlaps this kernel's tail).
//
// Compute per block of 16 tokens:
//  * head group G >= 2 (GQA): the group's query heads are the M dimension of
//    mma.sync m16n8k16 tiles (rows >= G are zero padding). S = Q K^T takes 8
//    k-steps over head_dim with K fragments from ldmatrix; P = exp2(S - m) is
//    re-packed in registers as the A operand of O += P V with V fragments from
//    ldmatrix.trans. Scores, P and O never leave registers.
//  * G == 1 (MHA): CUDA cores. Two lanes per token form the dot product from
//    16-byte shared loads (one shuffle joins the halves); the block maximum
//    takes 4 shuffles; for P V each lane owns 8 head dims and half the tokens.
//
// Tokens past the sequence end inside its last block are masked to -inf, and
// their V rows are zeroed in shared memory first (unused pool rows may hold
// any bits). A block id outside the pool is never loaded: the stage is marked
// invalid (K and V read as zero) and PA_DEVERR_BLOCK is raised. Every mbarrier
// wait gives up after 2 s and raises PA_DEVERR_TIMEOUT instead of hanging; the
// warp then issues no further copy, waits (bounded) for the ones it has in
// flight, leaves its state out of the merge, and a persistent CTA takes no
// further item.
#pragma once

#include <cudaTypedefs.h>

#include <mutex>

#include "decode_common.cuh"
#include "ptx.cuh"

namespace pagedkv {

constexpr int kStagedWarps = 4;
constexpr int kStagedStages = 2;                 // per warp
constexpr int kStageBytes = 8192;                // K + V of one block, one KV head
constexpr int kStagedSmem = kStagedWarps * kStagedStages * kStageBytes + 1024;
constexpr int kMergeRow = 128 + 8;  // floats per row of the warps' merge buffer
static_assert(kStagedWarps * 16 * kMergeRow * 4 <= kStagedWarps * kStagedStages * kStageBytes,
              "the merge buffer reuses the consumed stages");
constexpr uint64_t kWaitLimitNs = 2000000000ull; // 2 s

// Byte offset in a stage of the 16-byte chunk `chunk16` (0..15, head dims
// 8*chunk16 .. +7) of row `token` of the K (kv = 0) or V (kv = 1) tile. A
// stage is [d half][K|V][16 rows][128 B] with the 128-byte swizzle applied to
// the 16-byte chunk index within each row.
__device__ __forceinline__ uint32_t tile_chunk(int kv, int token, int chunk16) {
  return (uint32_t)((chunk16 >> 3) * 4096 + kv * 2048 + token * 128 + (((chunk16 & 7) ^ (token & 7)) << 4));
}

// Shared-memory state of a decode CTA (static part; the stages are dynamic).
struct StagedShared {
  uint64_t bars[kStagedWarps][kStagedStages];
  float red_m[kStagedWarps][16];
  float red_l[kStagedWarps][16];
  int32_t next_item;
  int32_t abort;  // a warp of this CTA gave up on a stage: take no further items
};

// Attention over partition `part` of sequence b for KV head g (all G query
// heads). `phase` holds, per stage of this warp, the parity of its mbarrier's
// next phase; it carries over between partitions of a persistent CTA.
template <bool kMMA, bool kAppend>
__device__ __forceinline__ void decode_partition(const CUtensorMap& tmap, const DecodeParams& p, uint8_t* smem,
                                                 StagedShared& sh, int32_t part, int32_t g, int32_t b,
                                                 int32_t L, uint32_t& phase) {
  const int32_t warp = threadIdx.x >> 5;
  const int32_t lane = threadIdx.x & 31;
  const int32_t G = p.group;
  const int32_t H = p.num_heads;
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
  auto& bars = sh.bars;
  auto& red_m = sh.red_m;
  auto& red_l = sh.red_l;

  const int32_t S = p.partition_tokens;
  const int32_t nparts = (L + S - 1) / S;
  const int32_t t0 = part * S;
  const int32_t t1 = min(t0 + S, L);
  const int32_t nb = (t1 - t0 + 15) >> 4;
  const int32_t my = nb > warp ? (nb - warp + kStagedWarps - 1) / kStagedWarps : 0;
  uint8_t* wsm = smem + warp * kStagedStages * kStageBytes;
  const uint32_t wsm_addr = smem_addr(wsm);
  const int32_t* table = p.block_tables + (size_t)b * p.max_blocks + (t0 >> 4);

  // Block ids of this warp's blocks, read once: lane i holds the id of the
  // warp's i-th block (partition block warp + 4i), so issuing a load never
  // waits on a table read.
  const int32_t my_blk = lane < my ? __ldg(table + warp + lane * kStagedWarps) : -1;

  // Fused append: the warp that will stage the block holding position L-1
  // fetches the new token's K/V row (lanes 0-15: K chunks, 16-31: V chunks)
  // and slot now, so the loads overlap the pipeline.
  const bool app_here = kAppend && t1 == L && ((nb - 1) % kStagedWarps) == warp;
  const int32_t app_iter = (nb - 1) / kStagedWarps;
  uint4 app_val = make_uint4(0, 0, 0, 0);
  int64_t app_slot = -1;
  if (app_here) {
    app_slot = __ldg(p.slot_mapping + b);
    app_val = __ldg(reinterpret_cast<const uint4*>((lane >> 4) ? p.v_new : p.k_new) +
                    ((size_t)b * p.num_kv_heads + g) * 16 + (lane & 15));
  }

  uint32_t valid_mask = 0;  // bit s: stage s holds a real block
  auto issue = [&](int32_t i) {
    const int32_t s = i % kStagedStages;
    const int32_t blk = __shfl_sync(0xffffffffu, my_blk, i);
    int32_t ok = 0;
    if (lane == 0) {
      uint64_t* bar = &bars[warp][s];
      if (blk >= 0 && blk < p.num_blocks) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, kStageBytes);
        tma_load_5d(wsm + s * kStageBytes, &tmap, bar, 0, 0, g, 0, blk);
        tma_load_5d(wsm + s * kStageBytes + 4096, &tmap, bar, 64, 0, g, 0, blk);
        ok = 1;
      } else {
        raise_device_error(PA_DEVERR_BLOCK);
        mbar_arrive(bar);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    valid_mask = ok ? (valid_mask | (1u << s)) : (valid_mask & ~(1u << s));
  };

  const int32_t gid = lane >> 2;  // mma row group
  const int32_t tig = lane & 3;   // thread in group

  // first loads in flight before anything else is read
  const int32_t npre = my < kStagedStages ? my : kStagedStages;
  for (int32_t i = 0; i < npre; ++i) issue(i);

  // ---- per-warp softmax state ---------------------------------------------
  // MMA: rows gid and gid+8 of the 16-row head tile.
  uint32_t qa[8][4];
  float o[16][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  // CUDA cores (G == 1): one row.
  float qr[8][8];
  float acc[8];
  if constexpr (kMMA) {
    const uint32_t* qw = reinterpret_cast<const uint32_t*>(
        reinterpret_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * H + (size_t)g * G) * 128);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int32_t lo = (16 * kk + 2 * tig) >> 1;  // word index of d = 16kk + 2tig
      qa[kk][0] = gid < G ? __ldg(qw + gid * 64 + lo) : 0u;
      qa[kk][1] = gid + 8 < G ? __ldg(qw + (gid + 8) * 64 + lo) : 0u;
      qa[kk][2] = gid < G ? __ldg(qw + gid * 64 + lo + 4) : 0u;
      qa[kk][3] = gid + 8 < G ? __ldg(qw + (gid + 8) * 64 + lo + 4) : 0u;
    }
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  } else {
    // QK: lane -> token (lane >> 1), head-dim half (lane & 1); the half reads
    // its 8 chunks in an order offset by 4 so the two halves of a token hit
    // different bank groups.
    const int32_t hq = lane & 1;
    const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * H + g) * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int32_t d0 = 64 * hq + 8 * (c ^ (hq << 2));
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(q + d0));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        qr[c][2 * i] = bf16lo(ws[i]) * p.scale_log2;
        qr[c][2 * i + 1] = bf16hi(ws[i]) * p.scale_log2;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  }


  for (int32_t i = 0; i < my; ++i) {
    const int32_t s = i % kStagedStages;
    const bool arrived = mbar_wait_bounded(&bars[warp][s], (phase >> s) & 1u, kWaitLimitNs);
    if (__any_sync(0xffffffffu, !arrived)) {
      // Gave up on this stage: raise PA_DEVERR_TIMEOUT, issue nothing more,
      // wait (bounded) for the copies already issued into this warp's stages
      // (blocks i .. min(i + stages, my) - 1) so none lands after the CTA
      // leaves, and drop this warp's state from the merge. The sequence's
      // output is then undefined; the error word says so.
      if (lane == 0) raise_device_error(PA_DEVERR_TIMEOUT);
      const int32_t issued = min(i + kStagedStages, my);
      for (int32_t k = i; k < issued; ++k) {
        const int32_t sk = k % kStagedStages;
        mbar_wait_bounded(&bars[warp][sk], (phase >> sk) & 1u, kWaitLimitNs);
        phase ^= 1u << sk;
      }
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
      if constexpr (kMMA) {
#pragma unroll
        for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.f;
      }
      if (lane == 0) sh.abort = 1;
      break;
    }
    phase ^= 1u << s;
    const int32_t tok0 = t0 + (warp + i * kStagedWarps) * 16;
    const int32_t nvalid = min(16, t1 - tok0);
    const bool valid = (valid_mask >> s) & 1u;
    const uint32_t st = wsm_addr + s * kStageBytes;
    if (valid && nvalid < 16) {
      // zero V rows past the sequence end (both head-dim halves)
      for (int32_t e = lane; e < (16 - nvalid) * 16; e += 32) {
        const int32_t row = nvalid + (e >> 4);
        *reinterpret_cast<uint4*>(wsm + s * kStageBytes + tile_chunk(1, row, e & 15)) = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }
    if constexpr (kAppend) {
      // Fused cache append: this block holds position L-1, the step's new
      // token. Its K/V row (this KV head) is written into the staged block and
      // stored to the pool at the token's slot, which must be that position's
      // slot through the table; otherwise PA_DEVERR_SLOT and nothing is written.
      if (app_here && i == app_iter) {
        const int32_t blk = __shfl_sync(0xffffffffu, my_blk, i);
        const int32_t row = nvalid - 1;
        if (app_slot >= 0) {
          if (valid && app_slot == (int64_t)blk * 16 + row) {
            const int32_t kv = lane >> 4;
            const int32_t c = lane & 15;
            *reinterpret_cast<uint4*>(wsm + s * kStageBytes + tile_chunk(kv, row, c)) = app_val;
            uint4* pool = reinterpret_cast<uint4*>(const_cast<void*>(p.pool));
            pool[(((size_t)blk * 2 + kv) * p.num_kv_heads + g) * 256 + row * 16 + c] = app_val;
            __syncwarp();
          } else if (lane == 0) {
            raise_device_error(PA_DEVERR_SLOT);
          }
        }
      }
    }

    if constexpr (kMMA) {
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      if (valid) {
        const int32_t tok = (lane & 7) + ((lane >> 4) << 3);
        const int32_t half = (lane >> 3) & 1;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4(st + tile_chunk(0, tok, 2 * kk + half), r0, r1, r2, r3);
          mma_bf16_16816(sc[0], qa[kk], r0, r1);
          mma_bf16_16816(sc[1], qa[kk], r2, r3);
        }
      }
      float bm0 = -INFINITY, bm1 = -INFINITY;
#pragma unroll
      for (int n = 0; n < 2; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int32_t tok = 8 * n + 2 * tig + (e & 1);
          const float x = tok < nvalid ? sc[n][e] * p.scale_log2 : -INFINITY;
          sc[n][e] = x;
          if (e < 2) bm0 = fmaxf(bm0, x);
          else bm1 = fmaxf(bm1, x);
        }
      }
      bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, 1));
      bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, 2));
      bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, 1));
      bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, 2));
      const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
      const float a0 = exp2f(m0 - mn0), a1 = exp2f(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      float pr[2][4];
#pragma unroll
      for (int n = 0; n < 2; ++n) {
        pr[n][0] = exp2f(sc[n][0] - mn0);
        pr[n][1] = exp2f(sc[n][1] - mn0);
        pr[n][2] = exp2f(sc[n][2] - mn1);
        pr[n][3] = exp2f(sc[n][3] - mn1);
      }
      l0 = l0 * a0 + ((pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]));
      l1 = l1 * a1 + ((pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]));
      if (__any_sync(0xffffffffu, a0 != 1.f || a1 != 1.f)) {
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          o[n][0] *= a0;
          o[n][1] *= a0;
          o[n][2] *= a1;
          o[n][3] *= a1;
        }
      }
      if (valid) {
        const uint32_t pa[4] = {pack_bf16x2(pr[0][0], pr[0][1]), pack_bf16x2(pr[0][2], pr[0][3]),
                                pack_bf16x2(pr[1][0], pr[1][1]), pack_bf16x2(pr[1][2], pr[1][3])};
        const int32_t tok = (lane & 7) + (((lane >> 3) & 1) << 3);
        const int32_t half = lane >> 4;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4_trans(st + tile_chunk(1, tok, 2 * jj + half), r0, r1, r2, r3);
          mma_bf16_16816(o[2 * jj], pa, r0, r1);
          mma_bf16_16816(o[2 * jj + 1], pa, r2, r3);
        }
      }
    } else {
      const int32_t tq = lane >> 1;
      const int32_t hq = lane & 1;
      float s_ = 0.f;
      if (valid) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(wsm + s * kStageBytes +
                                                          tile_chunk(0, tq, hq * 8 + (c ^ (hq << 2))));
          s_ = fmaf(bf16lo(w.x), qr[c][0], s_);
          s_ = fmaf(bf16hi(w.x), qr[c][1], s_);
          s_ = fmaf(bf16lo(w.y), qr[c][2], s_);
          s_ = fmaf(bf16hi(w.y), qr[c][3], s_);
          s_ = fmaf(bf16lo(w.z), qr[c][4], s_);
          s_ = fmaf(bf16hi(w.z), qr[c][5], s_);
          s_ = fmaf(bf16lo(w.w), qr[c][6], s_);
          s_ = fmaf(bf16hi(w.w), qr[c][7], s_);
        }
      }
      s_ += __shfl_xor_sync(0xffffffffu, s_, 1);
      s_ = tq < nvalid ? s_ : -INFINITY;
      float bm = s_;
#pragma unroll
      for (int off = 2; off < 32; off <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
      const float mn = fmaxf(m0, bm);
      const float a = exp2f(m0 - mn);
      m0 = mn;
      const float pt = exp2f(s_ - mn);
      l0 = l0 * a + (hq ? 0.f : pt);
      if (a != 1.f) {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] *= a;
      }
      if (valid) {
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int32_t t = 2 * it + (lane >> 4);
          const float pv = __shfl_sync(0xffffffffu, pt, 2 * t);
          const uint4 w = *reinterpret_cast<const uint4*>(wsm + s * kStageBytes + tile_chunk(1, t, lane & 15));
          acc[0] = fmaf(pv, bf16lo(w.x), acc[0]);
          acc[1] = fmaf(pv, bf16hi(w.x), acc[1]);
          acc[2] = fmaf(pv, bf16lo(w.y), acc[2]);
          acc[3] = fmaf(pv, bf16hi(w.y), acc[3]);
          acc[4] = fmaf(pv, bf16lo(w.z), acc[4]);
          acc[5] = fmaf(pv, bf16hi(w.z), acc[5]);
          acc[6] = fmaf(pv, bf16lo(w.w), acc[6]);
          acc[7] = fmaf(pv, bf16hi(w.w), acc[7]);
        }
      }
    }
    __syncwarp();
    if (i + kStagedStages < my) issue(i + kStagedStages);
  }

  // ---- merge the four warps' states ------------------------------------------
  __syncthreads();  // every warp has consumed all its stages
  // [4 warps][16 rows][128] fp32, rows kMergeRow floats apart: the 8 extra
  // words shift each row by 8 banks, so a warp's 8-row stores (and the
  // merge's reads) spread over all banks
  float* so = reinterpret_cast<float*>(smem);
  if constexpr (kMMA) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (tig == 0) {
      red_m[warp][gid] = m0;
      red_m[warp][gid + 8] = m1;
      red_l[warp][gid] = l0;
      red_l[warp][gid + 8] = l1;
    }
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      float* r0 = so + (warp * 16 + gid) * kMergeRow + 8 * n + 2 * tig;
      float* r1 = so + (warp * 16 + gid + 8) * kMergeRow + 8 * n + 2 * tig;
      *reinterpret_cast<float2*>(r0) = make_float2(o[n][0], o[n][1]);
      *reinterpret_cast<float2*>(r1) = make_float2(o[n][2], o[n][3]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 16);
    l0 = warp_sum(l0);
    if (lane == 0) {
      red_m[warp][0] = m0;
      red_l[warp][0] = l0;
    }
    if (lane < 16) {
      float* r = so + warp * 16 * kMergeRow + 8 * lane;
      *reinterpret_cast<float4*>(r) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      *reinterpret_cast<float4*>(r + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
  __syncthreads();

  for (int32_t i = threadIdx.x; i < G * 128; i += blockDim.x) {
    const int32_t h = i >> 7;
    const int32_t d = i & 127;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kStagedWarps; ++w) M = fmaxf(M, red_m[w][h]);
    float Ls = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < kStagedWarps; ++w) {
      const float e = exp2f(red_m[w][h] - M);  // 0 for a warp that had no block
      Ls = fmaf(red_l[w][h], e, Ls);
      A = fmaf(so[(w * 16 + h) * kMergeRow + d], e, A);
    }
    const size_t bh = (size_t)b * H + (size_t)g * G + h;
    if (nparts == 1) {
      out[bh * 128 + d] = __float2bfloat16_rn(A / Ls);
    } else {
      p.ws_acc[(bh * p.max_partitions + part) * 128 + d] = A;
      if (d == 0) {
        p.ws_ml[(bh * p.max_partitions + part) * 2] = M;
        p.ws_ml[(bh * p.max_partitions + part) * 2 + 1] = Ls;
      }
    }
  }
}

// Grid mode (work_items == null): CTA = (partition, KV head, sequence).
// Persistent mode: a grid of resident CTAs takes (sequence, partition, KV
// head) items from the plan kernel's list, largest partitions first, through
// an atomic counter, so no CTA is spent on an empty partition and the last
// items to finish are the smallest.
template <bool kMMA, bool kAppend>
__global__ void __launch_bounds__(128) decode_staged_kernel(const __grid_constant__ CUtensorMap tmap,
                                                            DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ StagedShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int32_t warp = threadIdx.x >> 5;
  const int32_t lane = threadIdx.x & 31;
  // the partition merge may be scheduled as soon as every CTA has started; it
  // waits for this grid's completion before reading any partition state
  grid_dependents_launch();
  int32_t grid_len = 0;
  if (p.work_items == nullptr) {
    // grid mode: leave at once when this partition is empty (most CTAs of
    // short sequences), before any set-up
    const int32_t part = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    grid_len = checked_len(p, b, part == 0 && g == 0 && threadIdx.x == 0);
    if (grid_len == 0) {
      if (part == 0) {
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
        for (int32_t i = threadIdx.x; i < p.group * 128; i += blockDim.x)
          out[((size_t)b * p.num_heads + (size_t)g * p.group) * 128 + i] = __float2bfloat16_rn(0.f);
      }
      return;
    }
    if (part >= (grid_len + p.partition_tokens - 1) / p.partition_tokens) return;
  }
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStagedStages; ++s) mbar_init(&sh.bars[warp][s], 1);
    fence_barrier_init();
    if (warp == 0) prefetch_tensormap(&tmap);
  }
  __syncwarp();
  uint32_t phase = 0;
  if (p.work_items == nullptr) {
    decode_partition<kMMA, kAppend>(tmap, p, smem, sh, blockIdx.x, blockIdx.y, blockIdx.z, grid_len, phase);
    return;
  }
  grid_dependency_wait();  // the plan kernel's item list is complete
  const int32_t total = __ldcg(p.work_header) * p.num_kv_heads;
  if (threadIdx.x == 0) {
    sh.next_item = atomicAdd(p.work_header + 1, 1);
    sh.abort = 0;
  }
  __syncthreads();
  int32_t item = sh.next_item;
  while (item < total && !sh.abort) {
    int32_t next = 0;
    if (threadIdx.x == 0) next = atomicAdd(p.work_header + 1, 1);  // in flight during the item
    const int32_t bp = __ldcg(p.work_items + item / p.num_kv_heads);
    const int32_t g = item % p.num_kv_heads;
    const int32_t b = bp >> 16;
    decode_partition<kMMA, kAppend>(tmap, p, smem, sh, bp & 0xffff, g, b, checked_len(p, b, false), phase);
    // this item's shared-memory reads (generic proxy) precede the next item's
    // TMA writes (async proxy)
    fence_proxy_async_smem();
    if (threadIdx.x == 0) sh.next_item = next;
    __syncthreads();
    item = sh.next_item;
  }
}

// Work list for the persistent mode, one CTA: every non-empty partition of
// every sequence as (b << 16 | part), full partitions first, then each
// sequence's last partition by decreasing size (counting sort on the size in
// blocks). Also raises PA_DEVERR_SEQLEN for bad lengths, writes zeros for
// sequences of length 0, and resets the item counter.
// Launched as a programmatic dependent of the kernel before it in the stream
// (often the previous step's decode), so its launch overlaps that kernel;
// nothing is read or written before that kernel has completed.
constexpr int kPlanThreads = 1024;
constexpr int kMaxPartitionBlocks = 128;  // partitions of at most 2048 tokens
static_assert(kMaxPartitionBlocks <= 4 * 32, "the plan's scan covers 4 sizes per lane of one warp");

__global__ void __launch_bounds__(kPlanThreads) decode_plan_kernel(DecodeParams p) {
  __shared__ int32_t cnt[kMaxPartitionBlocks + 1];
  __shared__ int32_t off[kMaxPartitionBlocks + 1];
  // the decode CTAs may start (and set up) now; they wait for this grid's
  // completion before reading the list
  grid_dependents_launch();
  grid_dependency_wait();  // the kernel before this one is complete (inputs written, old list read)
  const int32_t SB = p.partition_tokens >> 4;  // blocks per full partition (<= kMaxPartitionBlocks)
  for (int32_t i = threadIdx.x; i <= SB; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  for (int32_t b = threadIdx.x; b < p.num_seqs; b += blockDim.x) {
    const int32_t L = checked_len(p, b, true);
    if (L == 0) {
      uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)b * p.num_heads * 128);
      for (int32_t i = 0; i < p.num_heads * 16; ++i) o[i] = make_uint4(0, 0, 0, 0);
      continue;
    }
    const int32_t n = (L + p.partition_tokens - 1) / p.partition_tokens;
    const int32_t r = ((L + 15) >> 4) - (n - 1) * SB;
    if (n > 1) atomicAdd(&cnt[SB], n - 1);
    atomicAdd(&cnt[r], 1);
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    // exclusive prefix sum of the counts in decreasing size (positions
    // 0 .. SB-1 hold sizes SB .. 1): lane l sums positions 4l .. 4l+3, a
    // warp scan adds the lanes before it
    const int32_t lane = threadIdx.x;
    int32_t c[4], own = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int32_t sz = SB - (4 * lane + k);
      c[k] = sz >= 1 ? cnt[sz] : 0;
      own += c[k];
    }
    int32_t incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int32_t run = incl - own;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int32_t sz = SB - (4 * lane + k);
      if (sz >= 1) off[sz] = run;
      run += c[k];
    }
    if (lane == 31) {
      p.work_header[0] = incl;
      p.work_header[1] = 0;
    }
  }
  __syncthreads();
  for (int32_t b = threadIdx.x; b < p.num_seqs; b += blockDim.x) {
    const int32_t L = checked_len(p, b, false);
    if (L == 0) continue;
    const int32_t n = (L + p.partition_tokens - 1) / p.partition_tokens;
    const int32_t r = ((L + 15) >> 4) - (n - 1) * SB;
    for (int32_t part = 0; part + 1 < n; ++part) p.work_items[atomicAdd(&off[SB], 1)] = (b << 16) | part;
    p.work_items[atomicAdd(&off[r], 1)] = (b << 16) | (n - 1);
  }
}

// ---- host side ---------------------------------------------------------------

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// Tensor map of a bf16 head_dim-128 pool: (d 128, row 16, kv head, K|V, block),
// box (64, 16, 1, box_kv, 1) -- K and V of a block together (box_kv 2) or one of
// them (box_kv 1) -- 128-byte swizzle, zero fill outside the tensor.
inline pa_status encode_pool_map(const void* pool, int32_t num_kv_heads, int32_t num_blocks, CUtensorMap* map,
                                 uint32_t box_kv = 2) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t hkv = (cuuint64_t)num_kv_heads;
  const cuuint64_t dims[5] = {128, 16, hkv, 2, (cuuint64_t)num_blocks};
  const cuuint64_t strides[4] = {256, 4096, hkv * 4096, 2 * hkv * 4096};
  const cuuint32_t box[5] = {64, 16, 1, box_kv, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(pool), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return PA_OK;
}

// Launches one decode_staged_kernel variant: the grid-mode grid, or in
// persistent mode min(items, resident CTAs) CTAs as a programmatic dependent
// of the plan kernel.
template <bool kMMA, bool kAppend>
inline pa_status launch_staged_variant(const CUtensorMap& map, const DecodeParams& p, cudaStream_t st) {
  // once per device: the shared-memory limit and the resident CTAs per SM
  static PerDevice<int32_t> occupancy;
  int32_t per_sm = 1;
  cudaError_t e = occupancy.get(&per_sm, [](int32_t* v) {
    int32_t n = 0;
    cudaError_t r = cudaFuncSetAttribute(decode_staged_kernel<kMMA, kAppend>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kStagedSmem);
    if (r == cudaSuccess)
      r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_staged_kernel<kMMA, kAppend>, 128, kStagedSmem);
    *v = n > 0 ? n : 1;
    return r;
  });
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_decode: %s", cudaGetErrorString(e));
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = kStagedSmem;
  cfg.stream = st;
  if (p.work_items == nullptr) {
    cfg.gridDim = dim3(p.max_partitions, p.num_kv_heads, p.num_seqs);
  } else {
    const int64_t most = (int64_t)p.num_seqs * p.max_partitions * p.num_kv_heads;
    const int64_t resident = (int64_t)per_sm * device_sm_count();
    cfg.gridDim = dim3((unsigned)(most < resident ? most : resident));
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  e = cudaLaunchKernelEx(&cfg, decode_staged_kernel<kMMA, kAppend>, map, p);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_decode: launch failed: %s", cudaGetErrorString(e));
  return PA_OK;
}

inline pa_status launch_staged_bf16_d128(const DecodeParams& p, cudaStream_t st) {
  CUtensorMap map;
  pa_status s = encode_pool_map(p.pool, p.num_kv_heads, p.num_blocks, &map);
  if (s != PA_OK) return s;
  if (p.work_items != nullptr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kPlanThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, decode_plan_kernel, p);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_decode (plan): launch failed: %s", cudaGetErrorString(e));
  }
  const bool append = p.k_new != nullptr;
  if (p.group == 1 && !append) s = launch_staged_variant<false, false>(map, p, st);
  else if (p.group == 1) s = launch_staged_variant<false, true>(map, p, st);
  else if (!append) s = launch_staged_variant<true, false>(map, p, st);
  else s = launch_staged_variant<true, true>(map, p, st);
  if (s != PA_OK) return s;
  if (p.max_partitions <= 1) return PA_OK;
  cudaError_t e = launch_partition_merge<__nv_bfloat16, 128>(p, st);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_decode (merge): launch failed: %s", cudaGetErrorString(e));
  return PA_OK;
}

}  // namespace pagedkv
