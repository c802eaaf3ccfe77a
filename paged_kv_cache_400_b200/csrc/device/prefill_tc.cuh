// Paged prefill / chunked-prefill attention on the 5th-generation tensor core
// (tcgen05 MMA, accumulators in tensor memory), bf16 pools with head_dim 128.
//
// Same operation as prefill_kernel: sequence b holds L tokens of KV, its n
// newest are queries at positions L-n .. L-1, the query at position P attends
// causally to positions 0..P through the block table ("大模型推理性能优化：
// PagedAttention与Continuous Batching原理与实践" §2: prefill runs the whole prompt;
// §2.2: KV is gathered from fixed 16-token pages through the page table).
//
// Work unit = (two 128-row query tiles, KV head g, sequence b); a row is
// (query token, query head of g's group): each tile is 128/G tokens x G heads,
// so one staged KV tile serves every head of the group and both tiles (twice
// the MMA work per staged byte).
//
// Persistent CTAs: the grid has one CTA per unit, but a running CTA takes the
// next units itself by cancelling CTAs that have not started (cluster launch
// control), so about one CTA per SM runs, set up once, and one unit's start
// (Q and first K/V loads, first S) and end (last PV, output stores) overlap
// its neighbours' work instead of leaving the SM idle between CTAs. Up to 128
// sequences the units go out longest sequence first, so the grid ends on short
// ones; past that in sequence order.
//
// 416 threads in five roles:
//   warps 0-3, 4-7  softmax, one warp group per query tile: thread r owns row
//              r of its tile = tensor-memory lane r; at the end of a unit they
//              stage the normalised rows one head-dim half at a time, and one
//              TMA store per half copies a whole tile out while the warps go
//              on (plain stores for a sequence's last, partial tile);
//   warps 8-9  producers: stream the K/V tiles of 64 keys (four 16-token
//              blocks gathered through the table, one TMA box per block and
//              K|V and head-dim half) into a 4-stage ring that runs on across
//              units, each warp staging two of the four blocks (two warps
//              issue boxes about 1.5x as fast as one);
//   warps 10-11 MMA issuers (one thread each), one per query tile: S = Q K^T
//              into tensor memory, then O += P V with P read back from tensor
//              memory; the two tiles' MMA chains overlap on the tensor core;
//   warp 12    scheduler: takes the units (its own, then cancelled CTAs'),
//              publishes each to the other roles through a two-slot ring and
//              loads its Q tiles by TMA once the previous unit's S MMAs have
//              completed.
// Tensor memory (512 columns, allocated once): per tile t at 256 t, O [0,128)
// fp32 and two S buffers [128,192), [192,256) fp32, each overwritten in place
// by its P as packed bf16 pairs. Issue order per tile S_0, S_1, PV_0, S_2,
// PV_1, ... (S_{j+1} after PV_j instead when its K/V tile is not in yet); the
// S buffers alternate over the CTA's whole sequence of KV steps, so the next
// unit's S_0 and S_1 are computed while the softmax warps finish the current
// unit. The running max is only raised when a tile's max exceeds it by more
// than 2^8 (log2 domain), so O in tensor memory is rescaled rarely; O and the
// row sum l always share the same reference max, so the final O / l is exact
// up to rounding.
// Shared memory: Q 2 x 32 KB (reloaded per unit), 4 x 32 KB K/V stages (K and
// V halves 8 KB each, 128-byte swizzle, the canonical K-major / MN-major UMMA
// layouts), 2 x 16 KB output staging (half a tile each, the Q tile layout).
// Every wait gives up after 2 s (PA_DEVERR_TIMEOUT) and its role stops; the
// other roles' waits then run out in turn, and the CTA still frees its tensor
// memory before it exits. Phase tracking: every mbarrier is waited on at most
// one completion ahead of the last one its waiter consumed, so a parity wait
// is never ambiguous.
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

// Two query tiles of 128 rows share every staged KV tile: one CTA per SM (all
// 512 tensor-memory columns, 225 KB of shared memory), a 4-deep KV ring.
template <int kQTiles>
struct TcConfig {
  static constexpr int kStages = 4;
  static constexpr int kProducers = 2;              // producer warps, each stages half of every KV tile
  static constexpr int kSoftmaxWarps = kQTiles * 4;
  static constexpr int kProducerWarp = kQTiles * 4;          // first producer warp
  static constexpr int kMmaWarp = kQTiles * 4 + kProducers;  // first of kQTiles issuer warps, one per tile
  static constexpr int kSchedWarp = kMmaWarp + kQTiles;      // the scheduler
  static constexpr int kThreads = (kSchedWarp + 1) * 32;
  static constexpr uint32_t kTmemCols = kQTiles * 256;
  // readers of each published unit: the producers, the issuers, the softmax warps
  static constexpr uint32_t kUnitReaders = kProducers + kQTiles + kSoftmaxWarps;
  // Q tiles, the K/V ring, half an output tile of staging per query tile, alignment slack
  static constexpr int kSmem = kQTiles * kTcQBytes + kStages * kTcStageBytes + kQTiles * (kTcQBytes / 2) + 1024;
};
constexpr int kTcQTiles = 2;

// A unit as the scheduler publishes it; n < 0 ends the CTA's work.
struct TcUnit {
  int32_t b, g, unit, q0, n, L;
};

template <int kQTiles, int kStages>
struct PrefillTcShared {
  alignas(16) uint4 clc_resp;    // response of the last cancellation request
  int32_t unit_desc[2][6];       // published units (TcUnit), two slots
  uint64_t clc_bar;              // cancellation response written
  uint64_t unit_full[2];         // unit slot published
  uint64_t unit_empty[2];        // unit slot read by every reader
  uint64_t unit_taken;           // the producers have taken the latest unit (one arrival per producer warp)
  uint64_t q_full;               // both Q tiles of the current unit loaded
  uint64_t q_empty;              // every S MMA of the current unit complete (one commit per issuer)
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[kQTiles][2];   // S of tile t's KV step J ready: s_full[t][J & 1]
  uint64_t p_full[kQTiles][2];   // P of step J written (one arrival per softmax warp)
  uint64_t pv_done[kQTiles][2];  // PV of step J complete: pv_done[t][J & 1]
  uint64_t stage_free[kQTiles];  // tile t's previous output store has read its staging half
  uint64_t staged[kQTiles];      // tile t's half rows written to staging (one arrival per softmax warp)
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

// The launch enumerates work units, not a dense (unit, head, sequence) box:
// sequence b brings ceil(n_b / U) units of U new tokens for each KV head, so
// no CTA exists for the missing units of short sequences. A sequence's units
// are contiguous in the order, all its KV heads together, each head's units
// last-first (the longest first). Up to kTcSortedSeqs sequences the sequences
// go longest first (UnitOrder, below); past that in index order, looked up
// here: the calling warp finds idx's unit by a prefix sum of the unit counts,
// 32 sequences per pass, loading one pass ahead; sequences whose query range
// is malformed count no units (and set PA_DEVERR_SEQLEN, from the lookup of
// idx 0, which scans every sequence). Returns false when idx lies past the
// last unit (the grid size is an upper bound).
// A CTA's successive lookups come in increasing idx order (cancelled CTAs are
// handed out in launch order), so the scan resumes at the pass that held the
// previous unit (cursor: that pass's first sequence and the units before it):
// a CTA scans the sequences about once per launch, not once per unit.
struct UnitCursor {
  int32_t s0 = 0;    // first sequence of the pass to start at
  int32_t base = 0;  // units of the sequences before it, times the KV heads
};

__device__ __forceinline__ bool find_unit(const PrefillParams& p, int32_t num_seqs, int32_t U, int32_t idx,
                                          TcUnit& u, UnitCursor& cur) {
  const int32_t lane = threadIdx.x & 31;
  if (idx == 0 || idx < cur.base) cur = UnitCursor{};  // idx 0 scans every sequence (error check)
  int32_t base = cur.base;
  bool any_bad = false, found = false;
  int32_t a_nx = 0, e_nx = 0, l_nx = 0;
  if (cur.s0 + lane < num_seqs) {
    a_nx = __ldg(p.query_start + cur.s0 + lane);
    e_nx = __ldg(p.query_start + cur.s0 + lane + 1);
    l_nx = __ldg(p.seq_lens + cur.s0 + lane);
  }
  for (int32_t s0 = cur.s0; s0 < num_seqs; s0 += 32) {
    const int32_t s = s0 + lane;
    const int32_t a = a_nx, n = e_nx - a_nx, L = l_nx;
    if (s + 32 < num_seqs) {
      a_nx = __ldg(p.query_start + s + 32);
      e_nx = __ldg(p.query_start + s + 33);
      l_nx = __ldg(p.seq_lens + s + 32);
    }
    int32_t cnt = 0;
    if (s < num_seqs) {
      const bool bad = a < 0 || n < 0 || n > p.max_query_len || a + n > p.num_tokens;
      any_bad |= bad;
      cnt = bad ? 0 : (n + U - 1) / U * p.num_kv_heads;
    }
    int32_t incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t hit = __ballot_sync(0xffffffffu, idx >= base + incl - cnt && idx < base + incl);
    if (hit) {
      const int32_t src = __ffs(hit) - 1;
      const int32_t local = idx - (base + __shfl_sync(0xffffffffu, incl - cnt, src));
      const int32_t units = __shfl_sync(0xffffffffu, cnt, src) / p.num_kv_heads;
      u.b = s0 + src;
      u.g = local / units;
      u.unit = units - 1 - local % units;
      u.q0 = __shfl_sync(0xffffffffu, a, src);
      u.n = __shfl_sync(0xffffffffu, n, src);
      u.L = __shfl_sync(0xffffffffu, L, src);
      if (!found) cur = UnitCursor{s0, base};
      found = true;
      if (idx != 0) return true;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (idx == 0 && __any_sync(0xffffffffu, any_bad) && lane == 0) raise_device_error(PA_DEVERR_SEQLEN);
  return found;
}

// Up to this many sequences the units go out longest sequence first (see
// UnitOrder); beyond it in sequence order.
constexpr int kTcSortedSeqs = 128;

// The launch order of the units when the sequences are sorted by KV length L,
// longest first (ties by index): every sequence's units (all KV heads
// together, each head's units last-first) stay contiguous, sequence s's from
// index start[s / 32] on, cnt[s / 32] of them, held by lane s % 32. The
// longest units start first and the grid ends on short ones, so the SMs run
// out of work at nearly the same time. Built once per CTA by its scheduler
// warp, O(num_seqs^2 / 32) per lane; sequences whose query range is
// malformed count no units and set PA_DEVERR_SEQLEN.
struct UnitOrder {
  int32_t start[kTcSortedSeqs / 32];
  int32_t cnt[kTcSortedSeqs / 32];
};

__device__ __forceinline__ void build_unit_order(const PrefillParams& p, int32_t num_seqs, int32_t U,
                                                 UnitOrder& o) {
  constexpr int P = kTcSortedSeqs / 32;
  const int32_t lane = threadIdx.x & 31;
  int32_t L[P];
  bool any_bad = false;
#pragma unroll
  for (int pp = 0; pp < P; ++pp) {
    const int32_t s = pp * 32 + lane;
    L[pp] = -1;
    o.cnt[pp] = 0;
    o.start[pp] = 0;
    if (s < num_seqs) {
      const int32_t a = __ldg(p.query_start + s);
      const int32_t n = __ldg(p.query_start + s + 1) - a;
      const bool bad = a < 0 || n < 0 || n > p.max_query_len || a + n > p.num_tokens;
      any_bad |= bad;
      L[pp] = __ldg(p.seq_lens + s);
      o.cnt[pp] = bad ? 0 : (n + U - 1) / U * p.num_kv_heads;
    }
  }
  // start of s = the units of every sequence ahead of it: longer, or as long
  // with a lower index
#pragma unroll
  for (int qq = 0; qq < P; ++qq) {
    if (qq * 32 >= num_seqs) break;
#pragma unroll 4
    for (int src = 0; src < 32; ++src) {
      const int32_t Lo = __shfl_sync(0xffffffffu, L[qq], src);
      const int32_t co = __shfl_sync(0xffffffffu, o.cnt[qq], src);
      const int32_t so = qq * 32 + src;
#pragma unroll
      for (int pp = 0; pp < P; ++pp) {
        const int32_t s = pp * 32 + lane;
        if (Lo > L[pp] || (Lo == L[pp] && so < s)) o.start[pp] += co;
      }
    }
  }
  if (__any_sync(0xffffffffu, any_bad) && lane == 0) raise_device_error(PA_DEVERR_SEQLEN);
}

// Unit idx of a UnitOrder (the calling warp); false past the last unit.
__device__ __forceinline__ bool find_unit_sorted(const PrefillParams& p, const UnitOrder& o, int32_t idx,
                                                 TcUnit& u) {
  constexpr int P = kTcSortedSeqs / 32;
  int32_t seq = -1, st = 0, ct = 0;
#pragma unroll
  for (int pp = 0; pp < P; ++pp) {
    const uint32_t hit = __ballot_sync(0xffffffffu, idx >= o.start[pp] && idx < o.start[pp] + o.cnt[pp]);
    const int32_t src = hit ? __ffs(hit) - 1 : 0;
    const int32_t st_pp = __shfl_sync(0xffffffffu, o.start[pp], src);
    const int32_t ct_pp = __shfl_sync(0xffffffffu, o.cnt[pp], src);
    if (hit && seq < 0) {
      seq = pp * 32 + src;
      st = st_pp;
      ct = ct_pp;
    }
  }
  if (seq < 0) return false;
  const int32_t local = idx - st;
  const int32_t units = ct / p.num_kv_heads;
  u.b = seq;
  u.g = local / units;
  u.unit = units - 1 - local % units;
  u.q0 = __ldg(p.query_start + seq);
  u.n = __ldg(p.query_start + seq + 1) - u.q0;
  u.L = __ldg(p.seq_lens + seq);
  return true;
}

// KV tiles of a unit: returns the unit's count (its last query tile's) and
// sets nt[t] for each query tile (0 for a tile past the sequence's new tokens).
template <int kQTiles>
__device__ __forceinline__ int32_t unit_tiles(const TcUnit& u, int32_t QT, int32_t (&nt)[kQTiles],
                                              int32_t& nblocks) {
  const int32_t ctx = u.L - u.n;
  const int32_t tok_begin = u.unit * kQTiles * QT;
#pragma unroll
  for (int t = 0; t < kQTiles; ++t) {
    const int32_t tb = tok_begin + t * QT;
    nt[t] = tb < u.n ? ((ctx + min(u.n, tb + QT) - 1) / 16 + kTcBlocksPerTile) / kTcBlocksPerTile : 0;
  }
  nblocks = (ctx + min(u.n, tok_begin + kQTiles * QT) - 1) / 16 + 1;
  return (nblocks + kTcBlocksPerTile - 1) / kTcBlocksPerTile;
}

template <int kQTiles>
__global__ void __launch_bounds__(TcConfig<kQTiles>::kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap pool_map, const __grid_constant__ CUtensorMap q_map,
                      const __grid_constant__ CUtensorMap out_map, PrefillParams p, const uint4* __restrict__ pool,
                      int32_t num_seqs) {
  using Cfg = TcConfig<kQTiles>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ PrefillTcShared<kQTiles, S> sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = smem;
  uint8_t* kv_smem = smem + kQTiles * kTcQBytes;
  uint8_t* out_smem = kv_smem + S * kTcStageBytes;

  const int32_t G = p.group;
  const int32_t QT = 128 / G;  // tokens per 128-row tile
  const int32_t U = kQTiles * QT;
  const int32_t warp = threadIdx.x >> 5;
  const int32_t lane = threadIdx.x & 31;

  if (warp == Cfg::kSchedWarp && lane == 0) {
    mbar_init(&sh.clc_bar, 1);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.unit_full[i], 1);
      mbar_init(&sh.unit_empty[i], Cfg::kUnitReaders);
    }
    mbar_init(&sh.unit_taken, Cfg::kProducers);
    mbar_init(&sh.q_full, 1);
    mbar_init(&sh.q_empty, kQTiles);  // one commit (or arrival) per issuer
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
#pragma unroll
    for (int t = 0; t < kQTiles; ++t) {
      mbar_init(&sh.stage_free[t], 1);
      mbar_init(&sh.staged[t], 4);
    }
    fence_barrier_init();
    prefetch_tensormap(&pool_map);
    prefetch_tensormap(&q_map);
    prefetch_tensormap(&out_map);
  }
  if (warp == Cfg::kMmaWarp) {
    tmem_alloc(&sh.tmem_base, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sh.tmem_base;  // read by the MMA and softmax warps only

  // unit k from its slot (any subset of a warp's lanes may call this)
  auto read_unit = [&](uint32_t k, TcUnit& u) -> bool {
    if (!mbar_wait_bounded(&sh.unit_full[k & 1], (k >> 1) & 1u, kWaitLimitNs)) return false;
    const int32_t* d = sh.unit_desc[k & 1];
    u.b = d[0];
    u.g = d[1];
    u.unit = d[2];
    u.q0 = d[3];
    u.n = d[4];
    u.L = d[5];
    return true;
  };

  if (warp >= Cfg::kProducerWarp && warp < Cfg::kMmaWarp) {
    // ---- producers: warp pw stages blocks 2 pw, 2 pw + 1 of every 64-key tile -------
    const int32_t pw = warp - Cfg::kProducerWarp;

    // stages the unit's KV tiles (global tile index jkv0 + j) into the ring
    auto stream_kv = [&](const TcUnit& u, uint32_t jkv0) -> bool {
      int32_t nt[kQTiles];
      int32_t nblocks;
      const int32_t nt_max = unit_tiles<kQTiles>(u, QT, nt, nblocks);
      const int32_t* table = p.block_tables + (size_t)u.b * p.max_blocks;
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
        const uint32_t J = jkv0 + (uint32_t)j;
        const uint32_t s = J % S;
        if (J >= (uint32_t)S) {
          const bool ok = mbar_wait_bounded(&sh.kv_empty[s], (J / S - 1) & 1u, kWaitLimitNs);
          if (__any_sync(0xffffffffu, !ok)) {
            if (lane == 0) raise_device_error(PA_DEVERR_TIMEOUT);
            return false;
          }
        }
        uint8_t* st = kv_smem + s * kTcStageBytes;
        // TMA fills whole blocks inside the sequence; the warp writes the
        // sequence's partial last block row by row (rows past L zeroed) and
        // zeros for slots past the last block or with a bad id.
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
          const int32_t rows = (bi < nblocks && blk[m] >= 0) ? min(16, u.L - bi * 16) : 0;
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
              val = __ldg(pool + ((((size_t)blk[m] * 2 + kv) * p.num_kv_heads + u.g) * 16 + row) * 16 + c);
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
          tma_load_5d(st + tc_region(kv, half) + slot * 2048, &pool_map, &sh.kv_full[s], 64 * half, 0, u.g, kv,
                      my_blk);
        }
      }
      return true;
    };

    uint32_t k = 0;    // units taken
    uint32_t jkv = 0;  // KV tiles staged (both producer warps count alike)
    bool ok = true;
    for (;;) {
      TcUnit u;
      if (!__all_sync(0xffffffffu, read_unit(k, u))) {
        ok = false;
        break;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sh.unit_empty[k & 1]);
        if (u.n >= 0) mbar_arrive(&sh.unit_taken);
      }
      if (u.n < 0) break;
      ok = stream_kv(u, jkv);
      int32_t nt[kQTiles], nb;
      jkv += (uint32_t)unit_tiles<kQTiles>(u, QT, nt, nb);
      ++k;
      if (!ok) break;
    }
    // the asynchronous releases still owed to the ring land before the CTA exits
    if (ok && pw == 0)
      for (uint32_t J = jkv > (uint32_t)S ? jkv - S : 0; J < jkv && ok; ++J)
        ok = mbar_wait_bounded(&sh.kv_empty[J % S], (J / S) & 1u, kWaitLimitNs);
    if (!__all_sync(0xffffffffu, ok) && lane == 0) raise_device_error(PA_DEVERR_TIMEOUT);
  } else if (warp == Cfg::kSchedWarp) {
    // ---- scheduler: resolves the CTA's own unit, then cancels not-yet-started
    // CTAs and takes their units, publishing each to the other roles through a
    // two-slot ring, and loads each unit's Q tiles once the previous unit's S
    // MMAs have completed. The next unit is requested once the producers have
    // taken the last one, so the CTA holds at most one unit beyond the one in
    // its K/V ring.
    // The unit at CTA index i, unless i lies past the last unit, its sequence
    // is malformed, or a wait has timed out somewhere in the grid (then the
    // remaining units are skipped; the error stays set until the host reads it).
    UnitOrder order;
    UnitCursor cursor;
    const bool sorted = num_seqs <= kTcSortedSeqs;
    if (sorted) build_unit_order(p, num_seqs, U, order);
    auto resolve = [&](int32_t i, TcUnit& u) -> bool {
      if (!(sorted ? find_unit_sorted(p, order, i, u) : find_unit(p, num_seqs, U, i, u, cursor))) return false;
      if (u.L < u.n || (int64_t)u.L > (int64_t)p.max_blocks * 16) {
        if (u.unit == 0 && u.g == 0 && lane == 0) raise_device_error(PA_DEVERR_SEQLEN);
        return false;
      }
      return !(*reinterpret_cast<volatile unsigned int*>(&g_error_word) & PA_DEVERR_TIMEOUT);
    };
    bool ok = true;
    bool can_cancel = true;  // no request has come back empty yet
    uint32_t clc_phase = 0;
    // one cancellation request; false once none is left (or on a timeout)
    auto take_next = [&](TcUnit& u) -> bool {
      while (can_cancel && ok) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&sh.clc_bar, 16);
          clc_try_cancel(&sh.clc_resp, &sh.clc_bar);
        }
        // the response lands before anything else happens here
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&sh.clc_bar, clc_phase, kWaitLimitNs));
        clc_phase ^= 1u;
        if (!ok) break;
        int32_t x = 0;
        const bool got = clc_canceled_x(&sh.clc_resp, x);
        fence_proxy_async_smem();  // this read before the next response's write
        __syncwarp();
        if (!got) {
          can_cancel = false;
          break;
        }
        if (resolve(x, u)) return true;
      }
      return false;
    };
    TcUnit u;
    bool have = resolve((int32_t)blockIdx.x, u) || take_next(u);
    uint32_t k = 0;  // units published
    while (have && ok) {
      // unit k goes into slot k & 1 once every reader has taken unit k - 2
      if (k >= 2) ok = __all_sync(0xffffffffu, mbar_wait_bounded(&sh.unit_empty[k & 1], ((k >> 1) - 1) & 1u,
                                                                 kWaitLimitNs));
      if (!ok) break;
      if (lane == 0) {
        int32_t* d = sh.unit_desc[k & 1];
        d[0] = u.b;
        d[1] = u.g;
        d[2] = u.unit;
        d[3] = u.q0;
        d[4] = u.n;
        d[5] = u.L;
        mbar_arrive(&sh.unit_full[k & 1]);
      }
      // its Q tiles, once every S MMA of unit k - 1 has completed
      if (k >= 1) ok = __all_sync(0xffffffffu, mbar_wait_bounded(&sh.q_empty, (k - 1) & 1u, kWaitLimitNs));
      if (!ok) break;
      if (lane == 0) {
        const int32_t row = u.q0 + u.unit * U;
        mbar_arrive_expect_tx(&sh.q_full, kQTiles * kTcQBytes);
#pragma unroll
        for (int t = 0; t < kQTiles; ++t) {
          tma_load_3d(q_smem + t * kTcQBytes, &q_map, &sh.q_full, 0, u.g * G, row + t * QT);
          tma_load_3d(q_smem + t * kTcQBytes + kTcQBytes / 2, &q_map, &sh.q_full, 64, u.g * G, row + t * QT);
        }
      }
      ++k;
      // the next unit once the producers have taken this one
      if (!can_cancel) break;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&sh.unit_taken, (k - 1) & 1u, kWaitLimitNs));
      if (!ok) break;
      have = take_next(u);
    }
    // the end: an empty unit in the next slot stops every reader
    bool fin = true;
    if (k >= 2) fin = mbar_wait_bounded(&sh.unit_empty[k & 1], ((k >> 1) - 1) & 1u, kWaitLimitNs);
    if (__all_sync(0xffffffffu, fin) && lane == 0) {
      sh.unit_desc[k & 1][4] = -1;
      mbar_arrive(&sh.unit_full[k & 1]);
    }
    // the last unit's Q release (a commit) lands before the CTA exits
    if (ok && k >= 1) ok = __all_sync(0xffffffffu, mbar_wait_bounded(&sh.q_empty, (k - 1) & 1u, kWaitLimitNs));
    if (!ok && lane == 0) raise_device_error(PA_DEVERR_TIMEOUT);
  } else if (warp >= Cfg::kMmaWarp) {
    // ---- MMA issuers: warp kMmaWarp + t, one thread, drives query tile t -------------
    const int t = warp - Cfg::kMmaWarp;
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc_idesc_bf16(128, kTcKeys, false);
      constexpr uint32_t idesc_pv = tc_idesc_bf16(128, 128, true);
      const uint32_t qa = smem_addr(q_smem) + t * kTcQBytes;
      const uint32_t kv_addr = smem_addr(kv_smem);
      const uint32_t tm = tmem + t * 256;
      uint32_t k = 0;    // units taken
      uint32_t jkv = 0;  // KV tiles of the earlier units
      uint32_t js = 0;   // this tile's KV steps of the earlier units (S/P buffer JS & 1)
      bool ok = true;
      for (;;) {
        TcUnit u;
        ok = read_unit(k, u);
        if (!ok) break;
        mbar_arrive(&sh.unit_empty[k & 1]);
        if (u.n < 0) break;
        int32_t nt[kQTiles], nblocks;
        const int32_t nt_max = unit_tiles<kQTiles>(u, QT, nt, nblocks);
        const int32_t ntt = (kQTiles == 1 || t == 0) ? nt[0] : nt[kQTiles - 1];
        ok = mbar_wait_bounded(&sh.q_full, k & 1u, kWaitLimitNs);
        int32_t kv_ready = -1;  // KV tiles 0 .. kv_ready of the unit have been waited for, in order
        auto ensure_kv = [&](int32_t j) {
          for (int32_t i = kv_ready + 1; i <= j && ok; ++i) {
            const uint32_t J = jkv + (uint32_t)i;
            ok = mbar_wait_bounded(&sh.kv_full[J % S], (J / S) & 1u, kWaitLimitNs);
          }
          kv_ready = j;
        };
        // S_j = Q_t K_j^T: eight k-steps of 16 dims (32 bytes inside the
        // swizzled 128-byte rows; dims 64..127 in the second half region).
        // After the tile's last S of the unit its Q buffer is released.
        auto issue_s = [&](int32_t j) {
          ensure_kv(j);
          if (!ok) return;
          tc_fence_after_sync();
          const uint32_t J = jkv + (uint32_t)j, JS = js + (uint32_t)j;
          const uint32_t kaddr = kv_addr + (J % S) * kTcStageBytes;
          const uint32_t d = tm + 128 + 64 * (JS & 1);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * (kTcQBytes / 2) + (kk & 3) * 32;
            const uint32_t koff = (kk >> 2) * kTcHalfBytes + (kk & 3) * 32;
            tc_mma_ss(d, tc_desc_sw128(qa + off, 16, 1024), tc_desc_sw128(kaddr + koff, 16, 1024), idesc_s,
                      kk > 0);
          }
          tc_commit(&sh.s_full[t][JS & 1]);
          if (j == ntt - 1) tc_commit(&sh.q_empty);
        };
        if (ok && ntt > 0) issue_s(0);
        if (ok && ntt == 0) mbar_arrive(&sh.q_empty);  // this tile reads no Q in this unit
        for (int32_t j = 0; j < nt_max && ok; ++j) {
          const uint32_t J = jkv + (uint32_t)j;
          if (j < ntt) {
            const uint32_t JS = js + (uint32_t)j;
            // S_{j+1} goes ahead of PV_j when its K/V tile is already in;
            // otherwise PV_j is issued as soon as P_j is written and S_{j+1}
            // follows it, so a late K/V tile does not hold PV_j back
            bool s_next = false;
            if (j + 1 < ntt &&
                (kv_ready >= j + 1 || mbar_test_wait(&sh.kv_full[(J + 1) % S], ((J + 1) / S) & 1u))) {
              if (kv_ready < j + 1) kv_ready = j + 1;
              issue_s(j + 1);
              s_next = true;
            }
            ok = ok && mbar_wait_bounded(&sh.p_full[t][JS & 1], (JS >> 1) & 1u, kWaitLimitNs);
            if (!ok) break;
            tc_fence_after_sync();
            // O_t += P_j V_j: four k-steps of 16 keys; V is MN-major (dims
            // contiguous), its two 64-dim halves one leading offset apart,
            // 8-key groups 1024 B apart. The unit's first PV starts O afresh
            // (its P_0 is written only after the softmax warps have read the
            // previous unit's O).
            const uint32_t vaddr = kv_addr + (J % S) * kTcStageBytes + tc_region(1, 0);
            const uint32_t pa = tm + 128 + 64 * (JS & 1);
#pragma unroll
            for (int kk = 0; kk < kTcKeys / 16; ++kk)
              tc_mma_ts(tm, pa + 8 * kk, tc_desc_sw128(vaddr + kk * 2048, kTcHalfBytes, 1024), idesc_pv,
                        (j > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&sh.pv_done[t][JS & 1]);
            tc_commit(&sh.kv_empty[J % S]);
            if (j + 1 < ntt && !s_next) issue_s(j + 1);
          } else {
            // this tile never reads KV tile j; release it in order, after its load
            ensure_kv(j);
            if (ok) mbar_arrive(&sh.kv_empty[J % S]);
          }
        }
        jkv += (uint32_t)nt_max;
        js += (uint32_t)ntt;
        ++k;
        if (!ok) break;
      }
      if (!ok) raise_device_error(PA_DEVERR_TIMEOUT);
    }
  } else {
    // ---- softmax: warp group t, thread r owns row r of query tile t ----------------
    const int32_t t = warp >> 2;
    const int32_t r = threadIdx.x - 128 * t;
    const uint32_t lane_base = tmem + t * 256 + ((uint32_t)((warp & 3) * 32) << 16);
    uint8_t* stage = out_smem + t * (kTcQBytes / 2);  // half of this tile's output rows, in the Q tile layout
    const bool leader = r == 0;                 // issues the tile's output stores
    uint32_t k = 0;   // units taken
    uint32_t js = 0;  // this tile's KV steps of the earlier units
    uint32_t ne = 0;  // this tile's staged output halves so far
    bool ok = true;
    for (;;) {
      TcUnit u;
      if (!__all_sync(0xffffffffu, read_unit(k, u))) {
        ok = false;
        break;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.unit_empty[k & 1]);
      if (u.n < 0) break;
      int32_t nt[kQTiles], nblocks;
      unit_tiles<kQTiles>(u, QT, nt, nblocks);
      const int32_t ntt = (kQTiles == 1 || t == 0) ? nt[0] : nt[kQTiles - 1];
      const int32_t ctx = u.L - u.n;
      const int32_t tb = u.unit * U + t * QT;
      const int32_t tok = tb + r / G;
      const int32_t te = min(u.n, tb + QT);
      const bool valid = tok < te;
      const int32_t P = valid ? ctx + tok : ctx + te - 1;  // padding rows: any finite row
      float m_ref = -INFINITY, l = 0.f;
      for (int32_t j = 0; j < ntt; ++j) {
        const uint32_t JS = js + (uint32_t)j;
        const bool arrived = mbar_wait_bounded(&sh.s_full[t][JS & 1], (JS >> 1) & 1u, kWaitLimitNs);
        if (__any_sync(0xffffffffu, !arrived)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t sbuf = lane_base + 128 + 64 * (JS & 1);
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
                mbar_wait_bounded(&sh.pv_done[t][(JS - 1) & 1], ((JS - 1) >> 1) & 1u, kWaitLimitNs);
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
        if (lane == 0) mbar_arrive(&sh.p_full[t][JS & 1]);
      }
      if (ok && ntt > 0) {
        const uint32_t JL = js + (uint32_t)ntt - 1;  // the unit's last PV
        const bool done = mbar_wait_bounded(&sh.pv_done[t][JL & 1], (JL >> 1) & 1u, kWaitLimitNs);
        ok = !__any_sync(0xffffffffu, !done);
        if (ok) {
          tc_fence_after_sync();
          // O / l as bf16, one head-dim half at a time through the tile's
          // 16 KB staging half (the Q tile layout: 128-byte rows, 16-byte
          // chunks XOR-swizzled by row, which also spreads a warp's writes
          // over all banks). A whole tile leaves by one TMA store per half
          // that drains while the warps go on; the sequence's last, partial
          // tile (its rows after the new tokens belong to the next sequence)
          // by plain stores, each warp its own valid rows. The warps of the
          // group meet on mbarriers, so that every wait is bounded.
          const float inv = 1.f / l;
          const bool whole = te == tb + QT;
          const int32_t row0 = (warp & 3) * 32;
          uint4* out4 = reinterpret_cast<uint4*>(p.out);
#pragma unroll 1
          for (int half = 0; half < 2 && ok; ++half) {
            uint32_t o[64];
            tmem_ld64_wait(lane_base + 64 * half, o);
            // the tile's previous store has read the staging half
            if (leader) {
              bulk_wait_group_read0();
              mbar_arrive(&sh.stage_free[t]);
            }
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(&sh.stage_free[t], ne & 1u, kWaitLimitNs));
            if (!ok) break;
#pragma unroll
            for (int c = 0; c < 8; ++c) {  // dims 64 half + 8 c .. + 7
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv);
              *reinterpret_cast<uint4*>(stage + r * 128 + ((c ^ (r & 7)) << 4)) = w;
            }
            fence_proxy_async_smem();  // the staging writes before the TMA store reads them
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.staged[t]);
            if (leader) {
              ok = mbar_wait_bounded(&sh.staged[t], ne & 1u, kWaitLimitNs);
              if (ok && whole) {
                tma_store_3d(&out_map, stage, 64 * half, u.g * G, u.q0 + tb);
                bulk_commit_group();
              }
            }
            ok = __all_sync(0xffffffffu, ok);
            ++ne;
            if (ok && !whole) {
#pragma unroll 4
              for (int i = 0; i < 8; ++i) {  // four 128-byte half rows per instruction
                const int32_t rr = row0 + 4 * i + (lane >> 3);
                const int32_t c = lane & 7;
                const int32_t tk = tb + rr / G;
                if (tk < te)
                  out4[((size_t)(u.q0 + tk) * p.num_heads + (size_t)u.g * G + rr % G) * 16 + half * 8 + c] =
                      *reinterpret_cast<const uint4*>(stage + rr * 128 + ((c ^ (rr & 7)) << 4));
              }
            }
          }
        }
      }
      js += (uint32_t)ntt;
      ++k;
      if (!ok) break;
    }
    if (!ok && lane == 0) raise_device_error(PA_DEVERR_TIMEOUT);
    // the output stores have completed before the CTA exits
    if (leader) bulk_wait_group0();
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

inline pa_status launch_prefill_tc(const void* pool, int32_t num_blocks, const PrefillParams& p, int32_t num_seqs,
                                   cudaStream_t st) {
  using Cfg = TcConfig<kTcQTiles>;
  CUtensorMap pool_map, q_map, out_map;
  pa_status s = encode_pool_map(pool, p.num_kv_heads, num_blocks, &pool_map, 1);
  if (s != PA_OK) return s;
  s = encode_q_map(p.q, p.num_heads, p.num_tokens, p.group, &q_map);
  if (s != PA_OK) return s;
  s = encode_q_map(p.out, p.num_heads, p.num_tokens, p.group, &out_map);
  if (s != PA_OK) return s;
  static PerDevice<int32_t> smem_set;
  cudaError_t attr = set_smem_once(smem_set, prefill_tc_kernel<kTcQTiles>, Cfg::kSmem);
  if (attr != cudaSuccess) return fail(PA_ERR_CUDA, "pa_prefill: %s", cudaGetErrorString(attr));
  // one CTA per unit (an upper bound on the units of well-formed query
  // ranges: every sequence has at most max_query_len new tokens, and together
  // at most num_tokens); running CTAs cancel most of them and take their units
  const int64_t U = kTcQTiles * (128 / p.group);
  const int64_t units = std::min<int64_t>((int64_t)num_seqs * ((p.max_query_len + U - 1) / U),
                                          ((int64_t)p.num_tokens + (int64_t)num_seqs * (U - 1)) / U);
  const int64_t ctas = units * p.num_kv_heads;
  if (ctas <= 0) return PA_OK;
  if (ctas > INT32_MAX) return fail(PA_ERR_UNSUPPORTED, "pa_prefill: %lld work units", (long long)ctas);
  prefill_tc_kernel<kTcQTiles><<<(unsigned)ctas, Cfg::kThreads, Cfg::kSmem, st>>>(
      pool_map, q_map, out_map, p, reinterpret_cast<const uint4*>(pool), num_seqs);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "pa_prefill: launch failed: %s", cudaGetErrorString(e));
  return PA_OK;
}

}  // namespace pagedkv
