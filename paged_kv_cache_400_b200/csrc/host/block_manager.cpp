// Host block manager of the paged KV cache.
//
// Follows "如何通过PagedAttention实现LLM高性能推理：实战指南" §2.2 (free-block pool
// starting as range(num_blocks), allocation of ceil(num_tokens / 16) blocks
// from its front), "vLLM 原理：PagedAttention 和 Continuous Batching" / 工作原理
// (one page table per request; a new page only when the last is full; pages
// return at once when a request ends) and "优势 / 3. 支持共享" (requests
// sharing a prefix share its pages), with reference counts per block and
// copy-on-write of a shared partial last block.
//
// Data layout: the free list is a ring buffer of capacity num_blocks (it can
// never hold more), so push-back / pop-front are O(1) with no allocation; each
// sequence owns a std::vector<int32_t> page table.
#include <algorithm>
#include <cstring>
#include <unordered_map>
#include <vector>

#include "bm_internal.hpp"
#include "errors.hpp"

using pagedkv::fail;

namespace pagedkv {

std::string& last_error_slot() {
  static thread_local std::string s;
  return s;
}

}  // namespace pagedkv

extern "C" {

pa_status pa_bm_create(int32_t num_blocks, int32_t block_size,
                       const int32_t* initial_free_order, pa_bm** out) {
  if (!out) return fail(PA_ERR_INVALID_ARG, "pa_bm_create: out is NULL");
  *out = nullptr;
  if (block_size != PA_BLOCK_SIZE)
    return fail(PA_ERR_UNSUPPORTED, "pa_bm_create: block_size %d (only 16)", block_size);
  if (num_blocks <= 0)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_create: num_blocks %d", num_blocks);
  pa_bm* bm = new pa_bm();
  bm->num_blocks = num_blocks;
  bm->ring.resize(num_blocks);
  bm->refcount.assign(num_blocks, 0);
  if (initial_free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int32_t i = 0; i < num_blocks; ++i) {
      int32_t b = initial_free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete bm;
        return fail(PA_ERR_INVALID_ARG,
                    "pa_bm_create: initial_free_order is not a permutation (index %d)", i);
      }
      seen[b] = 1;
      bm->ring[i] = b;
    }
  } else {
    for (int32_t i = 0; i < num_blocks; ++i) bm->ring[i] = i;
  }
  bm->head = 0;
  bm->count = num_blocks;
  bm->block_hash.assign(num_blocks, 0);
  bm->has_hash.assign(num_blocks, 0);
  bm->valid.assign(num_blocks, 0);
  bm->ev_prev.assign(num_blocks, -1);
  bm->ev_next.assign(num_blocks, -1);
  bm->in_ev.assign(num_blocks, 0);
  *out = bm;
  return PA_OK;
}

void pa_bm_destroy(pa_bm* bm) { delete bm; }

pa_status pa_bm_allocate(pa_bm* bm, int64_t seq, int32_t num_tokens) {
  if (!bm) return fail(PA_ERR_INVALID_ARG, "pa_bm_allocate: bm is NULL");
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "pa_bm_allocate: num_tokens %d", num_tokens);
  if (bm->seqs.count(seq)) return fail(PA_ERR_SEQ_EXISTS, "pa_bm_allocate: seq %lld exists", (long long)seq);
  const int32_t n = pagedkv::blocks_for(num_tokens);
  if (n > bm->free_blocks())
    return fail(PA_ERR_NO_BLOCKS, "pa_bm_allocate: need %d blocks, %d free", n, bm->free_blocks());
  pagedkv::SeqState st;
  st.table.reserve(n + 1);
  for (int32_t i = 0; i < n; ++i) {
    int32_t b = bm->take_fresh();
    bm->refcount[b] = 1;
    st.table.push_back(b);
  }
  st.len = num_tokens;
  bm->seqs.emplace(seq, std::move(st));
  return PA_OK;
}

pa_status pa_bm_append_slot(pa_bm* bm, int64_t seq, int64_t* slot, int32_t* cow_src,
                            int32_t* cow_dst) {
  if (!bm || !slot || !cow_src || !cow_dst)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_append_slot: NULL argument");
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return fail(PA_ERR_UNKNOWN_SEQ, "pa_bm_append_slot: seq %lld", (long long)seq);
  pagedkv::SeqState& st = it->second;
  const int32_t pos = st.len;
  const int32_t row = pos % PA_BLOCK_SIZE;
  int32_t blk;
  int32_t cs = -1, cd = -1;
  if (row == 0) {
    // every page is full (or there is none): a fresh page
    if (bm->free_blocks() == 0) return fail(PA_ERR_NO_BLOCKS, "pa_bm_append_slot: no free block");
    blk = bm->take_fresh();
    bm->refcount[blk] = 1;
    st.table.push_back(blk);
  } else {
    const int32_t last = st.table.back();
    if (bm->refcount[last] > 1) {
      // shared partial page: copy-on-write
      if (bm->free_blocks() == 0) return fail(PA_ERR_NO_BLOCKS, "pa_bm_append_slot: no block for copy-on-write");
      blk = bm->take_fresh();
      bm->refcount[blk] = 1;
      bm->refcount[last] -= 1;
      st.table.back() = blk;
      cs = last;
      cd = blk;
    } else {
      blk = last;
    }
  }
  st.len = pos + 1;
  *slot = (int64_t)blk * PA_BLOCK_SIZE + row;
  *cow_src = cs;
  *cow_dst = cd;
  return PA_OK;
}

pa_status pa_bm_fork(pa_bm* bm, int64_t parent, int64_t child) {
  if (!bm) return fail(PA_ERR_INVALID_ARG, "pa_bm_fork: bm is NULL");
  auto it = bm->seqs.find(parent);
  if (it == bm->seqs.end()) return fail(PA_ERR_UNKNOWN_SEQ, "pa_bm_fork: parent %lld", (long long)parent);
  if (bm->seqs.count(child)) return fail(PA_ERR_SEQ_EXISTS, "pa_bm_fork: child %lld exists", (long long)child);
  pagedkv::SeqState st = it->second;  // copy of table and length
  for (int32_t b : st.table) bm->refcount[b] += 1;
  bm->seqs.emplace(child, std::move(st));
  return PA_OK;
}

pa_status pa_bm_free(pa_bm* bm, int64_t seq) {
  if (!bm) return fail(PA_ERR_INVALID_ARG, "pa_bm_free: bm is NULL");
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return fail(PA_ERR_UNKNOWN_SEQ, "pa_bm_free: seq %lld", (long long)seq);
  for (int32_t b : it->second.table) {
    if (--bm->refcount[b] == 0) bm->release(b);
  }
  bm->seqs.erase(it);
  return PA_OK;
}

int32_t pa_bm_num_free(const pa_bm* bm) { return bm ? bm->free_blocks() : 0; }
int32_t pa_bm_num_blocks(const pa_bm* bm) { return bm ? bm->num_blocks : 0; }

pa_status pa_bm_seq_len(const pa_bm* bm, int64_t seq, int32_t* len) {
  if (!bm || !len) return fail(PA_ERR_INVALID_ARG, "pa_bm_seq_len: NULL argument");
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return fail(PA_ERR_UNKNOWN_SEQ, "pa_bm_seq_len: seq %lld", (long long)seq);
  *len = it->second.len;
  return PA_OK;
}

pa_status pa_bm_refcount(const pa_bm* bm, int32_t block, int32_t* refcount) {
  if (!bm || !refcount) return fail(PA_ERR_INVALID_ARG, "pa_bm_refcount: NULL argument");
  if (block < 0 || block >= bm->num_blocks)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_refcount: block %d", block);
  *refcount = bm->refcount[block];
  return PA_OK;
}

pa_status pa_bm_block_table(const pa_bm* bm, int64_t seq, int32_t* out, int32_t cap, int32_t* n) {
  if (!bm || !n || (cap > 0 && !out) || cap < 0)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_block_table: bad argument");
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return fail(PA_ERR_UNKNOWN_SEQ, "pa_bm_block_table: seq %lld", (long long)seq);
  const auto& t = it->second.table;
  *n = (int32_t)t.size();
  if ((int32_t)t.size() > cap)
    return fail(PA_ERR_CAPACITY, "pa_bm_block_table: table %zu > cap %d", t.size(), cap);
  if (!t.empty()) std::memcpy(out, t.data(), t.size() * sizeof(int32_t));
  return PA_OK;
}

pa_status pa_bm_free_list(const pa_bm* bm, int32_t* out, int32_t cap, int32_t* n) {
  if (!bm || !n || (cap > 0 && !out) || cap < 0)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_free_list: bad argument");
  *n = bm->count;
  if (bm->count > cap) return fail(PA_ERR_CAPACITY, "pa_bm_free_list: %d > cap %d", bm->count, cap);
  for (int32_t i = 0; i < bm->count; ++i) out[i] = bm->ring[(bm->head + i) % bm->num_blocks];
  return PA_OK;
}

pa_status pa_bm_slots(const pa_bm* bm, int64_t seq, int32_t start, int32_t count, int64_t* out) {
  if (!bm || (count > 0 && !out)) return fail(PA_ERR_INVALID_ARG, "pa_bm_slots: NULL argument");
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return fail(PA_ERR_UNKNOWN_SEQ, "pa_bm_slots: seq %lld", (long long)seq);
  const auto& t = it->second.table;
  if (start < 0 || count < 0 || (int64_t)start + count > (int64_t)t.size() * PA_BLOCK_SIZE)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_slots: positions [%d, %d) outside the table", start, start + count);
  for (int32_t i = 0; i < count; ++i) {
    const int32_t p = start + i;
    out[i] = (int64_t)t[p / PA_BLOCK_SIZE] * PA_BLOCK_SIZE + p % PA_BLOCK_SIZE;
  }
  return PA_OK;
}

pa_status pa_bm_set_prefix_caching(pa_bm* bm, int32_t enable) {
  if (!bm) return fail(PA_ERR_INVALID_ARG, "pa_bm_set_prefix_caching: bm is NULL");
  if (!bm->seqs.empty() || bm->count != bm->num_blocks)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_set_prefix_caching: only on a fresh block manager");
  bm->prefix_caching = enable != 0;
  return PA_OK;
}

pa_status pa_bm_allocate_prefix(pa_bm* bm, int64_t seq, const int32_t* prompt_tokens,
                                int32_t num_prompt_tokens, int32_t num_tokens, int32_t* cached_tokens) {
  if (!bm || !cached_tokens || (num_prompt_tokens > 0 && !prompt_tokens))
    return fail(PA_ERR_INVALID_ARG, "pa_bm_allocate_prefix: NULL argument");
  if (num_prompt_tokens < 0 || num_tokens < num_prompt_tokens)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_allocate_prefix: %d prompt tokens, %d tokens", num_prompt_tokens,
                num_tokens);
  if (bm->seqs.count(seq))
    return fail(PA_ERR_SEQ_EXISTS, "pa_bm_allocate_prefix: seq %lld exists", (long long)seq);
  *cached_tokens = 0;
  if (!bm->prefix_caching) return pa_bm_allocate(bm, seq, num_tokens);
  const int32_t total = pagedkv::blocks_for(num_tokens);
  const int32_t full = num_prompt_tokens / PA_BLOCK_SIZE;
  std::vector<uint64_t> h(full);
  uint64_t parent = 0;
  for (int32_t i = 0; i < full; ++i) parent = h[i] = pagedkv::chain_hash(parent, prompt_tokens + i * PA_BLOCK_SIZE);
  // longest run of cached leading blocks
  std::vector<int32_t> hits;
  int32_t hits_evictable = 0, valid_prefix = 0;
  bool all_valid = true;
  for (int32_t i = 0; i < full; ++i) {
    auto it = bm->cache.find(h[i]);
    if (it == bm->cache.end()) break;
    const int32_t b = it->second;
    hits.push_back(b);
    if (bm->refcount[b] == 0) ++hits_evictable;
    if (all_valid && bm->valid[b]) ++valid_prefix;
    else all_valid = false;
  }
  const int32_t fresh = total - (int32_t)hits.size();
  if (fresh > bm->free_blocks() - hits_evictable)
    return fail(PA_ERR_NO_BLOCKS, "pa_bm_allocate_prefix: need %d new blocks, %d free (%d of them reused)", fresh,
                bm->free_blocks(), hits_evictable);
  pagedkv::SeqState st;
  st.table.reserve(total + 1);
  for (int32_t b : hits) {
    if (bm->refcount[b] == 0) bm->ev_remove(b);
    bm->refcount[b] += 1;
    st.table.push_back(b);
  }
  for (int32_t i = (int32_t)hits.size(); i < total; ++i) {
    const int32_t b = bm->take_fresh();
    bm->refcount[b] = 1;
    st.table.push_back(b);
    if (i < full) {
      // a new full prompt block: cached under its chain hash, valid once written
      auto it = bm->cache.find(h[i]);
      if (it != bm->cache.end()) {  // an unreachable leftover loses its entry
        bm->has_hash[it->second] = 0;
        bm->valid[it->second] = 0;
      }
      bm->cache[h[i]] = b;
      bm->block_hash[b] = h[i];
      bm->has_hash[b] = 1;
      bm->valid[b] = 0;
    }
  }
  st.len = num_tokens;
  bm->seqs.emplace(seq, std::move(st));
  *cached_tokens = valid_prefix * PA_BLOCK_SIZE;
  return PA_OK;
}

pa_status pa_bm_mark_written(pa_bm* bm, int64_t seq) {
  if (!bm) return fail(PA_ERR_INVALID_ARG, "pa_bm_mark_written: bm is NULL");
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return fail(PA_ERR_UNKNOWN_SEQ, "pa_bm_mark_written: seq %lld", (long long)seq);
  for (int32_t b : it->second.table)
    if (bm->has_hash[b]) bm->valid[b] = 1;
  return PA_OK;
}

pa_status pa_bm_evictable_list(const pa_bm* bm, int32_t* out, int32_t cap, int32_t* n) {
  if (!bm || !n || (cap > 0 && !out) || cap < 0)
    return fail(PA_ERR_INVALID_ARG, "pa_bm_evictable_list: bad argument");
  *n = bm->ev_count;
  if (bm->ev_count > cap) return fail(PA_ERR_CAPACITY, "pa_bm_evictable_list: %d > cap %d", bm->ev_count, cap);
  int32_t i = 0;
  for (int32_t b = bm->ev_head; b >= 0; b = bm->ev_next[b]) out[i++] = b;
  return PA_OK;
}

int32_t pa_bm_num_cached(const pa_bm* bm) { return bm ? (int32_t)bm->cache.size() : 0; }

pa_status pa_bm_pack(const pa_bm* bm, const int64_t* seqs, int32_t n, int32_t max_blocks,
                     int32_t* block_tables, int32_t* seq_lens, int64_t* last_slots) {
  if (!bm || n < 0 || max_blocks < 0 || (n > 0 && (!seqs || !block_tables || !seq_lens)))
    return fail(PA_ERR_INVALID_ARG, "pa_bm_pack: bad argument");
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seqs[i]);
    if (it == bm->seqs.end()) return fail(PA_ERR_UNKNOWN_SEQ, "pa_bm_pack: seq %lld", (long long)seqs[i]);
    if ((int32_t)it->second.table.size() > max_blocks)
      return fail(PA_ERR_CAPACITY, "pa_bm_pack: seq %lld has %zu blocks > %d", (long long)seqs[i],
                  it->second.table.size(), max_blocks);
  }
  for (int32_t i = 0; i < n; ++i) {
    const pagedkv::SeqState& st = bm->seqs.find(seqs[i])->second;
    int32_t* row = block_tables + (size_t)i * max_blocks;
    const int32_t nb = (int32_t)st.table.size();
    if (nb) std::memcpy(row, st.table.data(), nb * sizeof(int32_t));
    std::fill(row + nb, row + max_blocks, -1);
    seq_lens[i] = st.len;
    if (last_slots) {
      const int32_t p = st.len - 1;
      last_slots[i] = p < 0 ? -1 : (int64_t)st.table[p / PA_BLOCK_SIZE] * PA_BLOCK_SIZE + p % PA_BLOCK_SIZE;
    }
  }
  return PA_OK;
}

}  // extern "C"
