// Internal state of the host block manager (shared by the scheduler).
#pragma once

#include <cstdint>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"

namespace pagedkv {

// ceil(num_tokens / 16): pages for num_tokens tokens.
inline int32_t blocks_for(int32_t num_tokens) {
  return (num_tokens + PA_BLOCK_SIZE - 1) / PA_BLOCK_SIZE;
}

struct SeqState {
  std::vector<int32_t> table;  // logical page i -> physical block
  int32_t len = 0;             // tokens of KV held
};

}  // namespace pagedkv

struct pa_bm {
  int32_t num_blocks = 0;
  // FIFO free list as a ring buffer: entries ring[(head + i) % num_blocks],
  // i in [0, count), head first.
  std::vector<int32_t> ring;
  int32_t head = 0;
  int32_t count = 0;
  std::vector<int32_t> refcount;
  std::unordered_map<int64_t, pagedkv::SeqState> seqs;

  // ---- prefix caching (off unless enabled) --------------------------------
  // A full prompt block may carry the chained hash of the prompt up to its end;
  // `cache` maps such hashes to blocks. A hashed block whose KV has been
  // written (valid) and whose refcount drops to 0 goes to the evictable list
  // (least recently released first) instead of the free list; a fresh block is
  // taken from the free list, else by evicting the evictable head.
  bool prefix_caching = false;
  std::vector<uint64_t> block_hash;
  std::vector<uint8_t> has_hash;
  std::vector<uint8_t> valid;
  std::unordered_map<uint64_t, int32_t> cache;
  std::vector<int32_t> ev_prev, ev_next;
  std::vector<uint8_t> in_ev;
  int32_t ev_head = -1, ev_tail = -1, ev_count = 0;

  int32_t pop_front() {
    int32_t b = ring[head];
    head = (head + 1 == num_blocks) ? 0 : head + 1;
    --count;
    return b;
  }
  void push_back(int32_t b) {
    int32_t at = head + count;
    if (at >= num_blocks) at -= num_blocks;
    ring[at] = b;
    ++count;
  }

  int32_t free_blocks() const { return count + ev_count; }

  void ev_push_back(int32_t b) {
    ev_prev[b] = ev_tail;
    ev_next[b] = -1;
    if (ev_tail >= 0) ev_next[ev_tail] = b;
    else ev_head = b;
    ev_tail = b;
    in_ev[b] = 1;
    ++ev_count;
  }
  void ev_remove(int32_t b) {
    const int32_t p = ev_prev[b], n = ev_next[b];
    if (p >= 0) ev_next[p] = n;
    else ev_head = n;
    if (n >= 0) ev_prev[n] = p;
    else ev_tail = p;
    in_ev[b] = 0;
    --ev_count;
  }
  void unregister(int32_t b) {
    if (!has_hash[b]) return;
    auto it = cache.find(block_hash[b]);
    if (it != cache.end() && it->second == b) cache.erase(it);
    has_hash[b] = 0;
    valid[b] = 0;
  }
  // A block for new content (the caller checked free_blocks() > 0).
  int32_t take_fresh() {
    if (count > 0) return pop_front();
    const int32_t b = ev_head;
    ev_remove(b);
    unregister(b);
    return b;
  }
  // Refcount of b reached 0.
  void release(int32_t b) {
    if (has_hash[b] && valid[b]) {
      ev_push_back(b);
    } else {
      unregister(b);
      push_back(b);
    }
  }
};

namespace pagedkv {

// SplitMix64's output function (Stafford's "Mix13" finaliser).
inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Chained hash of a full block: the hash of everything before it (`parent`,
// 0 for the first block) and its 16 token ids.
inline uint64_t chain_hash(uint64_t parent, const int32_t* tokens) {
  uint64_t x = mix64(parent ^ 0x9E3779B97F4A7C15ull);
  for (int j = 0; j < PA_BLOCK_SIZE; ++j) x = mix64(x ^ (uint64_t)(uint32_t)tokens[j]);
  return x;
}

}  // namespace pagedkv
