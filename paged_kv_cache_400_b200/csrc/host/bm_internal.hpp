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
};
