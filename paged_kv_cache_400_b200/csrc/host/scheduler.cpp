// Continuous-batching step loop with recompute-mode preemption.
//
// Follows "vLLM 原理：PagedAttention 和 Continuous Batching" / "vLLM 的调度 / 调度流程"
// (each iteration: release finished requests' pages, admit waiting requests
// while pages are free, run one step, append each request's token) and
// "Preemption（抢占）" (when memory runs short a lower-priority request is
// suspended, its pages freed, and it later resumes by recomputation), and
// "大模型推理性能优化：PagedAttention与Continuous Batching原理与实践" §2.3 (a global
// request queue; finished requests leave at once; new ones join the next
// iteration). The step rules the pages leave open are fixed in pagedkv.h
// (pa_sched_create): FCFS queue, admission while ceil((prompt+generated)/16)
// blocks are free, newest-admitted running request as the preemption victim.
//
// All output arrays are member vectors reused across steps (no allocation in
// steady state once they have grown).
#include <algorithm>
#include <deque>
#include <numeric>
#include <vector>

#include "bm_internal.hpp"
#include "errors.hpp"

using pagedkv::fail;

struct pa_sched {
  pa_bm* bm = nullptr;
  int32_t n = 0;
  int32_t max_blocks = 0;
  std::vector<int32_t> arrival, prompt, output, generated;
  std::vector<int32_t> arrival_order;
  int32_t next_arrival = 0;
  std::deque<int64_t> waiting;
  std::vector<int64_t> running;
  std::vector<char> is_running;
  std::vector<int32_t> admit_len;
  std::vector<int32_t> admit_start;         // first position whose KV the admission writes
  std::vector<int32_t> tokens;              // prompt token ids (prefix caching), or empty
  std::vector<int64_t> token_offset;        // request i's prompt: tokens[token_offset[i] ...]
  // swap-mode preemption: host blocks (FIFO free list) hold preempted KV
  bool swap = false;
  int32_t host_blocks = 0;
  std::deque<int32_t> host_free;
  std::vector<std::vector<int32_t>> host_table;  // per request: its KV in host blocks, or empty
  std::vector<int32_t> swapped_len;              // tokens of KV held in host_table
  std::vector<char> swapping_in;                 // admitted this step from host blocks
  int32_t n_finished = 0;
  int32_t step_idx = 0;
  // step outputs
  std::vector<int64_t> o_running, o_decode_slots, o_prompt_seqs, o_prompt_slots;
  std::vector<int64_t> o_admitted, o_preempted, o_finished;
  std::vector<int32_t> o_seq_lens, o_block_tables, o_prompt_lens, o_cow_src, o_cow_dst, o_prompt_starts;
  int32_t o_cached_tokens = 0;
  std::vector<int32_t> o_swap_out_src, o_swap_out_dst, o_swap_in_src, o_swap_in_dst;
  std::vector<int64_t> o_swapped_out, o_swapped_in;
  std::vector<int64_t> slot_of;  // per request: slot appended this step
};

namespace {

void publish(pa_sched* s, pa_step_out* out) {
  out->num_running = (int32_t)s->o_running.size();
  out->max_blocks_per_seq = s->max_blocks;
  out->running = s->o_running.data();
  out->seq_lens = s->o_seq_lens.data();
  out->block_tables = s->o_block_tables.data();
  out->decode_slots = s->o_decode_slots.data();
  out->num_prompt_seqs = (int32_t)s->o_prompt_seqs.size();
  out->num_prompt_tokens = (int32_t)s->o_prompt_slots.size();
  out->prompt_seqs = s->o_prompt_seqs.data();
  out->prompt_lens = s->o_prompt_lens.data();
  out->prompt_slots = s->o_prompt_slots.data();
  out->num_cow = (int32_t)s->o_cow_src.size();
  out->cow_src = s->o_cow_src.data();
  out->cow_dst = s->o_cow_dst.data();
  out->num_admitted = (int32_t)s->o_admitted.size();
  out->admitted = s->o_admitted.data();
  out->num_preempted = (int32_t)s->o_preempted.size();
  out->preempted = s->o_preempted.data();
  out->num_finished = (int32_t)s->o_finished.size();
  out->finished = s->o_finished.data();
  out->num_waiting = (int32_t)s->waiting.size();
  out->num_free_blocks = s->bm->free_blocks();
  out->prompt_starts = s->o_prompt_starts.data();
  out->num_cached_tokens = s->o_cached_tokens;
  out->num_swap_out = (int32_t)s->o_swap_out_src.size();
  out->swap_out_src = s->o_swap_out_src.data();
  out->swap_out_dst = s->o_swap_out_dst.data();
  out->num_swap_in = (int32_t)s->o_swap_in_src.size();
  out->swap_in_src = s->o_swap_in_src.data();
  out->swap_in_dst = s->o_swap_in_dst.data();
  out->num_swapped_out = (int32_t)s->o_swapped_out.size();
  out->swapped_out = s->o_swapped_out.data();
  out->num_swapped_in = (int32_t)s->o_swapped_in.size();
  out->swapped_in = s->o_swapped_in.data();
}

// Preemption victim v in swap mode: when its KV was written before this step
// and none of its blocks is shared, its blocks are copied to host blocks
// (swap-out pairs, run before any other device work of the step) and it will
// come back by copying instead of recomputing. A request admitted from host
// blocks in this same step keeps its host copy. Otherwise (no swap mode, not
// enough host blocks, shared blocks, KV not yet written) it is recomputed.
pa_status swap_out_or_drop(pa_sched* s, int64_t v) {
  pa_bm* bm = s->bm;
  if (s->swapping_in[v]) {  // its KV is still in host blocks
    s->swapping_in[v] = 0;
    return PA_OK;
  }
  s->host_table[v].clear();
  if (!s->swap) return PA_OK;
  bool admitted_now = false;
  for (int64_t r : s->o_admitted) admitted_now |= (r == v);
  if (admitted_now) return PA_OK;
  auto it = bm->seqs.find(v);
  if (it == bm->seqs.end()) return fail(PA_ERR_UNKNOWN_SEQ, "pa_sched_step: victim %lld", (long long)v);
  const std::vector<int32_t>& table = it->second.table;
  if ((int32_t)table.size() > (int32_t)s->host_free.size()) return PA_OK;
  for (int32_t b : table)
    if (bm->refcount[b] != 1) return PA_OK;
  for (int32_t b : table) {
    const int32_t h = s->host_free.front();
    s->host_free.pop_front();
    s->host_table[v].push_back(h);
    s->o_swap_out_src.push_back(b);
    s->o_swap_out_dst.push_back(h);
  }
  s->swapped_len[v] = it->second.len;
  s->o_swapped_out.push_back(v);
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_sched_create(pa_bm* bm, const int32_t* arrival_step, const int32_t* prompt_len,
                          const int32_t* output_len, int32_t n_requests,
                          int32_t max_blocks_per_seq, pa_sched** out) {
  if (!out) return fail(PA_ERR_INVALID_ARG, "pa_sched_create: out is NULL");
  *out = nullptr;
  if (!bm || n_requests < 0 || max_blocks_per_seq <= 0 ||
      (n_requests > 0 && (!arrival_step || !prompt_len || !output_len)))
    return fail(PA_ERR_INVALID_ARG, "pa_sched_create: bad argument");
  for (int32_t i = 0; i < n_requests; ++i) {
    if (arrival_step[i] < 0 || prompt_len[i] < 1 || output_len[i] < 1)
      return fail(PA_ERR_INVALID_ARG, "pa_sched_create: request %d (arrival %d, prompt %d, output %d)",
                  i, arrival_step[i], prompt_len[i], output_len[i]);
    if ((int64_t)prompt_len[i] + output_len[i] > (int64_t)max_blocks_per_seq * PA_BLOCK_SIZE)
      return fail(PA_ERR_CAPACITY, "pa_sched_create: request %d needs more than %d blocks", i,
                  max_blocks_per_seq);
  }
  pa_sched* s = new pa_sched();
  s->bm = bm;
  s->n = n_requests;
  s->max_blocks = max_blocks_per_seq;
  s->arrival.assign(arrival_step, arrival_step + n_requests);
  s->prompt.assign(prompt_len, prompt_len + n_requests);
  s->output.assign(output_len, output_len + n_requests);
  s->generated.assign(n_requests, 0);
  s->is_running.assign(n_requests, 0);
  s->admit_len.assign(n_requests, 0);
  s->admit_start.assign(n_requests, 0);
  s->host_table.assign(n_requests, {});
  s->swapped_len.assign(n_requests, 0);
  s->swapping_in.assign(n_requests, 0);
  s->slot_of.assign(n_requests, -1);
  s->arrival_order.resize(n_requests);
  std::iota(s->arrival_order.begin(), s->arrival_order.end(), 0);
  std::stable_sort(s->arrival_order.begin(), s->arrival_order.end(),
                   [s](int32_t a, int32_t b) { return s->arrival[a] < s->arrival[b]; });
  *out = s;
  return PA_OK;
}

void pa_sched_destroy(pa_sched* s) { delete s; }

pa_status pa_sched_set_swap(pa_sched* s, int32_t num_host_blocks) {
  if (!s || num_host_blocks < 0) return fail(PA_ERR_INVALID_ARG, "pa_sched_set_swap: bad argument");
  if (s->step_idx != 0) return fail(PA_ERR_INVALID_ARG, "pa_sched_set_swap: only before the first step");
  s->swap = num_host_blocks > 0;
  s->host_blocks = num_host_blocks;
  s->host_free.clear();
  for (int32_t i = 0; i < num_host_blocks; ++i) s->host_free.push_back(i);
  return PA_OK;
}

pa_status pa_sched_set_prompt_tokens(pa_sched* s, const int32_t* tokens, const int64_t* offsets) {
  if (!s || !tokens || !offsets) return fail(PA_ERR_INVALID_ARG, "pa_sched_set_prompt_tokens: NULL argument");
  if (s->step_idx != 0) return fail(PA_ERR_INVALID_ARG, "pa_sched_set_prompt_tokens: only before the first step");
  if (!s->bm->prefix_caching)
    return fail(PA_ERR_INVALID_ARG, "pa_sched_set_prompt_tokens: the block manager's prefix caching is off");
  int64_t end = 0;
  for (int32_t i = 0; i < s->n; ++i) {
    if (offsets[i] < 0) return fail(PA_ERR_INVALID_ARG, "pa_sched_set_prompt_tokens: offset %d", i);
    end = std::max(end, offsets[i] + s->prompt[i]);
  }
  s->tokens.assign(tokens, tokens + end);
  s->token_offset.assign(offsets, offsets + s->n);
  return PA_OK;
}

pa_status pa_sched_step(pa_sched* s, pa_step_out* out) {
  if (!s || !out) return fail(PA_ERR_INVALID_ARG, "pa_sched_step: NULL argument");
  pa_bm* bm = s->bm;
  const int32_t step = s->step_idx++;
  s->o_running.clear();
  s->o_decode_slots.clear();
  s->o_prompt_seqs.clear();
  s->o_prompt_slots.clear();
  s->o_admitted.clear();
  s->o_preempted.clear();
  s->o_finished.clear();
  s->o_seq_lens.clear();
  s->o_block_tables.clear();
  s->o_prompt_lens.clear();
  s->o_cow_src.clear();
  s->o_cow_dst.clear();
  s->o_prompt_starts.clear();
  s->o_cached_tokens = 0;
  s->o_swap_out_src.clear();
  s->o_swap_out_dst.clear();
  s->o_swap_in_src.clear();
  s->o_swap_in_dst.clear();
  s->o_swapped_out.clear();
  s->o_swapped_in.clear();
  out->step = step;

  // 1. retire requests that generated all their tokens; pages return at once
  {
    size_t keep = 0;
    for (size_t i = 0; i < s->running.size(); ++i) {
      const int64_t r = s->running[i];
      if (s->generated[r] >= s->output[r]) {
        pa_status st = pa_bm_free(bm, r);
        if (st != PA_OK) return st;
        s->is_running[r] = 0;
        s->o_finished.push_back(r);
      } else {
        s->running[keep++] = r;
      }
    }
    s->running.resize(keep);
    s->n_finished += (int32_t)s->o_finished.size();
  }

  // 2. arrivals join the waiting tail in (arrival step, id) order
  while (s->next_arrival < s->n && s->arrival[s->arrival_order[s->next_arrival]] <= step) {
    s->waiting.push_back(s->arrival_order[s->next_arrival]);
    ++s->next_arrival;
  }

  // 3. admit from the head while its pages fit (first come, first served);
  //    with prompt tokens, the cached leading blocks of the prompt are reused
  //    and only the rest of its KV is (re)written
  while (!s->waiting.empty()) {
    const int64_t r = s->waiting.front();
    const int32_t total = s->prompt[r] + s->generated[r];
    int32_t cached = 0;
    pa_status st;
    const bool from_host = !s->host_table[r].empty();
    if (from_host) {
      // swapped out earlier: fresh device blocks, KV copied back (no recompute)
      st = pagedkv::blocks_for(total) > bm->free_blocks() ? PA_ERR_NO_BLOCKS : pa_bm_allocate(bm, r, total);
      cached = total;
    } else if (s->tokens.empty()) {
      st = pagedkv::blocks_for(total) > bm->free_blocks() ? PA_ERR_NO_BLOCKS : pa_bm_allocate(bm, r, total);
    } else {
      st = pa_bm_allocate_prefix(bm, r, s->tokens.data() + s->token_offset[r], s->prompt[r], total, &cached);
    }
    if (st == PA_ERR_NO_BLOCKS) {
      if (s->running.empty())
        return fail(PA_ERR_NO_BLOCKS, "pa_sched_step: request %lld can never fit (%d tokens, %d blocks)",
                    (long long)r, total, bm->num_blocks);
      break;
    }
    if (st != PA_OK) return st;
    s->waiting.pop_front();
    s->running.push_back(r);
    s->is_running[r] = 1;
    s->o_admitted.push_back(r);
    s->admit_len[r] = total;
    s->admit_start[r] = cached;
    s->swapping_in[r] = from_host ? 1 : 0;
  }

  // 4. grow every running request by one slot; preempt the newest on shortage
  for (size_t i = 0; i < s->running.size(); ++i) {
    const int64_t r = s->running[i];
    bool stop = false;
    for (;;) {
      int64_t slot;
      int32_t cs, cd;
      pa_status st = pa_bm_append_slot(bm, r, &slot, &cs, &cd);
      if (st == PA_OK) {
        s->slot_of[r] = slot;
        if (cs >= 0) {
          s->o_cow_src.push_back(cs);
          s->o_cow_dst.push_back(cd);
        }
        break;
      }
      if (st != PA_ERR_NO_BLOCKS) return st;
      const int64_t victim = s->running.back();
      s->running.pop_back();
      if ((st = swap_out_or_drop(s, victim)) != PA_OK) return st;
      st = pa_bm_free(bm, victim);
      if (st != PA_OK) return st;
      s->is_running[victim] = 0;
      s->waiting.push_front(victim);
      s->o_preempted.push_back(victim);
      if (victim == r) {
        if (s->running.empty())
          return fail(PA_ERR_NO_BLOCKS, "pa_sched_step: request %lld cannot grow alone", (long long)r);
        stop = true;
        break;
      }
    }
    if (stop) break;
  }

  // 5. describe the step's device work
  const size_t nr = s->running.size();
  s->o_running.assign(s->running.begin(), s->running.end());
  s->o_seq_lens.resize(nr);
  s->o_decode_slots.resize(nr);
  s->o_block_tables.resize(nr * (size_t)s->max_blocks);
  if (nr) {
    pa_status st = pa_bm_pack(bm, s->o_running.data(), (int32_t)nr, s->max_blocks,
                              s->o_block_tables.data(), s->o_seq_lens.data(), nullptr);
    if (st != PA_OK) return st;
  }
  for (size_t i = 0; i < nr; ++i) s->o_decode_slots[i] = s->slot_of[s->running[i]];
  for (int64_t r : s->o_admitted) {
    if (!s->is_running[r]) continue;  // admitted, then preempted in the same step
    if (s->swapping_in[r]) {
      // KV comes back from host blocks; those blocks are free after this step
      auto it = bm->seqs.find(r);
      if (it == bm->seqs.end()) return fail(PA_ERR_UNKNOWN_SEQ, "pa_sched_step: swapped-in %lld", (long long)r);
      const std::vector<int32_t>& dev = it->second.table;  // may hold this step's new block too
      const std::vector<int32_t>& host = s->host_table[r];
      for (size_t i = 0; i < host.size(); ++i) {
        s->o_swap_in_src.push_back(host[i]);
        s->o_swap_in_dst.push_back(dev[i]);
        s->host_free.push_back(host[i]);
      }
      s->host_table[r].clear();
      s->swapping_in[r] = 0;
      s->o_swapped_in.push_back(r);
      continue;
    }
    const int32_t n = s->admit_len[r];
    const int32_t start = s->admit_start[r];
    s->o_prompt_seqs.push_back(r);
    s->o_prompt_lens.push_back(n);
    s->o_prompt_starts.push_back(start);
    s->o_cached_tokens += start;
    const size_t at = s->o_prompt_slots.size();
    s->o_prompt_slots.resize(at + (n - start));
    pa_status st = pa_bm_slots(bm, r, start, n - start, s->o_prompt_slots.data() + at);
    if (st != PA_OK) return st;
    // this step's device work writes its KV: its cached blocks become reusable
    if (!s->tokens.empty() && (st = pa_bm_mark_written(bm, r)) != PA_OK) return st;
  }

  // 6. every running request generated one token
  for (int64_t r : s->running) s->generated[r] += 1;

  out->done = (s->n_finished == s->n) ? 1 : 0;
  publish(s, out);
  return PA_OK;
}

}  // extern "C"
