"""Oracle: plain, slow, CPU-only restatement of what the paged KV-cache path computes.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or link
anything here; only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline
and reference legs use it. It shares no code with the CUDA path
(paged_kv_cache_400_b200/): it imports numpy (and, in the pins, torch CPU ops as
an independent library check) and nothing else of this repository.

Modules
  attention      fp64 gather-through-block-table + textbook softmax attention,
                 the split-KV partition/merge reading, the literal cache append
                 and block copy.
  block_manager  integer block manager: FIFO free list, page tables, refcounts,
                 fork, copy-on-write of a shared partial last block, free.
  scheduler      integer continuous-batching step loop with recompute and
                 swap-mode preemption.

Sources: three web pages on PagedAttention —
  "大模型推理性能优化：PagedAttention与Continuous Batching原理与实践",
  "vLLM 原理：PagedAttention 和 Continuous Batching",
  "如何通过PagedAttention实现LLM高性能推理：实战指南".
Each function names the page section it follows.

Parity status: every function here is pinned by tests/test_oracle_pins.py and
tests/test_oracle_scheduler.py (swap mode included: hand-worked event lists for
each swap rule and a host-block accounting invariant on a random trace); the
scheduler's step-order details beyond the pinned policy points are checked by
invariants and by hand-written event lists on tiny traces only.
"""
