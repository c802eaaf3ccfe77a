"""Integer oracle of the continuous-batching step loop with recompute preemption.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Sources:
  "vLLM 原理：PagedAttention 和 Continuous Batching", "vLLM 的调度 / 调度流程":
      each iteration 1) releases the pages of finished requests and drops them
      from the running set, 2) admits waiting requests while free pages exist,
      allocating their pages, 3) runs one forward step over the running set,
      4) appends each request's new token to its KV cache.
      "Preemption（抢占）": when memory runs short a lower-priority request is
      suspended, its pages freed, and it resumes later by recomputation or,
      in swap mode, from a copy of its KV in CPU memory.
      "Continuous Batching": requests join as they arrive and leave as soon as
      they finish.
  "大模型推理性能优化：PagedAttention与Continuous Batching原理与实践" §2.3: a global
      request queue checked at every decode iteration; finished requests leave
      at once and free their pages; new requests join the next iteration.

Readings where the pages are silent or loose (listed in the design notes):
  * queue discipline is first come, first served: arrivals join the tail in
    (arrival step, id) order and admission takes the head (the printed loop's
    list pop would take the newest; the prose describes a request queue);
  * "has free pages" means the free list holds ceil((prompt + generated) / 16)
    blocks for the head request; admission stops at the first that does not fit;
  * the phase order within a step is retire, arrive, admit, grow, (device
    work), then generated += 1; a request admitted in a step decodes in it;
  * the preemption victim ("lower priority") is the most recently admitted
    running request; it goes back to the waiting head keeping its generated
    count; if the victim is the request that is growing, it is preempted and
    the grow phase ends (an error if nothing else is running: the pool cannot
    hold that request);
  * prompt K/V is (re)written only for requests admitted this step that are
    still running at its end;
  * swap mode: a victim whose KV was written before the step and whose
    blocks are not shared is copied to host blocks (FIFO host free list)
    instead of being dropped, and copied back into fresh blocks when admitted
    again; its host blocks are free again after that step; victims that do
    not qualify or find too few host blocks are recomputed;
  * with prompt token ids (prefix caching), admission allocates through the
    block manager's prefix cache and the prompt K/V is written from the first
    position not covered by already-written cached blocks; the blocks of
    requests admitted this step become reusable at its end.
"""
from __future__ import annotations

from collections import deque

from .block_manager import BMError, OracleBlockManager, blocks_for


class OracleScheduler:
    def __init__(self, bm: OracleBlockManager, arrival_step, prompt_len, output_len,
                 max_blocks_per_seq: int):
        n = len(arrival_step)
        if not (len(prompt_len) == n and len(output_len) == n):
            raise BMError("INVALID_ARG", "request arrays differ in length")
        for i in range(n):
            if arrival_step[i] < 0 or prompt_len[i] < 1 or output_len[i] < 1:
                raise BMError("INVALID_ARG", f"request {i}")
            if blocks_for(prompt_len[i] + output_len[i]) > max_blocks_per_seq:
                raise BMError("CAPACITY", f"request {i} exceeds the table width")
        self.bm = bm
        self.arrival = [int(x) for x in arrival_step]
        self.prompt = [int(x) for x in prompt_len]
        self.output = [int(x) for x in output_len]
        self.max_blocks = max_blocks_per_seq
        self.n = n
        self.generated = [0] * n
        self.arrival_order = sorted(range(n), key=lambda i: (self.arrival[i], i))
        self.next_arrival = 0
        self.waiting: deque[int] = deque()
        self.running: list[int] = []
        self.n_finished = 0
        self.step_idx = 0
        self.tokens = None   # per-request prompt token ids when prefix caching is used
        # swap-mode preemption ("vLLM 原理" / "Preemption（抢占）": Swap mode moves the
        # KV cache to the CPU; "PagedAttention与Continuous Batching原理与实践" §3.4 --swap-space)
        self.swap = False
        self.host_free: deque[int] = deque()
        self.host_table: dict[int, list[int]] = {}
        self.swapping_in: set[int] = set()

    def set_swap(self, num_host_blocks: int) -> None:
        if self.step_idx != 0 or num_host_blocks < 0:
            raise BMError("INVALID_ARG", "before the first step")
        self.swap = num_host_blocks > 0
        self.host_free = deque(range(num_host_blocks))

    def set_prompt_tokens(self, tokens) -> None:
        """Prompt token ids per request; admission then reuses cached prompt
        blocks (the block manager's prefix caching must be on)."""
        if self.step_idx != 0 or not self.bm.prefix_caching:
            raise BMError("INVALID_ARG", "before the first step, with prefix caching on")
        self.tokens = [list(t)[:self.prompt[i]] for i, t in enumerate(tokens)]

    def step(self) -> dict:
        s = self.step_idx
        self.step_idx += 1
        bm = self.bm

        # 1. retire finished requests, freeing their pages at once
        finished = [r for r in self.running if self.generated[r] >= self.output[r]]
        for r in finished:
            bm.free(r)
        self.running = [r for r in self.running if self.generated[r] < self.output[r]]
        self.n_finished += len(finished)

        # 2. arrivals join the waiting tail
        while (self.next_arrival < self.n
               and self.arrival[self.arrival_order[self.next_arrival]] <= s):
            self.waiting.append(self.arrival_order[self.next_arrival])
            self.next_arrival += 1

        # 3. admit from the head while its pages fit
        admitted = []
        admit_len = {}
        admit_start = {}
        while self.waiting:
            r = self.waiting[0]
            total = self.prompt[r] + self.generated[r]
            from_host = bool(self.host_table.get(r))
            try:
                if from_host:
                    # swapped out earlier: its KV is copied back, nothing recomputed
                    if blocks_for(total) > bm.num_free():
                        raise BMError("NO_BLOCKS", "")
                    bm.allocate(r, total)
                    start = total
                elif self.tokens is None:
                    if blocks_for(total) > bm.num_free():
                        raise BMError("NO_BLOCKS", "")
                    bm.allocate(r, total)
                    start = 0
                else:
                    start = bm.allocate_prefix(r, self.tokens[r], total)
            except BMError as e:
                if e.status != "NO_BLOCKS":
                    raise
                if not self.running:
                    raise BMError("NO_BLOCKS", f"request {r} can never fit")
                break
            self.waiting.popleft()
            self.running.append(r)
            admitted.append(r)
            admit_len[r] = total
            admit_start[r] = start
            if from_host:
                self.swapping_in.add(r)
            else:
                self.swapping_in.discard(r)

        # 4. grow every running request by one slot, preempting from the tail
        decode_slot = {}
        cow = []
        preempted = []
        swap_out, swapped_out = [], []

        def swap_out_or_drop(v):
            """Swap-mode victim: copy its blocks to host blocks when its KV was
            written before this step and no block is shared; a request that
            came from host blocks this step keeps its host copy."""
            if v in self.swapping_in:
                self.swapping_in.discard(v)
                return
            self.host_table.pop(v, None)
            if not self.swap or v in admitted:
                return
            table = bm.table(v)
            if len(table) > len(self.host_free) or any(bm.refcount[b] != 1 for b in table):
                return
            host = [self.host_free.popleft() for _ in table]
            self.host_table[v] = host
            swap_out.extend(zip(table, host))
            swapped_out.append(v)

        i = 0
        stop = False
        while i < len(self.running) and not stop:
            r = self.running[i]
            while True:
                try:
                    slot, cs, cd = bm.append_slot(r)
                except BMError as e:
                    if e.status != "NO_BLOCKS":
                        raise
                    victim = self.running.pop()
                    swap_out_or_drop(victim)
                    bm.free(victim)
                    self.waiting.appendleft(victim)
                    preempted.append(victim)
                    if victim == r:
                        if not self.running:
                            raise BMError("NO_BLOCKS", f"request {r} cannot grow alone")
                        stop = True
                        break
                    continue
                decode_slot[r] = slot
                if cs >= 0:
                    cow.append((cs, cd))
                break
            i += 1

        # 5. the step's device work, described by index arrays
        running = list(self.running)
        still = set(running)
        swap_in, swapped_in = [], []
        for r in admitted:
            if r in still and r in self.swapping_in:
                host = self.host_table.pop(r)
                swap_in.extend(zip(host, bm.table(r)))
                self.host_free.extend(host)       # free once this step's copies are queued
                self.swapping_in.discard(r)
                swapped_in.append(r)
        prompt_seqs = [r for r in admitted if r in still and r not in swapped_in]
        prompt_slots = []
        for r in prompt_seqs:
            prompt_slots.extend(bm.slots(r, admit_start[r], admit_len[r] - admit_start[r]))
            if self.tokens is not None:
                bm.mark_written(r)   # this step writes its KV: its cached blocks become reusable
        tables = []
        for r in running:
            tab = bm.table(r)
            tables.append(tab + [-1] * (self.max_blocks - len(tab)))

        # 6. every running request generated one token
        for r in running:
            self.generated[r] += 1

        done = (self.n_finished == self.n)
        return {
            "step": s,
            "done": int(done),
            "running": running,
            "seq_lens": [bm.seq_len(r) for r in running],
            "block_tables": tables,
            "decode_slots": [decode_slot[r] for r in running],
            "prompt_seqs": prompt_seqs,
            "prompt_lens": [admit_len[r] for r in prompt_seqs],
            "prompt_starts": [admit_start[r] for r in prompt_seqs],
            "num_cached_tokens": sum(admit_start[r] for r in prompt_seqs),
            "prompt_slots": prompt_slots,
            "cow": cow,
            "admitted": admitted,
            "preempted": preempted,
            "finished": finished,
            "num_waiting": len(self.waiting),
            "num_free_blocks": bm.num_free(),
            "swap_out": swap_out,
            "swap_in": swap_in,
            "swapped_out": swapped_out,
            "swapped_in": swapped_in,
        }
