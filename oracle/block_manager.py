"""Integer oracle of the paged-KV block manager.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Sources:
  "如何通过PagedAttention实现LLM高性能推理：实战指南" §2.2: a free-block pool
      that starts as deque(range(max_num_blocks)); allocate(seq_id, num_tokens)
      takes ceil(num_tokens / block_size) blocks from its left end and records
      them in the sequence's page table.
  "vLLM 原理：PagedAttention 和 Continuous Batching":
      "PagedAttention 的思路" — 16 tokens per page; 500 tokens -> 32 pages,
          1000 -> 63; pages need not be contiguous.
      "工作原理" — 1. one page table per request; 2. allocate on demand: with
          500 tokens in 32 pages, the 501st token still fits page 32 and the
          513th opens page 33; 3. a finished request's pages return at once.
      "优势 / 3. 支持共享" — requests with a common prefix share its KV pages
          (parallel sampling, beam search).
  "大模型推理性能优化：PagedAttention与Continuous Batching原理与实践" §2.2 — a free
      page list; new requests take pages from it; different logical blocks may
      map to one physical page.

Readings where the pages are silent (each also listed in the design notes):
  * allocation is all-or-nothing (the deque code would fail half way);
  * freed blocks go to the free-list tail in table order;
  * a shared block carries a reference count (one per table holding it);
  * copy-on-write: appending into a non-full last block that is shared takes
    a fresh block from the free-list head, copies the whole old block into it,
    decrements the old block's count and replaces the table entry; the last
    holder (count 1) writes in place; a full last block never copies.
"""
from __future__ import annotations

from collections import deque

BLOCK_SIZE = 16


class BMError(Exception):
    """Block-manager failure; `status` is one of NO_BLOCKS, UNKNOWN_SEQ,
    SEQ_EXISTS, INVALID_ARG, CAPACITY. The state is unchanged."""

    def __init__(self, status: str, msg: str = ""):
        super().__init__(f"{status}: {msg}")
        self.status = status


def blocks_for(num_tokens: int) -> int:
    """Pages for num_tokens tokens: ceil(num_tokens / 16) (the allocator of
    "实战指南" §2.2 and the 500 -> 32 / 1000 -> 63 example of "vLLM 原理")."""
    return (num_tokens + BLOCK_SIZE - 1) // BLOCK_SIZE


class OracleBlockManager:
    def __init__(self, num_blocks: int, initial_free_order=None):
        if initial_free_order is None:
            order = list(range(num_blocks))
        else:
            order = [int(x) for x in initial_free_order]
            if sorted(order) != list(range(num_blocks)):
                raise BMError("INVALID_ARG", "initial free order is not a permutation")
        self.num_blocks = num_blocks
        self.free_list = deque(order)
        self.refcount = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}

    # -- queries -----------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free_list)

    def table(self, seq: int) -> list[int]:
        self._need(seq)
        return list(self.tables[seq])

    def seq_len(self, seq: int) -> int:
        self._need(seq)
        return self.lens[seq]

    def slots(self, seq: int, start: int, count: int) -> list[int]:
        """Slots of positions [start, start+count): table[p//16]*16 + p%16."""
        self._need(seq)
        tab = self.tables[seq]
        if start < 0 or count < 0 or start + count > len(tab) * BLOCK_SIZE:
            raise BMError("INVALID_ARG", "positions outside the table")
        return [tab[p // BLOCK_SIZE] * BLOCK_SIZE + p % BLOCK_SIZE
                for p in range(start, start + count)]

    # -- operations --------------------------------------------------------
    def allocate(self, seq: int, num_tokens: int) -> list[int]:
        if seq in self.tables:
            raise BMError("SEQ_EXISTS", str(seq))
        if num_tokens < 0:
            raise BMError("INVALID_ARG", "negative token count")
        n = blocks_for(num_tokens)
        if n > len(self.free_list):
            raise BMError("NO_BLOCKS", f"need {n}, have {len(self.free_list)}")
        blocks = [self.free_list.popleft() for _ in range(n)]
        for blk in blocks:
            self.refcount[blk] = 1
        self.tables[seq] = blocks
        self.lens[seq] = num_tokens
        return list(blocks)

    def append_slot(self, seq: int):
        """One more token for seq; returns (slot, cow_src, cow_dst)."""
        self._need(seq)
        tab = self.tables[seq]
        pos = self.lens[seq]
        row = pos % BLOCK_SIZE
        cow_src = cow_dst = -1
        if row == 0:
            # every page is full (or there is none): open a fresh page
            if not self.free_list:
                raise BMError("NO_BLOCKS", "no block for a new page")
            blk = self.free_list.popleft()
            self.refcount[blk] = 1
            tab.append(blk)
        else:
            last = tab[-1]
            if self.refcount[last] > 1:
                if not self.free_list:
                    raise BMError("NO_BLOCKS", "no block for copy-on-write")
                blk = self.free_list.popleft()
                self.refcount[blk] = 1
                self.refcount[last] -= 1
                tab[-1] = blk
                cow_src, cow_dst = last, blk
            else:
                blk = last
        self.lens[seq] = pos + 1
        return blk * BLOCK_SIZE + row, cow_src, cow_dst

    def fork(self, parent: int, child: int) -> None:
        self._need(parent)
        if child in self.tables:
            raise BMError("SEQ_EXISTS", str(child))
        tab = list(self.tables[parent])
        for blk in tab:
            self.refcount[blk] += 1
        self.tables[child] = tab
        self.lens[child] = self.lens[parent]

    def free(self, seq: int) -> None:
        self._need(seq)
        for blk in self.tables.pop(seq):
            self.refcount[blk] -= 1
            if self.refcount[blk] == 0:
                self.free_list.append(blk)
        del self.lens[seq]

    def _need(self, seq: int) -> None:
        if seq not in self.tables:
            raise BMError("UNKNOWN_SEQ", str(seq))
