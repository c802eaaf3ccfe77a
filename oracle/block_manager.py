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

Prefix caching ("PagedAttention与Continuous Batching原理与实践" §3.4: with
--enable-prefix-caching, requests sharing a prompt prefix such as a system
prompt avoid recomputing it) is read as: full prompt blocks are keyed by the
chained hash of (previous blocks' hash, their 16 token ids); allocation shares
the longest run of cached leading blocks; a cached block whose refcount drops
to 0 stays findable on an evictable list (least recently released first) and
a fresh block comes from the free list, else by evicting that list's head; a
cached block may be reused only after its KV was written (mark_written).

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

from collections import OrderedDict, deque

BLOCK_SIZE = 16
_M64 = (1 << 64) - 1


class BMError(Exception):
    """Block-manager failure; `status` is one of NO_BLOCKS, UNKNOWN_SEQ,
    SEQ_EXISTS, INVALID_ARG, CAPACITY. The state is unchanged."""

    def __init__(self, status: str, msg: str = ""):
        super().__init__(f"{status}: {msg}")
        self.status = status


def mix64(z: int) -> int:
    """SplitMix64's output function (Stafford's "Mix13" 64-bit finaliser)."""
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def chain_hash(parent: int, tokens) -> int:
    """Hash of a full block of 16 token ids given the hash of the prompt before
    it (0 for the first block): one mix of the parent, then one per token."""
    x = mix64(parent ^ 0x9E3779B97F4A7C15)
    for t in tokens:
        x = mix64(x ^ (int(t) & 0xFFFFFFFF))
    return x


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
        # prefix caching ("PagedAttention与Continuous Batching原理与实践" §3.4,
        # --enable-prefix-caching: a common prompt prefix is not recomputed)
        self.prefix_caching = False
        self.block_hash: dict[int, int] = {}   # block -> chained hash
        self.valid: set[int] = set()           # hashed blocks whose KV was written
        self.cache: dict[int, int] = {}        # hash -> block
        self.evictable: OrderedDict[int, None] = OrderedDict()  # refcount-0 cached, oldest first

    # -- queries -----------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free_list) + len(self.evictable)

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
        if n > self.num_free():
            raise BMError("NO_BLOCKS", f"need {n}, have {self.num_free()}")
        blocks = [self._take_fresh() for _ in range(n)]
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
            if not self.num_free():
                raise BMError("NO_BLOCKS", "no block for a new page")
            blk = self._take_fresh()
            self.refcount[blk] = 1
            tab.append(blk)
        else:
            last = tab[-1]
            if self.refcount[last] > 1:
                if not self.num_free():
                    raise BMError("NO_BLOCKS", "no block for copy-on-write")
                blk = self._take_fresh()
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
                self._release(blk)
        del self.lens[seq]

    # -- prefix caching -----------------------------------------------------
    def set_prefix_caching(self, enable: bool) -> None:
        if self.tables or len(self.free_list) != self.num_blocks:
            raise BMError("INVALID_ARG", "only on a fresh block manager")
        self.prefix_caching = bool(enable)

    def allocate_prefix(self, seq: int, prompt_tokens, num_tokens: int) -> int:
        """allocate() that shares the longest run of cached leading full blocks
        of the prompt; returns the number of leading tokens whose KV is already
        written (16 x the leading shared blocks that are valid)."""
        if not self.prefix_caching:
            self.allocate(seq, num_tokens)
            return 0
        if seq in self.tables:
            raise BMError("SEQ_EXISTS", str(seq))
        prompt = list(prompt_tokens)
        if num_tokens < len(prompt):
            raise BMError("INVALID_ARG", "fewer tokens than the prompt")
        full = len(prompt) // BLOCK_SIZE
        hashes, parent = [], 0
        for i in range(full):
            parent = chain_hash(parent, prompt[i * BLOCK_SIZE:(i + 1) * BLOCK_SIZE])
            hashes.append(parent)
        hits = []
        for h in hashes:
            if h not in self.cache:
                break
            hits.append(self.cache[h])
        valid_prefix = 0
        for blk in hits:
            if blk not in self.valid:
                break
            valid_prefix += 1
        total = blocks_for(num_tokens)
        fresh = total - len(hits)
        reused_free = sum(1 for blk in hits if self.refcount[blk] == 0)
        if fresh > self.num_free() - reused_free:
            raise BMError("NO_BLOCKS", f"need {fresh} new blocks")
        table = []
        for blk in hits:
            if self.refcount[blk] == 0:
                del self.evictable[blk]
            self.refcount[blk] += 1
            table.append(blk)
        for i in range(len(hits), total):
            blk = self._take_fresh()
            self.refcount[blk] = 1
            table.append(blk)
            if i < full:
                old = self.cache.get(hashes[i])
                if old is not None:          # an unreachable leftover loses its entry
                    self.block_hash.pop(old, None)
                    self.valid.discard(old)
                self.cache[hashes[i]] = blk
                self.block_hash[blk] = hashes[i]
                self.valid.discard(blk)
        self.tables[seq] = table
        self.lens[seq] = num_tokens
        return valid_prefix * BLOCK_SIZE

    def mark_written(self, seq: int) -> None:
        self._need(seq)
        for blk in self.tables[seq]:
            if blk in self.block_hash:
                self.valid.add(blk)

    def _unregister(self, blk: int) -> None:
        h = self.block_hash.pop(blk, None)
        if h is not None and self.cache.get(h) == blk:
            del self.cache[h]
        self.valid.discard(blk)

    def _take_fresh(self) -> int:
        """A block for new content: the free list's head, else the least
        recently released cached block (evicted)."""
        if self.free_list:
            return self.free_list.popleft()
        blk, _ = self.evictable.popitem(last=False)
        self._unregister(blk)
        return blk

    def _release(self, blk: int) -> None:
        """Refcount of blk reached 0: a written cached block stays findable on
        the evictable list; anything else returns to the free list."""
        if blk in self.block_hash and blk in self.valid:
            self.evictable[blk] = None
        else:
            self._unregister(blk)
            self.free_list.append(blk)

    def _need(self, seq: int) -> None:
        if seq not in self.tables:
            raise BMError("UNKNOWN_SEQ", str(seq))
