"""Automatic prefix caching (CPU): the oracle against its rules and published
hash vectors, and the C++ block manager / scheduler against the oracle.

The pages' claim ("PagedAttention与Continuous Batching原理与实践" §3.4, --enable-
prefix-caching): requests sharing a prompt prefix, such as one system prompt,
do not recompute it. Here that means they share its full KV blocks and only
the KV after the cached prefix is written.
"""
import json
import os

import numpy as np
import pytest

from oracle.block_manager import BMError, OracleBlockManager, blocks_for, chain_hash, mix64
from oracle.scheduler import OracleScheduler
from paged_kv_cache_400_b200 import binding as bd

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "splitmix64.json")
GAMMA = 0x9E3779B97F4A7C15


def test_mix64_matches_published_splitmix64_outputs():
    for case in json.load(open(GOLDEN))["cases"]:
        state = case["seed"]
        for want in case["outputs"]:
            state = (state + GAMMA) & ((1 << 64) - 1)
            assert mix64(state) == int(want, 0)


def cached_bm(n=64):
    bm = OracleBlockManager(n)
    bm.set_prefix_caching(True)
    return bm


def toks(rng, n, vocab=50):
    return [int(x) for x in rng.integers(0, vocab, size=n)]


def test_same_prompt_shares_full_blocks_once_written():
    rng = np.random.default_rng(0)
    prompt = toks(rng, 50)                 # 3 full blocks + 2 tokens
    bm = cached_bm()
    assert bm.allocate_prefix(1, prompt, 51) == 0
    # not yet written: a second request may share the blocks but must write them
    assert bm.allocate_prefix(2, prompt, 50) == 0
    assert bm.table(2)[:3] == bm.table(1)[:3]
    bm.mark_written(1)
    assert bm.allocate_prefix(3, prompt, 60) == 48
    t1, t3 = bm.table(1), bm.table(3)
    assert t3[:3] == t1[:3] and t3[3] != t1[3]          # the partial block stays private
    assert [bm.refcount[b] for b in t1[:3]] == [3, 3, 3]
    assert bm.num_free() == 64 - 3 - 3                  # 3 shared + 3 private last blocks


def test_only_equal_prefixes_share():
    rng = np.random.default_rng(1)
    base = toks(rng, 64)
    bm = cached_bm()
    bm.allocate_prefix(1, base, 64)
    bm.mark_written(1)
    fork = base[:40] + toks(rng, 24)                    # first 40 tokens equal
    assert bm.allocate_prefix(2, fork, 64) == 32
    assert bm.table(2)[:2] == bm.table(1)[:2] and bm.table(2)[2] != bm.table(1)[2]
    shifted = [7] + base[:63]                           # same tokens, other positions
    assert bm.allocate_prefix(3, shifted, 64) == 0
    assert not set(bm.table(3)) & set(bm.table(1))
    # the hash of a block depends on every earlier block
    assert chain_hash(0, base[16:32]) != chain_hash(chain_hash(0, base[:16]), base[16:32])


def test_freed_blocks_stay_cached_until_evicted_lru():
    rng = np.random.default_rng(2)
    a, b = toks(rng, 32), toks(rng, 32)
    bm = cached_bm(6)
    bm.allocate_prefix(1, a, 32)
    bm.allocate_prefix(2, b, 32)
    bm.mark_written(1)
    bm.mark_written(2)
    bm.free(1)
    bm.free(2)
    assert bm.num_free() == 6
    ev = list(bm.evictable)
    assert len(ev) == 4 and len(bm.free_list) == 2
    # a hit takes its blocks back from the evictable list, no free block used
    assert bm.allocate_prefix(3, a, 32) == 32
    assert len(bm.free_list) == 2 and list(bm.evictable) == ev[2:]
    # new content uses the free list first, then evicts the least recently freed
    c = toks(rng, 64)
    bm.allocate_prefix(4, c, 64)                        # needs 4: 2 free + 2 evicted
    assert list(bm.evictable) == [] and ev[2] in bm.table(4) and ev[3] in bm.table(4)
    bm.free(3)
    assert bm.allocate_prefix(5, b, 32) == 0            # b's blocks were evicted


def test_unwritten_blocks_leave_no_cache_and_allocation_is_atomic():
    rng = np.random.default_rng(3)
    p = toks(rng, 48)
    bm = cached_bm(4)
    bm.allocate_prefix(1, p, 48)
    bm.free(1)                                          # never written
    assert len(bm.cache) == 0 and len(bm.free_list) == 4
    bm.allocate_prefix(2, p, 48)
    bm.mark_written(2)
    state = (list(bm.free_list), list(bm.evictable), dict(bm.cache), list(bm.refcount))
    with pytest.raises(BMError) as e:
        bm.allocate_prefix(3, p, 48 + 32)               # 3 shared + 2 fresh, only 1 free
    assert e.value.status == "NO_BLOCKS"
    assert (list(bm.free_list), list(bm.evictable), dict(bm.cache), list(bm.refcount)) == state


def test_scheduler_writes_only_the_uncached_suffix():
    rng = np.random.default_rng(4)
    system = toks(rng, 40)
    prompts = [system + toks(rng, 10 + 3 * i) for i in range(5)]
    bm = cached_bm(200)
    s = OracleScheduler(bm, [0, 1, 1, 2, 2], [len(p) for p in prompts], [4] * 5, 16)
    s.set_prompt_tokens(prompts)
    out = [s.step() for _ in range(3)]
    assert out[0]["prompt_starts"] == [0]
    assert out[1]["prompt_starts"] == [32, 32] and out[2]["prompt_starts"] == [32, 32]
    for o in out[1:]:
        assert len(o["prompt_slots"]) == sum(n - 32 for n in o["prompt_lens"])


# ---------------------------------------------------------------------------
# C++ against the oracle
# ---------------------------------------------------------------------------
def same(obm, cbm, seqs):
    assert obm.num_free() == cbm.num_free()
    assert list(obm.free_list) == cbm.free_list()
    assert list(obm.evictable) == cbm.evictable_list()
    assert len(obm.cache) == cbm.num_cached()
    for q in seqs:
        assert obm.table(q) == cbm.block_table(q) and obm.seq_len(q) == cbm.seq_len(q)
    for b in range(obm.num_blocks):
        assert obm.refcount[b] == cbm.refcount(b)


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_random_operations_with_prefix_caching(seed):
    rng = np.random.default_rng(50 + seed)
    N = 96
    obm, cbm = OracleBlockManager(N), bd.BlockManager(N)
    obm.set_prefix_caching(True)
    cbm.set_prefix_caching(True)
    systems = [toks(rng, int(rng.integers(16, 70)), vocab=20) for _ in range(4)]
    live, nxt = [], 0
    for i in range(3000):
        op = int(rng.integers(0, 6))
        if op <= 1:
            prompt = systems[int(rng.integers(0, 4))] + toks(rng, int(rng.integers(0, 40)), vocab=20)
            extra = int(rng.integers(0, 20))
            try:
                o = obm.allocate_prefix(nxt, prompt, len(prompt) + extra)
            except BMError as e:
                o = e.status
            try:
                c = cbm.allocate_prefix(nxt, prompt, len(prompt) + extra)
            except bd.PagedKVError as e:
                c = e.status
            assert o == c, (i, o, c)
            if not isinstance(o, str):
                live.append(nxt)
            nxt += 1
        elif op == 2 and live:
            q = live[int(rng.integers(0, len(live)))]
            obm.mark_written(q)
            cbm.mark_written(q)
        elif op == 3 and live:
            q = live[int(rng.integers(0, len(live)))]
            try:
                o = obm.append_slot(q)
            except BMError as e:
                o = e.status
            try:
                c = cbm.append_slot(q)
            except bd.PagedKVError as e:
                c = e.status
            assert o == c
        elif op == 4 and live:
            q = live[int(rng.integers(0, len(live)))]
            obm.fork(q, nxt)
            cbm.fork(q, nxt)
            live.append(nxt)
            nxt += 1
        elif op == 5 and live:
            q = live.pop(int(rng.integers(0, len(live))))
            obm.free(q)
            cbm.free(q)
        if i % 50 == 0:
            same(obm, cbm, live)
    same(obm, cbm, live)


def test_prefix_trace_replay_is_identical():
    from paged_kv_cache_400_b200 import workloads as wl
    case = wl.prefix_trace_case(seed=2, n_requests=400, rate=20.0, num_blocks=3000, num_layers=1)
    obm, cbm = OracleBlockManager(case.num_blocks), bd.BlockManager(case.num_blocks)
    obm.set_prefix_caching(True)
    cbm.set_prefix_caching(True)
    osch = OracleScheduler(obm, case.arrival_step, case.prompt_len, case.output_len, case.table_width)
    csch = bd.Scheduler(cbm, case.arrival_step, case.prompt_len, case.output_len, case.table_width)
    osch.set_prompt_tokens(case.prompt_tokens)
    csch.set_prompt_tokens(case.prompt_tokens)
    cached = preempted = 0
    while True:
        o, c = osch.step(), csch.step()
        for key in ("running", "seq_lens", "decode_slots", "prompt_seqs", "prompt_lens", "prompt_starts",
                    "prompt_slots", "admitted", "preempted", "finished"):
            assert list(o[key]) == c[key].tolist(), (o["step"], key)
        assert o["num_free_blocks"] == c["num_free_blocks"] and o["done"] == c["done"]
        cached += o["num_cached_tokens"]
        preempted += len(o["preempted"])
        if o["done"]:
            break
    assert cached > 0 and preempted > 0
