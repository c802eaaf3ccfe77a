"""Pins of the oracle's continuous-batching loop (CPU only).

The pages fix the policy points checked here: requests leave as soon as they
finish and their pages return at once; waiting requests join while pages are
free; growth allocates a page only when the last one is full; a preempted
request gives back its pages and later resumes by recomputation. The expected
event lists below were worked out by hand from those rules on tiny pools.
"""
import numpy as np
import pytest

from oracle.block_manager import BMError, OracleBlockManager, blocks_for
from oracle.scheduler import OracleScheduler


def run(num_blocks, arrival, prompt, output, width=8):
    bm = OracleBlockManager(num_blocks)
    s = OracleScheduler(bm, arrival, prompt, output, width)
    steps = []
    while True:
        out = s.step()
        steps.append(out)
        if out["done"]:
            return steps, bm


def test_hand_worked_trace_without_preemption():
    # 4 blocks; r0: t=0, prompt 20, 3 tokens; r1: t=0, 16, 2; r2: t=1, 10, 1
    steps, bm = run(4, [0, 0, 1], [20, 16, 10], [3, 2, 1])
    s0, s1, s2, s3 = steps
    assert s0["admitted"] == [0, 1] and s0["running"] == [0, 1]
    assert s0["block_tables"] == [[0, 1] + [-1] * 6, [2, 3] + [-1] * 6]
    assert s0["decode_slots"] == [20, 48] and s0["seq_lens"] == [21, 17]
    assert s0["prompt_seqs"] == [0, 1] and s0["prompt_lens"] == [20, 16]
    assert s0["prompt_slots"] == list(range(0, 20)) + list(range(32, 48))
    assert s0["num_free_blocks"] == 0
    # r2 arrives, no page free, waits
    assert s1["admitted"] == [] and s1["num_waiting"] == 1
    assert s1["decode_slots"] == [21, 49] and s1["seq_lens"] == [22, 18]
    # r1 finished (2 tokens): its pages [2, 3] return; r2 takes page 2
    assert s2["finished"] == [1] and s2["admitted"] == [2]
    assert s2["running"] == [0, 2] and s2["decode_slots"] == [22, 42]
    assert s2["prompt_slots"] == list(range(32, 42)) and s2["seq_lens"] == [23, 11]
    assert s2["num_free_blocks"] == 1
    assert s3["finished"] == [0, 2] and s3["done"] == 1 and s3["running"] == []
    assert list(bm.free_list) == [3, 0, 1, 2]


def test_hand_worked_trace_with_preemption():
    # 2 blocks; r0: prompt 16, 2 tokens; r1: prompt 15, 3 tokens; both at t=0
    steps, bm = run(2, [0, 0], [16, 15], [2, 3])
    s0, s1, s2, s3, s4, s5 = steps
    # r0 needs a second page; the newest running request (r1) is preempted
    assert s0["admitted"] == [0, 1] and s0["preempted"] == [1]
    assert s0["running"] == [0] and s0["decode_slots"] == [16]
    assert s0["prompt_seqs"] == [0] and s0["prompt_slots"] == list(range(16))
    assert s0["num_waiting"] == 1
    assert s1["admitted"] == [] and s1["decode_slots"] == [17]
    # r0 done; r1 recomputed from its prompt (generated 0) into page 0
    assert s2["finished"] == [0] and s2["admitted"] == [1]
    assert s2["prompt_slots"] == list(range(15)) and s2["decode_slots"] == [15]
    assert s3["decode_slots"] == [16] and s3["block_tables"][0][:2] == [0, 1]
    assert s4["decode_slots"] == [17] and s4["seq_lens"] == [18]
    assert s5["finished"] == [1] and s5["done"] == 1


def test_preempted_request_resumes_with_generated_tokens():
    # 4 blocks: r0 (prompt 40, 20 tokens) and r1 (prompt 10, 30 tokens) start
    # together; r1 is evicted when it needs a second page, and every
    # re-admission recomputes prompt + generated tokens of KV.
    prompt, output = [40, 10], [20, 30]
    bm = OracleBlockManager(4)
    s = OracleScheduler(bm, [0, 0], prompt, output, 8)
    generated = [0, 0]
    readmitted_with_progress = 0
    while True:
        out = s.step()
        for r, n in zip(out["prompt_seqs"], out["prompt_lens"]):
            assert n == prompt[r] + generated[r]
            readmitted_with_progress += generated[r] > 0
        for r in out["preempted"]:
            assert r not in out["running"]
        for r in out["running"]:
            generated[r] += 1
        if out["done"]:
            break
    assert generated == output and readmitted_with_progress > 0
    assert bm.num_free() == 4


def test_self_preemption_alone_is_an_error():
    bm = OracleBlockManager(1)
    s = OracleScheduler(bm, [0], [16], [2], 4)
    with pytest.raises(BMError) as e:
        s.step()
    assert e.value.status == "NO_BLOCKS"


def test_never_fitting_request_is_an_error():
    bm = OracleBlockManager(2)
    s = OracleScheduler(bm, [0], [40], [1], 4)
    with pytest.raises(BMError):
        s.step()


def test_invariants_on_random_trace():
    rng = np.random.default_rng(11)
    n = 300
    arrival = np.sort(rng.integers(0, 40, size=n))
    prompt = rng.integers(1, 200, size=n)
    output = np.minimum(rng.geometric(1 / 30, size=n), 300)
    N = 200
    bm = OracleBlockManager(N, rng.permutation(N))
    s = OracleScheduler(bm, arrival, prompt, output, 40)
    generated = np.zeros(n, int)
    finished_at = {}
    total_preempt = 0
    while True:
        out = s.step()
        total_preempt += len(out["preempted"])
        # page accounting
        held = {}
        for r, tab in bm.tables.items():
            assert len(tab) == blocks_for(bm.lens[r])
            for blk in tab:
                held[blk] = held.get(blk, 0) + 1
        assert len(bm.free_list) + len(held) == N
        assert not (set(bm.free_list) & set(held))
        assert all(bm.refcount[b] == c for b, c in held.items())
        # every running request holds exactly its length's pages, and its
        # length is prompt + generated (+1 for this step's token)
        for r, L, tab in zip(out["running"], out["seq_lens"], out["block_tables"]):
            assert L == prompt[r] + generated[r] + 1
            assert sum(1 for x in tab if x >= 0) == blocks_for(L)
        for r in out["running"]:
            generated[r] += 1
        for r in out["finished"]:
            finished_at[r] = out["step"]
            assert generated[r] == output[r]
        # nothing runs before it arrives
        assert all(arrival[r] <= out["step"] for r in out["running"])
        if out["done"]:
            break
    assert len(finished_at) == n and total_preempt > 0
    assert bm.num_free() == N


# ---------------------------------------------------------------------------
# Swap-mode preemption ("vLLM 原理：PagedAttention 和 Continuous Batching",
# "Preemption（抢占）": the second mode moves a suspended request's KV to CPU
# memory and brings it back instead of recomputing it; "大模型推理性能优化…" §3.4
# --swap-space). Readings pinned here, each expectation worked out by hand:
#   * a victim qualifies when its KV was written before this step (it was not
#     admitted in it) and none of its blocks is shared; it then takes host
#     blocks from the head of a FIFO host free list, one per device block, in
#     table order (swap_out pairs are (device, host));
#   * a victim that does not qualify, or finds too few host blocks, is
#     recomputed, exactly as without swap;
#   * re-admission of a swapped-out request takes fresh device blocks for
#     prompt + generated tokens, writes no prompt KV, and copies its host blocks
#     back (swap_in pairs are (host, device)); the host blocks return to the
#     host list's tail at the end of that step;
#   * a request admitted from host blocks and preempted again in the same step
#     keeps its host copy (no pairs, no host block freed).
# The same expectations are checked on the C++ scheduler through the C ABI.
# ---------------------------------------------------------------------------

def _ints(x):
    return [int(v) for v in x]


def _pairs(x):
    return [(int(a), int(b)) for a, b in x]


def _swap_run(impl, num_blocks, host_blocks, arrival, prompt, output, width=8, tokens=None):
    """Runs a tiny trace to completion on the oracle or the C++ scheduler;
    returns the per-step outputs and the scheduler."""
    if impl == "oracle":
        bm = OracleBlockManager(num_blocks)
        if tokens is not None:
            bm.set_prefix_caching(True)
        s = OracleScheduler(bm, arrival, prompt, output, width)
    else:
        from paged_kv_cache_400_b200 import binding as bd
        bm = bd.BlockManager(num_blocks)
        if tokens is not None:
            bm.set_prefix_caching(True)
        s = bd.Scheduler(bm, arrival, prompt, output, width)
    if tokens is not None:
        s.set_prompt_tokens(tokens)
    s.set_swap(host_blocks)
    steps = []
    while True:
        out = s.step()
        steps.append(out)
        if out["done"]:
            return steps, s, bm


IMPLS = ["oracle", "cpp"]


@pytest.mark.parametrize("impl", IMPLS)
def test_swap_out_and_in_hand_worked(impl):
    # 3 device blocks, 4 host blocks; r0: t=0, prompt 16, 3 tokens;
    # r1: t=1, prompt 15, 3 tokens.
    steps, sched, bm = _swap_run(impl, 3, 4, [0, 1], [16, 15], [3, 3])
    assert len(steps) == 6
    s0, s1, s2, s3, s4, s5 = steps
    # step 0: r0 takes block 0, opens block 1 for position 16
    assert _ints(s0["running"]) == [0] and _ints(s0["decode_slots"]) == [16]
    assert _pairs(s0["swap_out"]) == [] and _pairs(s0["swap_in"]) == []
    # step 1: r1 (15 tokens) takes block 2; its KV is written this step
    assert _ints(s1["admitted"]) == [1] and _ints(s1["decode_slots"]) == [17, 47]
    assert _ints(s1["prompt_slots"]) == list(range(32, 47))
    # step 2: r1 needs a block for position 16, none is free: r1 (the newest)
    # is the victim; its one block (2) was written before the step and is
    # private, so it goes to host block 0 (head of the host list)
    assert _ints(s2["preempted"]) == [1] and _ints(s2["swapped_out"]) == [1]
    assert _pairs(s2["swap_out"]) == [(2, 0)] and _pairs(s2["swap_in"]) == []
    assert _ints(s2["running"]) == [0] and _ints(s2["decode_slots"]) == [18]
    assert s2["num_waiting"] == 1 and s2["num_free_blocks"] == 1
    # step 3: r0 finishes, blocks [0, 1] return behind 2 (free list 2, 0, 1);
    # r1 is admitted from host: 16 tokens (prompt 15 + 1 generated) in block
    # 2, nothing recomputed, host block 0 copied back into block 2; position
    # 16 opens block 0
    assert _ints(s3["finished"]) == [0] and _ints(s3["admitted"]) == [1]
    assert _ints(s3["swapped_in"]) == [1] and _pairs(s3["swap_in"]) == [(0, 2)]
    assert _pairs(s3["swap_out"]) == []
    assert _ints(s3["prompt_seqs"]) == [] and _ints(s3["prompt_slots"]) == []
    assert _ints(s3["decode_slots"]) == [0] and _ints(s3["seq_lens"]) == [17]
    assert [int(x) for x in s3["block_tables"][0][:2]] == [2, 0]
    assert _ints(s4["decode_slots"]) == [1] and _ints(s4["swapped_in"]) == []
    assert _ints(s5["finished"]) == [1] and s5["done"] == 1
    if impl == "oracle":
        # host block 0 went back to the tail after the swap-in step
        assert list(sched.host_free) == [1, 2, 3, 0] and sched.host_table == {}
        assert list(bm.free_list) == [1, 2, 0]
    else:
        assert bm.free_list() == [1, 2, 0]


@pytest.mark.parametrize("impl", IMPLS)
def test_swap_victim_admitted_this_step_is_recomputed(impl):
    # The recompute trace of test_hand_worked_trace_with_preemption with 4 host
    # blocks: r1 is preempted in the step that admitted it, before any of its
    # KV was written, so swap mode changes nothing.
    steps, sched, _ = _swap_run(impl, 2, 4, [0, 0], [16, 15], [2, 3])
    s0, s1, s2, s3, s4, s5 = steps
    assert _ints(s0["admitted"]) == [0, 1] and _ints(s0["preempted"]) == [1]
    assert _ints(s0["swapped_out"]) == [] and _pairs(s0["swap_out"]) == []
    assert _ints(s2["admitted"]) == [1] and _ints(s2["prompt_slots"]) == list(range(15))
    assert _ints(s2["swapped_in"]) == [] and _pairs(s2["swap_in"]) == []
    for s in steps:
        assert _pairs(s["swap_out"]) == [] and _pairs(s["swap_in"]) == []
    if impl == "oracle":
        assert list(sched.host_free) == [0, 1, 2, 3]


@pytest.mark.parametrize("impl", IMPLS)
def test_swap_with_too_few_host_blocks_is_recomputed(impl):
    # 5 device blocks, 1 host block; r0: t=0, prompt 32, 3 tokens; r1: t=1,
    # prompt 31, 3 tokens. r1 holds 2 blocks when it is preempted: one host
    # block is not enough, so it is recomputed.
    steps, sched, _ = _swap_run(impl, 5, 1, [0, 1], [32, 31], [3, 3])
    s0, s1, s2, s3 = steps[:4]
    assert _ints(s0["decode_slots"]) == [32]                  # r0: blocks 0, 1; opens 2
    assert _ints(s1["admitted"]) == [1] and _ints(s1["decode_slots"]) == [33, 79]
    assert _ints(s1["prompt_slots"]) == list(range(48, 79))   # blocks 3, 4
    assert _ints(s2["preempted"]) == [1] and _ints(s2["swapped_out"]) == []
    assert _pairs(s2["swap_out"]) == []
    # r0 finishes (free list 3, 4, 0, 1, 2); r1 recomputes its 32 tokens in
    # blocks 3, 4 and opens block 0 for position 32
    assert _ints(s3["finished"]) == [0] and _ints(s3["admitted"]) == [1]
    assert _ints(s3["prompt_seqs"]) == [1] and _ints(s3["prompt_lens"]) == [32]
    assert _ints(s3["prompt_slots"]) == list(range(48, 80))
    assert _ints(s3["decode_slots"]) == [0] and _pairs(s3["swap_in"]) == []
    if impl == "oracle":
        assert list(sched.host_free) == [0]


@pytest.mark.parametrize("impl", IMPLS)
def test_swap_victim_with_shared_block_is_recomputed(impl):
    # Prefix caching on, 4 device blocks, 8 host blocks. r0 (t=0) and r1 (t=1)
    # have 30-token prompts with the same first 16 tokens; r1 reuses r0's
    # cached block 0 (refcount 2). At step 3 r1 needs a block for position 32
    # and none is free: it is the victim, and because block 0 is shared it is
    # recomputed, not swapped.
    common = list(range(100, 116))
    tokens = [common + list(range(200, 214)), common + list(range(300, 314))]
    steps, sched, _ = _swap_run(impl, 4, 8, [0, 1], [30, 30], [4, 5], tokens=tokens)
    s0, s1, s2, s3, s4 = steps[:5]
    assert _ints(s0["prompt_slots"]) == list(range(30)) and _ints(s0["decode_slots"]) == [30]
    # r1: block 0 shared (16 cached tokens), block 2 fresh for positions 16-29
    assert _ints(s1["prompt_starts"]) == [16] and _ints(s1["prompt_slots"]) == list(range(32, 46))
    assert [int(x) for x in s1["block_tables"][1][:2]] == [0, 2]
    assert _ints(s2["decode_slots"]) == [48, 47]              # r0 opens block 3
    assert _ints(s3["preempted"]) == [1] and _ints(s3["swapped_out"]) == []
    assert _pairs(s3["swap_out"]) == [] and _ints(s3["decode_slots"]) == [49]
    # step 4: r0 finishes; r1 is admitted again through the cache (block 0,
    # now on the evictable list) plus fresh block 2, recomputing positions
    # 16-31 from its cached prefix on, and opens block 1 for position 32
    assert _ints(s4["finished"]) == [0] and _ints(s4["admitted"]) == [1]
    assert _ints(s4["prompt_starts"]) == [16] and _ints(s4["prompt_lens"]) == [32]
    assert _ints(s4["prompt_slots"]) == list(range(32, 48))
    assert _ints(s4["decode_slots"]) == [16] and _pairs(s4["swap_in"]) == []
    if impl == "oracle":
        assert list(sched.host_free) == list(range(8))


@pytest.mark.parametrize("impl", IMPLS)
def test_swapped_in_then_preempted_keeps_host_copy(impl):
    # As test_swap_out_and_in_hand_worked, but r0 generates 5 tokens: after r1
    # is swapped out (step 2), steps 3 and 4 admit it from host into the one
    # free block and preempt it again when it needs a block for position 16;
    # it keeps its host copy (no pairs, host block 0 stays taken). Step 5: r0
    # has finished, r1 is swapped in.
    steps, sched, _ = _swap_run(impl, 3, 4, [0, 1], [16, 15], [5, 3])
    assert _pairs(steps[2]["swap_out"]) == [(2, 0)]
    for s in steps[3:5]:
        assert _ints(s["admitted"]) == [1] and _ints(s["preempted"]) == [1]
        assert _ints(s["running"]) == [0]
        assert _pairs(s["swap_out"]) == [] and _pairs(s["swap_in"]) == []
        assert _ints(s["swapped_out"]) == [] and _ints(s["swapped_in"]) == []
        assert _ints(s["prompt_seqs"]) == []
    assert _ints(steps[3]["decode_slots"]) == [19] and _ints(steps[4]["decode_slots"]) == [20]
    s5 = steps[5]
    assert _ints(s5["finished"]) == [0] and _ints(s5["swapped_in"]) == [1]
    assert _pairs(s5["swap_in"]) == [(0, 2)] and _ints(s5["decode_slots"]) == [0]
    assert _ints(s5["prompt_seqs"]) == []
    if impl == "oracle":
        assert list(sched.host_free) == [1, 2, 3, 0]


@pytest.mark.parametrize("host_blocks", [40, 400])
def test_invariants_on_random_trace_with_swap(host_blocks):
    """The invariants of test_invariants_on_random_trace with swap mode on,
    plus host-block accounting: free host blocks and the blocks held by
    swapped-out requests partition the host pool; only waiting requests hold
    host blocks; a swap-out moves exactly the victim's private blocks; a
    swap-in fills exactly the blocks of prompt + generated tokens and writes
    no prompt KV."""
    rng = np.random.default_rng(12)
    n = 300
    arrival = np.sort(rng.integers(0, 40, size=n))
    prompt = rng.integers(1, 200, size=n)
    output = np.minimum(rng.geometric(1 / 30, size=n), 300)
    N = 200
    bm = OracleBlockManager(N, rng.permutation(N))
    s = OracleScheduler(bm, arrival, prompt, output, 40)
    s.set_swap(host_blocks)
    generated = np.zeros(n, int)
    host_of = {}            # request -> host blocks, tracked from the pairs
    n_out = n_in = n_pre = 0
    while True:
        tables_before = {r: list(t) for r, t in bm.tables.items()}
        out = s.step()
        n_pre += len(out["preempted"])
        # swap-out pairs: per swapped-out victim, its whole table before the
        # step (a victim never grew this step: it was the running tail)
        i = 0
        for r in out["swapped_out"]:
            tab = tables_before[r]
            got = out["swap_out"][i:i + len(tab)]
            i += len(tab)
            assert [d for d, _ in got] == tab
            assert r in out["preempted"] and r not in out["running"]
            host_of[r] = [h for _, h in got]
            n_out += 1
        assert i == len(out["swap_out"])
        i = 0
        for r in out["swapped_in"]:
            h = host_of.pop(r)
            got = out["swap_in"][i:i + len(h)]
            i += len(h)
            assert [x for x, _ in got] == h
            assert len(h) == blocks_for(prompt[r] + generated[r])
            k = out["running"].index(r)
            assert [d for _, d in got] == out["block_tables"][k][:len(h)]
            assert r not in out["prompt_seqs"]
            n_in += 1
        assert i == len(out["swap_in"])
        # host accounting
        held = [b for r in s.host_table for b in s.host_table[r]]
        assert sorted(list(s.host_free) + held) == list(range(host_blocks))
        assert set(s.host_table) == set(host_of)
        assert all(s.host_table[r] == host_of[r] for r in host_of)
        assert set(s.host_table) <= set(s.waiting)
        # device accounting, as without swap
        held_dev = {}
        for r, tab in bm.tables.items():
            assert len(tab) == blocks_for(bm.lens[r])
            for blk in tab:
                held_dev[blk] = held_dev.get(blk, 0) + 1
        assert len(bm.free_list) + len(held_dev) == N
        assert all(bm.refcount[b] == c for b, c in held_dev.items())
        for r, L in zip(out["running"], out["seq_lens"]):
            assert L == prompt[r] + generated[r] + 1
        for r in out["running"]:
            generated[r] += 1
        for r in out["finished"]:
            assert generated[r] == output[r]
        if out["done"]:
            break
    assert n_out > 0 and n_in > 0 and n_pre > n_out
    assert bm.num_free() == N and len(s.host_free) == host_blocks
