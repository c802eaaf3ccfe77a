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
