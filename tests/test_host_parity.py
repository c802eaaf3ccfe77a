"""Host C++ block manager and scheduler (through the C ABI) against the
integer oracle: every table, slot, copy-on-write pair, free list and step
event must be identical (CPU only)."""
import numpy as np
import pytest

from oracle.block_manager import BMError, OracleBlockManager
from oracle.scheduler import OracleScheduler
from paged_kv_cache_400_b200 import binding as bd
from paged_kv_cache_400_b200 import workloads as wl
from paged_kv_cache_400_b200.scenario import prepare_decode_step


def same_state(obm, cbm, seqs):
    assert obm.num_free() == cbm.num_free()
    assert list(obm.free_list) == cbm.free_list()
    for s in seqs:
        assert obm.table(s) == cbm.block_table(s)
        assert obm.seq_len(s) == cbm.seq_len(s)
    for b in range(obm.num_blocks):
        assert obm.refcount[b] == cbm.refcount(b)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_operation_sequences(seed):
    rng = np.random.default_rng(100 + seed)
    N = 64
    order = rng.permutation(N)
    obm, cbm = OracleBlockManager(N, order), bd.BlockManager(N, order)
    live, nxt = [], 0
    for i in range(4000):
        op = int(rng.integers(0, 5))
        try:
            if op == 0:
                n = int(rng.integers(0, 90))
                oerr = None
                try:
                    obm.allocate(nxt, n)
                except BMError as e:
                    oerr = e.status
                try:
                    cbm.allocate(nxt, n)
                    cerr = None
                except bd.PagedKVError as e:
                    cerr = e.status
                assert oerr == cerr
                if oerr is None:
                    live.append(nxt)
                nxt += 1
            elif op in (1, 2) and live:
                s = live[int(rng.integers(0, len(live)))]
                try:
                    o = obm.append_slot(s)
                except BMError as e:
                    o = e.status
                try:
                    c = cbm.append_slot(s)
                except bd.PagedKVError as e:
                    c = e.status
                assert o == c
            elif op == 3 and live:
                s = live[int(rng.integers(0, len(live)))]
                obm.fork(s, nxt)
                cbm.fork(s, nxt)
                live.append(nxt)
                nxt += 1
            elif op == 4 and live:
                s = live.pop(int(rng.integers(0, len(live))))
                obm.free(s)
                cbm.free(s)
        finally:
            if i % 97 == 0:
                same_state(obm, cbm, live)
    same_state(obm, cbm, live)
    for s in live:
        L = obm.seq_len(s)
        assert obm.slots(s, 0, L) == cbm.slots(s, 0, L).tolist()


@pytest.mark.parametrize("make", [wl.tiny_case, wl.mha_case, wl.gqa_case, wl.prefix_case])
def test_workload_step_indices_match(make):
    case = make(0)
    prep = prepare_decode_step(case)
    obm = OracleBlockManager(case.num_blocks, case.free_order)
    for op in case.ops:
        getattr(obm, {"allocate": "allocate", "fork": "fork", "free": "free",
                      "append": "append_slot"}[op[0]])(*op[1:])
    slots, cows = [], []
    for s in case.batch:
        slot, a, b = obm.append_slot(s)
        slots.append(slot)
        if a >= 0:
            cows.append((a, b))
    assert prep.slot_mapping.tolist() == slots
    assert list(zip(prep.cow_src.tolist(), prep.cow_dst.tolist())) == cows
    for i, s in enumerate(case.batch):
        t = obm.table(s)
        assert prep.block_tables[i].tolist() == t + [-1] * (case.table_width - len(t))
        assert prep.seq_lens[i] == obm.seq_len(s)
    if case.name == "shared_prefix":
        assert len(cows) == 3 * 8


def compare_steps(o, c):
    for key in ("step", "done", "num_waiting", "num_free_blocks"):
        assert o[key] == c[key], key
    for key in ("running", "seq_lens", "decode_slots", "prompt_seqs", "prompt_lens",
                "prompt_slots", "admitted", "preempted", "finished"):
        assert list(o[key]) == c[key].tolist(), (o["step"], key)
    assert o["cow"] == c["cow"]
    assert np.array_equal(np.asarray(o["block_tables"], np.int32).reshape(c["block_tables"].shape),
                          c["block_tables"])


def replay_both(case, n_steps=None):
    obm = OracleBlockManager(case.num_blocks)
    cbm = bd.BlockManager(case.num_blocks)
    osch = OracleScheduler(obm, case.arrival_step, case.prompt_len, case.output_len, case.table_width)
    csch = bd.Scheduler(cbm, case.arrival_step, case.prompt_len, case.output_len, case.table_width)
    steps = preempts = 0
    while True:
        o, c = osch.step(), csch.step()
        compare_steps(o, c)
        steps += 1
        preempts += len(o["preempted"])
        if o["done"] or (n_steps and steps >= n_steps):
            return steps, preempts


def test_small_trace_replay_is_identical():
    case = wl.trace_case(seed=3, n_requests=300, rate=20.0, num_blocks=2500, num_layers=1)
    steps, preempts = replay_both(case)
    assert preempts > 0 and steps > 50


def test_full_trace_replay_is_identical():
    """The 2000-request arrival trace on the 40000-block pool, every step."""
    case = wl.trace_case(seed=0)
    steps, preempts = replay_both(case)
    assert steps > 500 and preempts > 0


def test_scheduler_rejects_oversized_request():
    bm = bd.BlockManager(10)
    with pytest.raises(bd.PagedKVError) as e:
        bd.Scheduler(bm, [0], [100], [100], 4)
    assert e.value.status == "CAPACITY"


@pytest.mark.parametrize("host_blocks", [0, 300, 5000])
def test_swap_mode_trace_replay_is_identical(host_blocks):
    """Swap-mode preemption (few host blocks: swap and recompute mixed; many:
    every eligible victim swapped) replays identically in C++ and the oracle."""
    case = wl.trace_case(seed=3, n_requests=300, rate=20.0, num_blocks=2500, num_layers=1)
    obm, cbm = OracleBlockManager(case.num_blocks), bd.BlockManager(case.num_blocks)
    osch = OracleScheduler(obm, case.arrival_step, case.prompt_len, case.output_len, case.table_width)
    csch = bd.Scheduler(cbm, case.arrival_step, case.prompt_len, case.output_len, case.table_width)
    osch.set_swap(host_blocks)
    csch.set_swap(host_blocks)
    outs = swapped = 0
    while True:
        o, c = osch.step(), csch.step()
        compare_steps(o, c)
        assert o["swap_out"] == c["swap_out"] and o["swap_in"] == c["swap_in"]
        assert list(o["swapped_out"]) == c["swapped_out"].tolist()
        assert list(o["swapped_in"]) == c["swapped_in"].tolist()
        outs += len(o["preempted"])
        swapped += len(o["swapped_out"])
        if o["done"]:
            break
    assert outs > 0
    assert (swapped > 0) == (host_blocks > 0)
    if host_blocks == 300:
        assert 0 < swapped < outs
