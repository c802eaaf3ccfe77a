"""Host side of the prefill step (no GPU): the library block manager's tables
and new-token slots for the prefill workloads are bit-exact with the oracle
block manager's, and the oracle's one-row sampling used at full size agrees
with its whole-step prefill."""
import numpy as np

from paged_kv_cache_400_b200 import workloads as wl
from paged_kv_cache_400_b200.scenario import prepare_prefill_step

from oracle_side import oracle_prefill_all, oracle_prefill_indices, oracle_prefill_rows


def _same(case):
    prep = prepare_prefill_step(case)
    ost = oracle_prefill_indices(case)
    assert prep.slot_mapping.tolist() == ost.slots
    assert prep.seq_lens.tolist() == ost.lens
    for b, tab in enumerate(ost.tables):
        assert prep.block_tables[b, :len(tab)].tolist() == tab
    assert prep.query_start[0] == 0 and prep.query_start[-1] == case.num_tokens
    assert np.all(np.diff(prep.query_start) == np.asarray(case.query_lens))


def test_prefill_indices_bit_exact():
    _same(wl.prefill_case(0))
    _same(wl.chunked_prefill_case(0))
    _same(wl.prefill_custom("c", 1, [0, 5, 16, 33], [7, 64, 1, 0], 32, 8))


def test_row_sampling_matches_whole_step():
    case = wl.prefill_custom("s", 2, [0, 19, 3], [21, 17, 5], 4, 2)
    ost = oracle_prefill_indices(case)
    whole, _ = oracle_prefill_all(case, ost)
    picks = [(b, i) for b in range(3) for i in range(case.query_lens[b])]
    rows = oracle_prefill_rows(case, ost, picks)
    assert np.allclose(rows, whole, rtol=0, atol=1e-12)


def test_prefill_flop_count_closed_form():
    """The prefill roofline's algorithmic FLOPs: for every new position p of a
    sequence, each query head scores p + 1 keys and sums p + 1 values, 2 x 128
    FLOPs each. The bench's closed form against a brute-force count."""
    import bench
    case = wl.prefill_custom("f", 3, [0, 7, 100, 16], [5, 1, 33, 0], 32, 8)
    brute = 0
    for c, n in zip(case.ctx_lens, case.query_lens):
        for p in range(c, c + n):
            brute += case.num_heads * (p + 1) * 2 * 2 * case.head_dim
    assert bench.prefill_flops(case) == brute


def test_engine_prefill_indices_match_oracle_replay():
    """DecodeEngine.prefill_indices (host side of the step loop's prefill):
    per admitted prompt, its rows of the step's block tables, KV length =
    prompt length, and query_start over the new positions, against the
    oracle scheduler's replay of the same trace (CPU)."""
    import torch
    from oracle.block_manager import OracleBlockManager
    from oracle.scheduler import OracleScheduler
    from paged_kv_cache_400_b200.engine import DecodeEngine
    trace = wl.trace_case(seed=3, n_requests=60, rate=8.0, num_blocks=400, num_layers=1, output_cap=80)
    eng = DecodeEngine(trace.num_blocks, 1, 4, 2, 128, trace.arrival_step, trace.prompt_len,
                       trace.output_len, trace.table_width, trace.scale, "cpu")
    obm = OracleBlockManager(trace.num_blocks)
    osch = OracleScheduler(obm, trace.arrival_step, trace.prompt_len, trace.output_len, trace.table_width)
    seen = 0
    while True:
        idx = eng.schedule()
        o = osch.step()
        if len(idx.prompt_seqs):
            bt, sl, qs, mx = eng.prefill_indices(idx)
            bt, sl, qs = bt.numpy(), sl.numpy(), qs.numpy()
            running = o["running"]
            starts = o.get("prompt_starts", [0] * len(o["prompt_seqs"]))
            for k, req in enumerate(o["prompt_seqs"]):
                row = running.index(req)
                assert sl[k] == o["prompt_lens"][k]
                n_new = o["prompt_lens"][k] - starts[k]
                assert qs[k + 1] - qs[k] == n_new
                width = (o["prompt_lens"][k] + 15) // 16
                assert bt[k, :width].tolist() == o["block_tables"][row][:width]
            assert qs[0] == 0 and mx == max(int(a) - int(b) for a, b in zip(o["prompt_lens"], starts))
            seen += len(o["prompt_seqs"])
        if idx.done:
            break
    eng.close()
    assert seen >= 60


def test_prefill_indices_skip_swapped_in_requests():
    """Swap-mode preemption: a request swapped back in has its KV restored by
    block copies, so it is not among the step's prompts and gets no prefill
    rows; every prompt that is prefilled is fresh or recomputed (CPU, through
    the library's scheduler)."""
    from types import SimpleNamespace

    import torch
    from paged_kv_cache_400_b200 import binding as bd
    from paged_kv_cache_400_b200.engine import DecodeEngine
    trace = wl.trace_case(seed=5, n_requests=240, rate=16.0, num_blocks=1800, num_layers=1, output_cap=300)
    bm = bd.BlockManager(trace.num_blocks)
    sched = bd.Scheduler(bm, trace.arrival_step, trace.prompt_len, trace.output_len, trace.table_width)
    sched.set_swap(600)
    # DecodeEngine's host-side methods on a stand-in engine (no device pools)
    eng = SimpleNamespace(sched=sched, device=torch.device("cpu"))
    swapped_in_total = prompts_total = 0
    while True:
        idx = DecodeEngine.schedule(eng)
        swapped = {int(d) for d in idx.swap_in[:, 1]} if len(idx.swap_in) else set()
        if len(idx.prompt_seqs):
            bt, sl, qs, mx = DecodeEngine.prefill_indices(eng, idx)
            prompts_total += len(idx.prompt_seqs)
            assert (np.diff(qs.numpy()) == idx.prompt_lens - idx.prompt_starts).all()
            # no prefilled prompt's table holds a block the step swaps in
            width = (idx.prompt_lens + 15) // 16
            for k in range(len(idx.prompt_seqs)):
                assert not (set(bt.numpy()[k, :width[k]].tolist()) & swapped)
        swapped_in_total += len(idx.swap_in)
        if idx.done:
            break
    sched.close()
    bm.close()
    assert prompts_total > 200 and swapped_in_total > 0
