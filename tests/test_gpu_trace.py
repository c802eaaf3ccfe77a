"""GPU parity of the continuous-batching trace: the C++ scheduler drives the
device loop (prompt append, decode-token append, paged decode per layer) over
an arrival trace with preemptions; at sampled steps the fp64 oracle, with its
own scheduler replay, block tables and pool built from the generator's K/V,
must agree with the GPU attention output of every sampled request.

The K/V of (layer, request, position) are a fixed function of those
coordinates, so a request recomputed after preemption must see exactly the
values it had before; any misplaced write in any earlier step shows up as an
attention mismatch here.
"""
import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle.block_manager import OracleBlockManager
from oracle.scheduler import OracleScheduler
from paged_kv_cache_400_b200 import workloads as wl
from paged_kv_cache_400_b200.engine import DecodeEngine

from oracle_side import oracle_trace_row, storage_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def layer_inputs(trace, eng, idx, layer, device):
    reqs_p, pos_p = eng.prompt_positions(idx)
    k_p, v_p = trace.kv_values(layer, reqs_p, pos_p, device)
    k_d, v_d = trace.kv_values(layer, idx.running, idx.seq_lens.astype(np.int64) - 1, device)
    q = trace.q_values(layer, idx.step, idx.running, device)
    return {"q": q, "k_dec": k_d, "v_dec": v_d, "k_prompt": k_p, "v_prompt": v_p}


def oracle_attention(trace, layer, step, req, table, length):
    """Oracle: scatter the request's K/V (generator values) through its own
    block table into a compact pool, then gather-and-attend in fp64."""
    return oracle_trace_row(trace, layer, step, req, table, length)[0]


def test_trace_with_preemption_matches_oracle():
    trace = wl.trace_case(seed=5, n_requests=240, rate=16.0, num_blocks=1800, num_layers=2,
                          output_cap=300)
    eng = DecodeEngine(trace.num_blocks, trace.num_layers, trace.num_heads, trace.num_kv_heads,
                       trace.head_dim, trace.arrival_step, trace.prompt_len, trace.output_len,
                       trace.table_width, trace.scale, DEV)
    obm = OracleBlockManager(trace.num_blocks)
    osch = OracleScheduler(obm, trace.arrival_step, trace.prompt_len, trace.output_len, trace.table_width)
    rng = np.random.default_rng(0)
    checked = preempted_seen = steps = 0
    max_err = 0.0
    while True:
        idx = eng.schedule()
        o = osch.step()
        assert idx.running.tolist() == o["running"]
        assert idx.decode_slots.tolist() == o["decode_slots"]
        assert idx.prompt_slots.tolist() == o["prompt_slots"]
        preempted_seen += len(o["preempted"])
        steps += 1
        if len(idx.running):
            inputs = [layer_inputs(trace, eng, idx, l, DEV) for l in range(trace.num_layers)]
            outs = eng.run_layers(idx, inputs)
            sample_step = checked < 40 and ((idx.step % 20 == 0) or
                                            (len(o["preempted"]) and idx.step % 3 == 0))
            if sample_step:
                layer = int(rng.integers(0, trace.num_layers))
                rows = rng.choice(len(idx.running), size=min(3, len(idx.running)), replace=False)
                got = outs[layer].float().cpu().numpy()
                for i in rows:
                    r = int(idx.running[i])
                    ref = oracle_attention(trace, layer, idx.step, r, o["block_tables"][i][
                        :(o["seq_lens"][i] + 15) // 16], o["seq_lens"][i])
                    err = float(np.abs(got[i] - ref).max())
                    max_err = max(max_err, err)
                    assert err <= 1e-2, (idx.step, r, err)
                    checked += 1
        if idx.done:
            break
    import paged_kv_cache_400_b200 as pk
    assert pk.pa_get_device_error() == 0
    assert preempted_seen > 0 and checked >= 20, (preempted_seen, checked, steps)
    eng.close()


def test_full_size_trace_matches_oracle():
    """The continuous-batching config at its stated size: 2000 requests,
    Poisson(50) arrivals per step, prompts U[16, 1024], outputs geometric (mean
    200, cap 2048), one 40 000-block pool (one layer: every layer runs the same
    calls on a pool of its own). Every step's running set, lengths, block
    tables, decode slots and prompt slots equal the oracle scheduler's; at least
    40 (step, request) attention rows are compared with the fp64 oracle, among
    them requests right after a preemption and re-admission (their prompt and
    generated tokens' K/V rewritten by recompute) and again a few steps later."""
    trace = wl.trace_case(seed=0, num_layers=1)
    eng = DecodeEngine(trace.num_blocks, trace.num_layers, trace.num_heads, trace.num_kv_heads,
                       trace.head_dim, trace.arrival_step, trace.prompt_len, trace.output_len,
                       trace.table_width, trace.scale, DEV)
    obm = OracleBlockManager(trace.num_blocks)
    osch = OracleScheduler(obm, trace.arrival_step, trace.prompt_len, trace.output_len, trace.table_width)
    rng = np.random.default_rng(3)
    preempted_ever, follow = set(), {}
    checked = readmit_checked = later_checked = steps = 0
    while True:
        idx = eng.schedule()
        o = osch.step()
        steps += 1
        assert idx.running.tolist() == o["running"]
        assert idx.seq_lens.tolist() == o["seq_lens"]
        assert idx.decode_slots.tolist() == o["decode_slots"]
        assert idx.prompt_slots.tolist() == o["prompt_slots"]
        assert idx.prompt_seqs.tolist() == o["prompt_seqs"]
        if len(idx.running):
            assert np.array_equal(idx.block_tables, np.asarray(o["block_tables"], np.int32))
        readmitted = [r for r in o["prompt_seqs"] if r in preempted_ever]
        preempted_ever.update(o["preempted"])
        if len(idx.running):
            inputs = [layer_inputs(trace, eng, idx, 0, DEV)]
            outs = eng.run_layers(idx, inputs)
            row_of = {int(r): i for i, r in enumerate(idx.running)}
            picks = []
            if readmit_checked < 16:
                for r in readmitted[:2]:
                    picks.append((r, "readmit"))
                    follow.setdefault(r, idx.step + 5)
            for r, at in list(follow.items()):
                if at == idx.step and r in row_of:
                    picks.append((r, "later"))
                    del follow[r]
            if idx.step % 50 == 0:
                picks.append((int(idx.running[int(rng.integers(len(idx.running)))]), "random"))
            if picks:
                got = outs[0].float().cpu().numpy()
                for r, why in picks:
                    i = row_of[r]
                    L = o["seq_lens"][i]
                    ref = oracle_attention(trace, 0, idx.step, r, o["block_tables"][i][:(L + 15) // 16], L)
                    err = float(np.abs(got[i] - ref).max())
                    assert err <= 1e-2, (idx.step, r, why, err)
                    checked += 1
                    readmit_checked += why == "readmit"
                    later_checked += why == "later"
        if idx.done:
            break
    import paged_kv_cache_400_b200 as pk
    assert pk.pa_get_device_error() == 0
    eng.close()
    assert steps > 1000 and len(preempted_ever) > 0
    assert checked >= 40 and readmit_checked >= 10 and later_checked >= 5, \
        (checked, readmit_checked, later_checked)


def test_graphed_layer_loop_matches_oracle():
    """The same trace with each step's decode over all layers replayed as a CUDA
    graph per batch bucket (padded rows inert)."""
    from paged_kv_cache_400_b200.engine import GraphedLayers
    trace = wl.trace_case(seed=6, n_requests=120, rate=12.0, num_blocks=1200, num_layers=2,
                          output_cap=120)
    eng = DecodeEngine(trace.num_blocks, trace.num_layers, trace.num_heads, trace.num_kv_heads,
                       trace.head_dim, trace.arrival_step, trace.prompt_len, trace.output_len,
                       trace.table_width, trace.scale, DEV)
    graphed = GraphedLayers(eng, max_batch=128, bucket=32)
    obm = OracleBlockManager(trace.num_blocks)
    osch = OracleScheduler(obm, trace.arrival_step, trace.prompt_len, trace.output_len, trace.table_width)
    rng = np.random.default_rng(1)
    checked = 0
    while True:
        idx = eng.schedule()
        o = osch.step()
        if len(idx.running):
            reqs_p, pos_p = eng.prompt_positions(idx)
            inputs, stacked = trace.step_inputs(idx.step, idx.running, idx.seq_lens, reqs_p, pos_p, DEV,
                                                stacked=True)
            outs = graphed.run(idx, inputs, stacked)
            if idx.step % 15 == 0 and checked < 30:
                layer = int(rng.integers(0, trace.num_layers))
                got = outs[layer].float().cpu().numpy()
                for i in rng.choice(len(idx.running), size=min(3, len(idx.running)), replace=False):
                    r = int(idx.running[i])
                    ref = oracle_attention(trace, layer, idx.step, r,
                                           o["block_tables"][i][:(o["seq_lens"][i] + 15) // 16],
                                           o["seq_lens"][i])
                    assert float(np.abs(got[i] - ref).max()) <= 1e-2
                    checked += 1
        if idx.done:
            break
    import paged_kv_cache_400_b200 as pk
    assert pk.pa_get_device_error() == 0
    assert checked >= 10 and len(graphed.graphs) >= 2
    eng.close()


def test_shared_prompt_trace_with_prefix_caching_matches_oracle():
    """Requests share system prompts; with prefix caching their full system
    prompt blocks are reused and never rewritten. Each sampled output must
    still equal the oracle's attention over the request's whole prompt."""
    trace = wl.prefix_trace_case(seed=7, n_requests=160, rate=12.0, num_blocks=2600, num_layers=2,
                                 n_system=3)
    trace.output_len = np.minimum(trace.output_len, 150).astype(np.int32)
    eng = DecodeEngine(trace.num_blocks, trace.num_layers, trace.num_heads, trace.num_kv_heads,
                       trace.head_dim, trace.arrival_step, trace.prompt_len, trace.output_len,
                       trace.table_width, trace.scale, DEV, prompt_tokens=trace.prompt_tokens)
    obm = OracleBlockManager(trace.num_blocks)
    obm.set_prefix_caching(True)
    osch = OracleScheduler(obm, trace.arrival_step, trace.prompt_len, trace.output_len, trace.table_width)
    osch.set_prompt_tokens(trace.prompt_tokens)
    rng = np.random.default_rng(2)
    checked = hits_checked = cached_total = 0
    started_cached = set()
    while True:
        idx = eng.schedule()
        o = osch.step()
        assert idx.prompt_slots.tolist() == o["prompt_slots"]
        assert idx.prompt_starts.tolist() == o["prompt_starts"]
        cached_total += int(idx.prompt_starts.sum())
        started_cached.update(int(r) for r, a in zip(idx.prompt_seqs, idx.prompt_starts) if a > 0)
        if len(idx.running):
            inputs = [layer_inputs(trace, eng, idx, l, DEV) for l in range(trace.num_layers)]
            outs = eng.run_layers(idx, inputs)
            if idx.step % 7 == 0 and checked < 40:
                layer = int(rng.integers(0, trace.num_layers))
                got = outs[layer].float().cpu().numpy()
                for i in rng.choice(len(idx.running), size=min(3, len(idx.running)), replace=False):
                    r = int(idx.running[i])
                    ref = oracle_attention(trace, layer, idx.step, r,
                                           o["block_tables"][i][:(o["seq_lens"][i] + 15) // 16],
                                           o["seq_lens"][i])
                    assert float(np.abs(got[i] - ref).max()) <= 1e-2, (idx.step, r)
                    checked += 1
                    hits_checked += r in started_cached
        if idx.done:
            break
    import paged_kv_cache_400_b200 as pk
    assert pk.pa_get_device_error() == 0
    assert cached_total > 0 and hits_checked >= 5 and checked >= 20, (cached_total, hits_checked, checked)
    eng.close()


def oracle_prefill_row(trace, layer, req, table, length, pos):
    """Oracle: the prompt token at `pos` of a request whose first `length`
    positions hold the generator's K/V (written through its own table),
    attending causally to positions 0..pos, in fp64."""
    ids = sorted(set(table))
    remap = {b: i for i, b in enumerate(ids)}
    pool = np.zeros((len(ids), 2, trace.num_kv_heads, 16, trace.head_dim), dtype=np.uint16)
    k, v = trace.kv_values(layer, [req] * length, np.arange(length), "cpu")
    slots = [remap[table[p // 16]] * 16 + p % 16 for p in range(length)]
    assert oa.reshape_and_cache(pool, storage_bits(k), storage_bits(v), slots) == []
    q = storage_bits(trace.prompt_q_values(layer, [req], [pos], "cpu"))
    tab = [[remap[b] for b in table]]
    return oa.paged_prefill(q, pool, tab, [pos + 1], [1], trace.scale, "bf16")[0]


def test_trace_with_prefill_attention_matches_oracle():
    """The step loop with prefill attention on: each step's admitted prompts
    (fresh and recomputed after preemption) attend causally over their paged KV
    (pa_prefill after the prompt append). Sampled prompt rows match the fp64
    oracle; decode outputs of the same steps are unaffected."""
    from oracle_side import prefill_tolerance_ok
    trace = wl.trace_case(seed=7, n_requests=120, rate=12.0, num_blocks=1200, num_layers=2,
                          output_cap=200)
    eng = DecodeEngine(trace.num_blocks, trace.num_layers, trace.num_heads, trace.num_kv_heads,
                       trace.head_dim, trace.arrival_step, trace.prompt_len, trace.output_len,
                       trace.table_width, trace.scale, DEV)
    rng = np.random.default_rng(1)
    checked = prompts_seen = 0
    while True:
        idx = eng.schedule()
        if len(idx.running):
            reqs_p, pos_p = eng.prompt_positions(idx)
            inputs, _ = trace.step_inputs(idx.step, idx.running, idx.seq_lens, reqs_p, pos_p, DEV,
                                          stacked=True, prefill=True)
            eng.run_layers(idx, inputs)
            if len(idx.prompt_seqs):
                prompts_seen += len(idx.prompt_seqs)
                assert eng.prefill_out is not None and len(eng.prefill_out) == trace.num_layers
                assert pk_device_error() == 0
                if checked < 24:
                    layer = int(rng.integers(0, trace.num_layers))
                    starts = np.concatenate([[0], np.cumsum(idx.prompt_lens - idx.prompt_starts)])
                    row_of = {int(r): i for i, r in enumerate(idx.running)}
                    got_all = eng.prefill_out[layer].float().cpu().numpy()
                    for k in rng.choice(len(idx.prompt_seqs), size=min(2, len(idx.prompt_seqs)), replace=False):
                        req = int(idx.prompt_seqs[k])
                        n_new = int(idx.prompt_lens[k] - idx.prompt_starts[k])
                        for i in {0, n_new - 1, int(rng.integers(n_new))}:
                            pos = int(idx.prompt_starts[k]) + i
                            table = idx.block_tables[row_of[req]].tolist()
                            ref = oracle_prefill_row(trace, layer, req, table, int(idx.prompt_lens[k]), pos)
                            ok, err, _ = prefill_tolerance_ok(got_all[int(starts[k]) + i], ref)
                            assert ok, (idx.step, req, pos, err)
                            checked += 1
            else:
                assert eng.prefill_out is None
        if idx.done:
            break
    eng.close()
    assert checked >= 24 and prompts_seen >= 100


def pk_device_error():
    import paged_kv_cache_400_b200 as pk
    return pk.pa_get_device_error()


def test_prefix_cached_prompts_prefill_matches_oracle():
    """Prefill attention with prefix caching: a request whose system prompt
    blocks are cached prefills only its positions from prompt_starts on, yet
    those rows attend over the whole prompt, cached prefix included (written
    by an earlier request). Sampled rows of cache-hit prompts vs the oracle."""
    from oracle_side import prefill_tolerance_ok
    trace = wl.prefix_trace_case(seed=9, n_requests=90, rate=10.0, num_blocks=2400, num_layers=2, n_system=2)
    trace.output_len = np.minimum(trace.output_len, 120).astype(np.int32)
    eng = DecodeEngine(trace.num_blocks, trace.num_layers, trace.num_heads, trace.num_kv_heads,
                       trace.head_dim, trace.arrival_step, trace.prompt_len, trace.output_len,
                       trace.table_width, trace.scale, DEV, prompt_tokens=trace.prompt_tokens)
    rng = np.random.default_rng(4)
    hits = checked = 0
    while True:
        idx = eng.schedule()
        if len(idx.running):
            reqs_p, pos_p = eng.prompt_positions(idx)
            inputs, _ = trace.step_inputs(idx.step, idx.running, idx.seq_lens, reqs_p, pos_p, DEV,
                                          stacked=True, prefill=True)
            eng.run_layers(idx, inputs)
            cached = [k for k in range(len(idx.prompt_seqs)) if idx.prompt_starts[k] > 0]
            if cached and checked < 24:
                layer = int(rng.integers(0, trace.num_layers))
                starts = np.concatenate([[0], np.cumsum(idx.prompt_lens - idx.prompt_starts)])
                row_of = {int(r): i for i, r in enumerate(idx.running)}
                got_all = eng.prefill_out[layer].float().cpu().numpy()
                for k in cached[:2]:
                    req = int(idx.prompt_seqs[k])
                    n_new = int(idx.prompt_lens[k] - idx.prompt_starts[k])
                    table = idx.block_tables[row_of[req]].tolist()
                    for i in {0, n_new - 1, int(rng.integers(n_new))}:
                        pos = int(idx.prompt_starts[k]) + i
                        ref = oracle_prefill_row(trace, layer, req, table, int(idx.prompt_lens[k]), pos)
                        ok, err, _ = prefill_tolerance_ok(got_all[int(starts[k]) + i], ref)
                        assert ok, (idx.step, req, pos, err)
                        checked += 1
                    hits += 1
        if idx.done:
            break
    eng.close()
    assert pk_device_error() == 0
    assert hits >= 5 and checked >= 15
