"""GPU parity of paged prefill / chunked prefill (pa_reshape_and_cache of the
new tokens, then pa_prefill, through the C ABI) against the fp64 oracle on the
same seeded inputs.

Bars: slot mappings, tables and the appended pool bit-exact; attention
|err| <= 1e-2 + 2^-8 |ref| (bf16 storage of the result), fp32 accumulation.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_400_b200 as pk
from paged_kv_cache_400_b200 import binding as bd
from paged_kv_cache_400_b200 import workloads as wl
from paged_kv_cache_400_b200.scenario import prepare_prefill_step

from oracle_side import (oracle_prefill_all, oracle_prefill_indices, oracle_prefill_rows,
                         prefill_tolerance_ok, storage_bits)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True, params=["tcgen05", "mma_sync"])
def prefill_kernel(request):
    """Every test runs on each prefill kernel: the product library's tcgen05
    kernel and the comparison build's mma.sync kernel (a library of its own)."""
    variant = {"tcgen05": None, "mma_sync": "prefill_mma_sync"}[request.param]
    with bd.use_variant(variant):
        yield request.param


def device_prefill(case, prep, pool=None):
    if pool is None:
        pool = case.make_pool(DEV)
    q = case.make_q(DEV)
    k, v = case.make_kv_new(DEV)
    if case.num_tokens:
        pk.pa_reshape_and_cache(k, v, pool, torch.from_numpy(prep.slot_mapping).to(DEV))
    out = torch.zeros_like(q)
    pk.pa_prefill(out, q, pool, torch.from_numpy(prep.block_tables).to(DEV),
                  torch.from_numpy(prep.seq_lens).to(DEV), torch.from_numpy(prep.query_start).to(DEV),
                  case.scale, case.max_query_len)
    torch.cuda.synchronize()
    return pool, out


def check_indices(case, prep, ost):
    assert prep.slot_mapping.tolist() == ost.slots
    assert prep.seq_lens.tolist() == ost.lens
    for b, tab in enumerate(ost.tables):
        assert prep.block_tables[b, :len(tab)].tolist() == tab


def check_full(case):
    prep = prepare_prefill_step(case)
    ost = oracle_prefill_indices(case)
    check_indices(case, prep, ost)
    pool, out = device_prefill(case, prep)
    assert pk.pa_get_device_error() == 0
    ref, ref_pool = oracle_prefill_all(case, ost)
    assert np.array_equal(storage_bits(pool), ref_pool)
    ok, err, worst = prefill_tolerance_ok(out.float().cpu().numpy(), ref)
    assert ok, f"{case.name}: max|err| {err}, worst err/bar {worst}"
    return err


def test_whole_prompts_ragged():
    # lengths across tile and block boundaries: 1, 15, 16, 17, 64, 65, 100, 129
    case = wl.prefill_custom("prompts", 1, [0] * 8, [1, 15, 16, 17, 64, 65, 100, 129], 32, 8)
    check_full(case)


def test_chunked_with_context():
    case = wl.prefill_custom("chunks", 2, [0, 5, 16, 33, 200, 1], [7, 64, 1, 100, 65, 16], 32, 8)
    check_full(case)


@pytest.mark.parametrize("heads", [(8, 8), (8, 4), (8, 2), (8, 1), (16, 1)])
def test_head_groups(heads):
    H, Hkv = heads
    case = wl.prefill_custom(f"g{H // Hkv}", 3, [0, 40, 3], [70, 33, 130], H, Hkv)
    check_full(case)


def test_empty_sequences_mixed():
    case = wl.prefill_custom("empty", 4, [0, 20, 0, 17], [0, 0, 37, 0], 32, 8)
    prep = prepare_prefill_step(case)
    pool, out = device_prefill(case, prep)
    assert pk.pa_get_device_error() == 0
    ost = oracle_prefill_indices(case)
    ref, _ = oracle_prefill_all(case, ost)
    ok, err, _ = prefill_tolerance_ok(out.float().cpu().numpy(), ref)
    assert ok, err


def test_many_sequences_ragged():
    # 75 sequences (three passes of the kernel's 32-sequence unit lookup),
    # zero-length ones among them, chunks across tile and block boundaries
    rng = np.random.default_rng(14)
    n = rng.integers(0, 140, size=75)
    n[[0, 31, 32, 33, 63, 74]] = [0, 0, 65, 1, 0, 129]
    ctx = rng.integers(0, 90, size=75)
    case = wl.prefill_custom("many", 14, ctx.tolist(), n.tolist(), 16, 4)
    check_full(case)


def test_more_sequences_than_the_sorted_order():
    # 150 sequences: past 128 the units go out in sequence order (the lookup
    # by prefix sum over passes of 32); equal lengths among them (ties)
    rng = np.random.default_rng(16)
    n = rng.integers(0, 70, size=150)
    n[[0, 64, 127, 128, 149]] = [0, 33, 0, 65, 1]
    ctx = rng.integers(0, 40, size=150)
    ctx[100:110] = 7
    n[100:110] = 20
    case = wl.prefill_custom("many150", 16, ctx.tolist(), n.tolist(), 16, 8)
    check_full(case)


def test_a_thousand_short_sequences():
    # 1000 sequences past the sorted order: every CTA's lookups resume from
    # the pass of its previous unit (31 passes of 32 sequences)
    rng = np.random.default_rng(19)
    n = rng.integers(0, 40, size=1000)
    ctx = rng.integers(0, 24, size=1000)
    case = wl.prefill_custom("thousand", 19, ctx.tolist(), n.tolist(), 16, 8)
    check_full(case)


@pytest.mark.parametrize("nseq", [128, 129])
def test_sorted_order_boundary(nseq):
    # exactly the sorted order's 128 sequences (all four 32-sequence slots
    # full) and one more (index order); many equal lengths, some empty
    rng = np.random.default_rng(17 + nseq)
    n = rng.integers(0, 48, size=nseq)
    n[::7] = 16
    ctx = np.where(np.arange(nseq) % 5 == 0, 0, rng.integers(0, 30, size=nseq))
    case = wl.prefill_custom(f"order{nseq}", 17, ctx.tolist(), n.tolist(), 16, 8)
    check_full(case)


@pytest.mark.parametrize("where", [1, 40, 140])
def test_malformed_query_ranges_flagged(where):
    # a decreasing query_start (n < 0) or a range past the last q row makes
    # the sequence count no work and sets PA_DEVERR_SEQLEN, also when it comes
    # after the first 32 sequences or past the sorted order's 128; the
    # sequences before it are unaffected
    lens = [20] * 150
    case = wl.prefill_custom("badq", 15, [0] * 150, lens, 32, 8)
    prep = prepare_prefill_step(case)
    pool = case.make_pool(DEV)
    k, v = case.make_kv_new(DEV)
    pk.pa_reshape_and_cache(k, v, pool, torch.from_numpy(prep.slot_mapping).to(DEV))
    q = case.make_q(DEV)
    bt = torch.from_numpy(prep.block_tables).to(DEV)
    sl = torch.from_numpy(prep.seq_lens).to(DEV)
    ost = oracle_prefill_indices(case)
    ref = oracle_prefill_rows(case, ost, [(0, 0), (0, 19), (where - 1, 0), (where - 1, 19)])
    for bad in ("decreasing", "past_end"):
        qs = prep.query_start.copy()
        if bad == "decreasing":
            qs[where + 1] = qs[where] - 5
        else:
            qs[where + 1:] = case.num_tokens + 7
        out = torch.zeros_like(q)
        pk.pa_prefill(out, q, pool, bt, sl, torch.from_numpy(qs).to(DEV), case.scale, case.max_query_len)
        torch.cuda.synchronize()
        assert pk.pa_get_device_error() == pk.PA_DEVERR_SEQLEN, bad
        rows = [0, 19, int(qs[where - 1]), int(qs[where - 1]) + 19]
        ok, err, _ = prefill_tolerance_ok(out[rows].float().cpu().numpy(), ref)
        assert ok, (bad, err)


def test_nothing_to_do():
    pool = torch.zeros((4, 2, 8, 16, 128), dtype=torch.bfloat16, device=DEV)
    q = torch.zeros((0, 32, 128), dtype=torch.bfloat16, device=DEV)
    z = torch.zeros((0,), dtype=torch.int32, device=DEV)
    pk.pa_prefill(q, q, pool, torch.zeros((0, 1), dtype=torch.int32, device=DEV), z,
                  torch.zeros((1,), dtype=torch.int32, device=DEV), 0.1, 0)
    torch.cuda.synchronize()
    assert pk.pa_get_device_error() == 0


def test_max_group_long_prompt():
    # one 2000-token prompt with G = 16 (4-token tiles: 500 CTAs on one sequence)
    case = wl.prefill_custom("long_g16", 5, [0], [2000], 16, 1)
    prep = prepare_prefill_step(case)
    ost = oracle_prefill_indices(case)
    check_indices(case, prep, ost)
    pool, out = device_prefill(case, prep)
    assert pk.pa_get_device_error() == 0
    picks = [(0, i) for i in (0, 1, 2, 3, 15, 16, 17, 511, 1024, 1999)]
    ref = oracle_prefill_rows(case, ost, picks)
    got = np.stack([out[i].float().cpu().numpy() for _, i in picks])
    ok, err, _ = prefill_tolerance_ok(got, ref)
    assert ok, err


def _sampled(case, n_random, seed):
    prep = prepare_prefill_step(case)
    ost = oracle_prefill_indices(case)
    check_indices(case, prep, ost)
    pool, out = device_prefill(case, prep)
    assert pk.pa_get_device_error() == 0
    rng = np.random.default_rng(seed)
    longest = int(np.argmax(case.query_lens))
    picks = [(longest, 0), (longest, case.query_lens[longest] - 1), (0, 0),
             (len(case.query_lens) - 1, case.query_lens[-1] - 1)]
    for _ in range(n_random):
        b = int(rng.integers(len(case.query_lens)))
        picks.append((b, int(rng.integers(case.query_lens[b]))))
    ref = oracle_prefill_rows(case, ost, picks)
    starts = prep.query_start
    got = np.stack([out[int(starts[b]) + i].float().cpu().numpy() for b, i in picks])
    ok, err, _ = prefill_tolerance_ok(got, ref)
    assert ok, err


def test_prefill_full_size_sampled():
    _sampled(wl.prefill_case(0), 24, 0)


def test_chunked_prefill_full_size_sampled():
    _sampled(wl.chunked_prefill_case(0), 24, 1)


def test_long_context_chunk():
    # a 96-token chunk after 30 000 cached tokens (1882 blocks): long KV loops,
    # block ids read in many batches, a wide table
    case = wl.prefill_custom("long_ctx", 9, [30000, 200], [96, 40], 32, 8)
    prep = prepare_prefill_step(case)
    ost = oracle_prefill_indices(case)
    check_indices(case, prep, ost)
    pool, out = device_prefill(case, prep)
    assert pk.pa_get_device_error() == 0
    picks = [(0, 0), (0, 31), (0, 32), (0, 95), (1, 0), (1, 39)]
    ref = oracle_prefill_rows(case, ost, picks)
    got = np.stack([out[int(prep.query_start[b]) + i].float().cpu().numpy() for b, i in picks])
    ok, err, _ = prefill_tolerance_ok(got, ref)
    assert ok, err


def test_mha_full_prompts_sampled():
    # G = 1: 128 tokens per query tile, whole prompts up to 1000 tokens
    case = wl.prefill_custom("mha_prompts", 10, [0, 0, 0, 0], [1000, 129, 128, 5], 32, 32)
    prep = prepare_prefill_step(case)
    ost = oracle_prefill_indices(case)
    pool, out = device_prefill(case, prep)
    assert pk.pa_get_device_error() == 0
    picks = [(0, 0), (0, 127), (0, 128), (0, 255), (0, 999), (1, 128), (2, 127), (3, 4)]
    ref = oracle_prefill_rows(case, ost, picks)
    got = np.stack([out[int(prep.query_start[b]) + i].float().cpu().numpy() for b, i in picks])
    ok, err, _ = prefill_tolerance_ok(got, ref)
    assert ok, err


def test_physical_permutation_is_bit_invariant():
    # relabelling every physical block (pool rows moved, tables rewritten) must
    # not change a single output bit: placement never enters the arithmetic
    case = wl.prefill_custom("perm", 11, [0, 45, 300], [90, 64, 33], 32, 8)
    prep = prepare_prefill_step(case)
    pool, out = device_prefill(case, prep)
    perm = torch.from_numpy(np.random.default_rng(3).permutation(case.num_blocks)).to(DEV)
    pool2 = torch.empty_like(pool)
    pool2[perm] = pool
    bt = torch.from_numpy(prep.block_tables).to(DEV).long()
    bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0)], bt).int()
    out2 = torch.zeros_like(out)
    pk.pa_prefill(out2, case.make_q(DEV), pool2, bt2.contiguous(), torch.from_numpy(prep.seq_lens).to(DEV),
                  torch.from_numpy(prep.query_start).to(DEV), case.scale, case.max_query_len)
    torch.cuda.synchronize()
    assert pk.pa_get_device_error() == 0
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_repeated_calls_are_deterministic():
    case = wl.prefill_custom("det", 12, [10, 500], [200, 77], 32, 8)
    prep = prepare_prefill_step(case)
    pool, out = device_prefill(case, prep)
    args = (case.make_q(DEV), pool, torch.from_numpy(prep.block_tables).to(DEV),
            torch.from_numpy(prep.seq_lens).to(DEV), torch.from_numpy(prep.query_start).to(DEV),
            case.scale, case.max_query_len)
    for _ in range(3):
        again = torch.zeros_like(out)
        pk.pa_prefill(again, *args)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), again.view(torch.int16))


def _prefill_args(case):
    prep = prepare_prefill_step(case)
    pool = case.make_pool(DEV)
    k, v = case.make_kv_new(DEV)
    pk.pa_reshape_and_cache(k, v, pool, torch.from_numpy(prep.slot_mapping).to(DEV))
    return (case.make_q(DEV), pool, torch.from_numpy(prep.block_tables).to(DEV),
            torch.from_numpy(prep.seq_lens).to(DEV), torch.from_numpy(prep.query_start).to(DEV),
            case.scale, case.max_query_len)


def test_concurrent_launches_on_two_streams():
    # two launches in flight at once on two streams: each grid's running CTAs
    # take only that grid's units, so both outputs equal their lone runs bit
    # for bit
    a = _prefill_args(wl.chunked_prefill_case(3, batch=12, chunk=256))
    b = _prefill_args(wl.prefill_case(4, batch=24))
    ref_a, ref_b = torch.zeros_like(a[0]), torch.zeros_like(b[0])
    pk.pa_prefill(ref_a, *a)
    pk.pa_prefill(ref_b, *b)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for _ in range(3):
        got_a, got_b = torch.zeros_like(a[0]), torch.zeros_like(b[0])
        torch.cuda.synchronize()
        with torch.cuda.stream(s1):
            pk.pa_prefill(got_a, *a)
        with torch.cuda.stream(s2):
            pk.pa_prefill(got_b, *b)
        torch.cuda.synchronize()
        assert pk.pa_get_device_error() == 0
        assert torch.equal(got_a.view(torch.int16), ref_a.view(torch.int16))
        assert torch.equal(got_b.view(torch.int16), ref_b.view(torch.int16))


def test_graph_replay_matches_eager():
    args = _prefill_args(wl.prefill_custom("graph", 18, [0, 100, 7, 0], [300, 45, 1, 129], 32, 8))
    ref = torch.zeros_like(args[0])
    pk.pa_prefill(ref, *args)
    torch.cuda.synchronize()
    out = torch.zeros_like(args[0])
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        pk.pa_prefill(out, *args)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert pk.pa_get_device_error() == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_last_row_matches_decode():
    # the newest token's prefill row attends to the whole sequence, as decode does
    case = wl.prefill_custom("vs_decode", 6, [100, 0, 31], [50, 77, 1], 32, 8)
    prep = prepare_prefill_step(case)
    pool, out = device_prefill(case, prep)
    last = torch.from_numpy(prep.query_start[1:] - 1).long().to(DEV)
    q = case.make_q(DEV)[last].contiguous()
    dec = torch.empty_like(q)
    bt = torch.from_numpy(prep.block_tables).to(DEV)
    sl = torch.from_numpy(prep.seq_lens).to(DEV)
    ws = pk.alloc_workspace(3, 32, pool, int(prep.seq_lens.max()))
    pk.pa_decode(dec, q, pool, bt, sl, case.scale, int(prep.seq_lens.max()), ws)
    torch.cuda.synchronize()
    assert pk.pa_get_device_error() == 0
    assert (dec.float() - out[last].float()).abs().max().item() <= 1e-2


def test_bad_lengths_flagged():
    case = wl.prefill_custom("bad", 7, [0, 0], [20, 20], 32, 8)
    prep = prepare_prefill_step(case)
    pool = case.make_pool(DEV)
    before = pool.clone()
    q = case.make_q(DEV)
    out = torch.zeros_like(q)
    sl = torch.tensor([20, 10], dtype=torch.int32, device=DEV)   # n = 20 > L = 10
    pk.pa_prefill(out, q, pool, torch.from_numpy(prep.block_tables).to(DEV), sl,
                  torch.from_numpy(prep.query_start).to(DEV), case.scale, case.max_query_len)
    torch.cuda.synchronize()
    assert pk.pa_get_device_error() == pk.PA_DEVERR_SEQLEN
    assert torch.equal(pool, before)
    assert out[20:].abs().max().item() == 0.0   # the bad sequence is skipped


def test_bad_block_flagged():
    # block 1 of the table (positions 16..31) points outside the pool: flagged,
    # never read; rows 0..15 attend to block 0 only and stay exact
    case = wl.prefill_custom("badblk", 8, [0], [40], 32, 8)
    prep = prepare_prefill_step(case)
    pool = case.make_pool(DEV)
    k, v = case.make_kv_new(DEV)
    pk.pa_reshape_and_cache(k, v, pool, torch.from_numpy(prep.slot_mapping).to(DEV))
    bt = prep.block_tables.copy()
    bt[0, 1] = case.num_blocks + 5
    q = case.make_q(DEV)
    out = torch.zeros_like(q)
    pk.pa_prefill(out, q, pool, torch.from_numpy(bt).to(DEV), torch.from_numpy(prep.seq_lens).to(DEV),
                  torch.from_numpy(prep.query_start).to(DEV), case.scale, case.max_query_len)
    torch.cuda.synchronize()
    assert pk.pa_get_device_error() == pk.PA_DEVERR_BLOCK
    ost = oracle_prefill_indices(case)
    ref = oracle_prefill_rows(case, ost, [(0, i) for i in range(16)])
    ok, err, _ = prefill_tolerance_ok(out[:16].float().cpu().numpy(), ref)
    assert ok, err
    assert torch.isfinite(out.float()).all()


def test_unsupported_rejected():
    pool = torch.zeros((4, 2, 3, 16, 128), dtype=torch.bfloat16, device=DEV)
    q = torch.zeros((1, 9, 128), dtype=torch.bfloat16, device=DEV)  # G = 3
    one = torch.ones((1,), dtype=torch.int32, device=DEV)
    qs = torch.tensor([0, 1], dtype=torch.int32, device=DEV)
    with pytest.raises(pk.PagedKVError):
        pk.pa_prefill(q, q, pool, torch.zeros((1, 1), dtype=torch.int32, device=DEV), one, qs, 0.1, 1)
