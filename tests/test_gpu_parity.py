"""GPU parity: cache append, block copy and paged decode (through the C ABI)
against the fp64 oracle on the same seeded inputs.

Bars: indices, cache writes and block copies bit-exact; attention
fp32 max|err|/max|ref| <= 2e-5, bf16 max|err| <= 1e-2 (fp64 reference).
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_400_b200 as pk
from paged_kv_cache_400_b200 import workloads as wl
from paged_kv_cache_400_b200.scenario import prepare_decode_step

from oracle_side import oracle_indices, oracle_outputs, storage_bits, tolerance_ok

pytestmark = pytest.mark.gpu
DEV = "cuda"


def device_step(case, prep, pool=None):
    """The path as a user runs it: copy-on-write copies, append, decode."""
    if pool is None:
        pool = case.make_pool(DEV)
    q = case.make_q(DEV)
    k, v = case.make_kv_new(DEV)
    if len(prep.cow_src):
        pk.pa_copy_blocks(pool, torch.from_numpy(prep.cow_src).to(DEV),
                          torch.from_numpy(prep.cow_dst).to(DEV))
    pk.pa_reshape_and_cache(k, v, pool, torch.from_numpy(prep.slot_mapping).to(DEV))
    out = torch.empty_like(q)
    ws = pk.alloc_workspace(len(case.batch), case.num_heads, pool, case.max_seq_len)
    pk.pa_decode(out, q, pool, torch.from_numpy(prep.block_tables).to(DEV),
                 torch.from_numpy(prep.seq_lens).to(DEV), case.scale, case.max_seq_len, ws)
    assert pk.pa_get_device_error() == 0
    return pool, out


def check_case(case, sample=None):
    prep = prepare_decode_step(case)
    ost = oracle_indices(case)
    # indices: bit-exact with the oracle block manager
    assert prep.slot_mapping.tolist() == ost.slots
    assert list(zip(prep.cow_src.tolist(), prep.cow_dst.tolist())) == ost.cows
    assert prep.seq_lens.tolist() == ost.lens
    pool, out = device_step(case, prep)
    if sample is None:
        sample = list(range(len(case.batch)))
    ref = oracle_outputs(case, ost, sample)
    got = storage_bits(out[sample].float()).astype(np.float64) if case.dtype == "f32" else \
        out[sample].float().cpu().numpy().astype(np.float64)
    ok, err = tolerance_ok(case, got, ref)
    assert ok, f"{case.name}: error {err}"
    return prep, pool, out, err


# ---------------------------------------------------------------------------
# the five workload shapes
# ---------------------------------------------------------------------------
def test_tiny_fp32_full():
    case = wl.tiny_case(0)
    prep, pool, out, err = check_case(case)
    # whole pool bit-exact against the oracle's append on the generator's pool
    from oracle import attention as oa
    ref_pool = storage_bits(case.make_pool("cpu")).copy()
    k, v = case.make_kv_new("cpu")
    oa.reshape_and_cache(ref_pool, storage_bits(k), storage_bits(v), prep.slot_mapping)
    assert np.array_equal(storage_bits(pool).view(np.uint32), ref_pool.view(np.uint32))


def test_tiny_fp32_full_mantissa():
    """The tiny fp32 config with inputs whose fp32 significands are full (x *
    1.05 rounded once), so products in q.k and p.v round: held to the same
    2e-5 relative bar, and the appended pool bit-exact."""
    case = wl.tiny_case(0, full_mantissa=True)
    prep, pool, out, err = check_case(case)
    from oracle import attention as oa
    ref_pool = storage_bits(case.make_pool("cpu")).copy()
    k, v = case.make_kv_new("cpu")
    oa.reshape_and_cache(ref_pool, storage_bits(k), storage_bits(v), prep.slot_mapping)
    assert np.array_equal(storage_bits(pool).view(np.uint32), ref_pool.view(np.uint32))


@pytest.mark.parametrize("dim,heads,kv", [(64, 2, 2), (128, 8, 2), (64, 6, 1), (128, 32, 8)])
def test_fp32_full_mantissa_shapes(dim, heads, kv):
    """fp32 with full-significand inputs across tiles, ragged tails and several
    partitions (lengths 1 to 4096 on a 4096 bound), against the 2e-5 bar."""
    lens = [1, 15, 16, 17, 33, 129, 511, 513, 1025, 2048, 3001, 4096]
    case = wl.custom_case(f"f32full_{dim}_{heads}_{kv}", 8, lens, 1024, heads, kv, dim, "f32", 256, 4096,
                          full_mantissa=True)
    check_case(case)


def test_mha_every_sequence():
    """The Llama-2-7B-shaped MHA config at its stated size, all 64 sequences
    compared element by element with the fp64 oracle."""
    check_case(wl.mha_case(0))


def test_gqa_every_sequence():
    """The Llama-3-8B-shaped GQA batch of 256 at its stated size, every
    sequence compared element by element with the fp64 oracle."""
    check_case(wl.gqa_case(0))


def test_gqa_fused_step_every_sequence():
    """The same batch through pa_append_decode (the benchmarked step): every
    sequence against the oracle, and the appended pool rows bit-exact."""
    case = wl.gqa_case(0)
    prep = prepare_decode_step(case)
    ost = oracle_indices(case)
    pool = case.make_pool(DEV)
    q = case.make_q(DEV)
    k, v = case.make_kv_new(DEV)
    out = torch.empty_like(q)
    slots = torch.from_numpy(prep.slot_mapping).to(DEV)
    ws = pk.alloc_workspace(len(case.batch), case.num_heads, pool, case.max_seq_len)
    pk.pa_append_decode(out, q, k, v, pool, slots, torch.from_numpy(prep.block_tables).to(DEV),
                        torch.from_numpy(prep.seq_lens).to(DEV), case.scale, case.max_seq_len, ws)
    assert pk.pa_get_device_error() == 0
    blk, row = slots // 16, slots % 16
    assert torch.equal(pool[blk, 0, :, row, :], k) and torch.equal(pool[blk, 1, :, row, :], v)
    ref = oracle_outputs(case, ost, range(len(case.batch)))
    ok, err = tolerance_ok(case, out.float().cpu().numpy().astype(np.float64), ref)
    assert ok, err


def test_shared_prefix_with_copy_on_write():
    case = wl.prefix_case(0)
    sample = None  # every sequence: the 32 prefix sharers and the 8 x 4 samples
    prep, pool, out, err = check_case(case, sample)
    assert len(prep.cow_src) == 24
    # copied blocks are bit-identical to their sources except the appended row
    src = case.pool_blocks(prep.cow_src.tolist(), DEV)
    dst = pool[torch.from_numpy(prep.cow_dst).to(DEV).long()]
    slots = {int(s) for s in prep.slot_mapping}
    for i, d in enumerate(prep.cow_dst.tolist()):
        rows = [s % 16 for s in slots if s // 16 == d]
        keep = [r for r in range(16) if r not in rows]
        assert torch.equal(dst[i][:, :, keep], src[i][:, :, keep])


def test_pool_outside_appended_slots_is_untouched():
    case = wl.gqa_case(0)
    prep = prepare_decode_step(case)
    pool, _ = device_step(case, prep)
    ref = case.make_pool(DEV)
    k, v = case.make_kv_new(DEV)
    slots = torch.from_numpy(prep.slot_mapping).to(DEV)
    blk, row = slots // 16, slots % 16
    assert torch.equal(pool[blk, 0, :, row, :], k)
    assert torch.equal(pool[blk, 1, :, row, :], v)
    ref[blk, 0, :, row, :] = k
    ref[blk, 1, :, row, :] = v
    assert torch.equal(pool, ref)


# ---------------------------------------------------------------------------
# shapes, ragged tails, partitions
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype,dim,heads,kv", [
    ("f32", 64, 2, 2), ("f32", 128, 8, 2), ("bf16", 64, 4, 4), ("bf16", 128, 4, 4),
    ("bf16", 128, 8, 4), ("bf16", 128, 16, 4), ("bf16", 128, 32, 4), ("bf16", 128, 16, 1),
    ("bf16", 64, 12, 3), ("f32", 64, 6, 1),
])
def test_shapes_and_groups(dtype, dim, heads, kv):
    lens = [1, 2, 15, 16, 17, 31, 33, 100, 128, 129, 511, 512, 513, 700, 1025, 1500]
    case = wl.custom_case(f"shape_{dtype}_{dim}_{heads}_{kv}", 7, lens, 2048, heads, kv, dim,
                          dtype, 128, 2048)
    check_case(case)


def test_long_sequences_many_partitions():
    lens = [8192, 8191, 4097, 3, 16]
    case = wl.custom_case("long", 11, lens, 4096, 32, 8, 128, "bf16", 512, 8192)
    check_case(case)


@pytest.mark.parametrize("max_seq_len", [16384, 65536])
def test_long_max_context_uses_the_work_list(max_seq_len):
    # >= 32 partitions per sequence: persistent decode over the plan kernel's list
    lens = [1, 17, 512, 513, 3000, 9000, 16384, 5, 0, 700] if max_seq_len == 16384 else \
        [70000 // 2, 33, 1, 1025, 40000]
    lens = [n for n in lens if n >= 1]
    width = max_seq_len // 16
    case = wl.custom_case(f"wl_{max_seq_len}", 17, lens, 8192, 32, 8, 128, "bf16", width, max_seq_len)
    check_case(case)
    mha = wl.custom_case(f"wl_mha_{max_seq_len}", 18, [3, 4000, 12000], 2048, 32, 32, 128, "bf16", width,
                         max_seq_len)
    check_case(mha)


def _work_list_case():
    # 24 sequences up to 8192 tokens on 8 KV heads: four 2048-token partitions
    # at most, the persistent decode over the plan kernel's work list
    lens = [8192, 8191, 6145, 6144, 4097, 4096, 2049, 2048, 2047, 1, 16, 17, 3000, 5000, 7000, 100,
            1500, 2500, 3500, 4500, 5500, 6500, 7500, 33]
    return wl.custom_case("wl_graph", 19, lens, 8192, 32, 8, 128, "bf16", 512, 8192)


def test_work_list_ignores_stale_workspace_contents():
    # the plan kernel rewrites the item list, its count and the item counter
    # on every call, so whatever the workspace holds on entry (here all bits
    # set, then what a previous call left) gives the same output
    case = _work_list_case()
    prep, pool, ref, _ = check_case(case)
    q = case.make_q(DEV)
    bt = torch.from_numpy(prep.block_tables).to(DEV)
    sl = torch.from_numpy(prep.seq_lens).to(DEV)
    assert pk.pa_decode_partition_tokens(len(case.batch), 32, pool, 8192) == 2048
    ws = pk.alloc_workspace(len(case.batch), case.num_heads, pool, case.max_seq_len)
    ws.fill_(255)
    for _ in range(2):
        out = torch.empty_like(ref)
        pk.pa_decode(out, q, pool, bt, sl, case.scale, case.max_seq_len, ws)
        assert pk.pa_get_device_error() == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_work_list_decode_in_a_cuda_graph():
    # the plan kernel is a programmatic dependent of the kernel before it:
    # captured after a device copy (a non-kernel node before the plan) and
    # twice in a row (the second plan follows the first call's merge kernel);
    # replays are bit-identical to eager calls
    case = _work_list_case()
    prep, pool, ref, _ = check_case(case)
    q_src = case.make_q(DEV)
    q = torch.empty_like(q_src)
    bt = torch.from_numpy(prep.block_tables).to(DEV)
    sl = torch.from_numpy(prep.seq_lens).to(DEV)
    ws = pk.alloc_workspace(len(case.batch), case.num_heads, pool, case.max_seq_len)
    out1, out2 = torch.empty_like(ref), torch.empty_like(ref)
    q.copy_(q_src)
    pk.pa_decode(out1, q, pool, bt, sl, case.scale, case.max_seq_len, ws)   # eager first (attributes)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            q.copy_(q_src)
            pk.pa_decode(out1, q, pool, bt, sl, case.scale, case.max_seq_len, ws)
            pk.pa_decode(out2, q, pool, bt, sl, case.scale, case.max_seq_len, ws)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(3):
        out1.zero_()
        out2.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert pk.pa_get_device_error() == 0
        assert torch.equal(out1.view(torch.int16), ref.view(torch.int16))
        assert torch.equal(out2.view(torch.int16), ref.view(torch.int16))
    del g


def test_single_token_sequences():
    case = wl.custom_case("ones", 12, [1] * 40, 128, 32, 8, 128, "bf16", 4, 64)
    _, _, out, _ = check_case(case)


def test_zero_length_sequence_gives_zeros():
    case = wl.custom_case("zero", 13, [5, 40], 64, 4, 2, 64, "bf16", 8, 128)
    prep = prepare_decode_step(case)
    pool = case.make_pool(DEV)
    q = case.make_q(DEV)
    out = torch.full_like(q, 7.0)
    bt = torch.from_numpy(prep.block_tables).to(DEV)
    sl = torch.tensor([0, 40], dtype=torch.int32, device=DEV)
    pk.pa_decode(out, q, pool, bt, sl, case.scale, 128)
    assert pk.pa_get_device_error() == 0
    assert torch.all(out[0] == 0)
    assert not torch.any(out[1] == 7.0)


def test_empty_batch_and_empty_append_are_noops():
    case = wl.tiny_case(0)
    pool = case.make_pool(DEV)
    before = pool.clone()
    e = torch.empty(0, 2, 64, device=DEV)
    pk.pa_reshape_and_cache(e, e, pool, torch.empty(0, dtype=torch.int64, device=DEV))
    q = torch.empty(0, 2, 64, device=DEV)
    pk.pa_decode(q, q.clone(), pool, torch.empty(0, 4, dtype=torch.int32, device=DEV),
                 torch.empty(0, dtype=torch.int32, device=DEV), 0.1, 64)
    assert torch.equal(pool, before) and pk.pa_get_device_error() == 0


def test_physical_permutation_is_bit_invariant_on_gpu():
    case = wl.custom_case("perm", 14, [17, 300, 1000, 2047], 512, 32, 8, 128, "bf16", 128, 2048)
    prep = prepare_decode_step(case)
    pool, out = device_step(case, prep)
    perm = torch.randperm(case.num_blocks, generator=torch.Generator().manual_seed(3)).to(DEV)
    pool2 = torch.empty_like(pool)
    pool2[perm] = pool
    bt = torch.from_numpy(prep.block_tables).to(DEV).long()
    bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0)], bt).to(torch.int32)
    out2 = torch.empty_like(out)
    ws = pk.alloc_workspace(len(case.batch), case.num_heads, pool, case.max_seq_len)
    pk.pa_decode(out2, case.make_q(DEV), pool2, bt2, torch.from_numpy(prep.seq_lens).to(DEV),
                 case.scale, case.max_seq_len, ws)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_repeated_calls_are_deterministic():
    case = wl.custom_case("det", 15, [3000, 20, 900], 1024, 32, 8, 128, "bf16", 256, 4096)
    prep = prepare_decode_step(case)
    pool, out = device_step(case, prep)
    ws = pk.alloc_workspace(3, 32, pool, 4096)
    for _ in range(3):
        out2 = torch.empty_like(out)
        pk.pa_decode(out2, case.make_q(DEV), pool, torch.from_numpy(prep.block_tables).to(DEV),
                     torch.from_numpy(prep.seq_lens).to(DEV), case.scale, 4096, ws)
        assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


# ---------------------------------------------------------------------------
# device-side index checks: flagged and skipped, never dereferenced
# ---------------------------------------------------------------------------
def test_out_of_range_slot_is_flagged_and_skipped():
    case = wl.tiny_case(0)
    pool = case.make_pool(DEV)
    before = pool.clone()
    k, v = case.make_kv_new(DEV)
    slots = torch.tensor([64 * 16, -1, 5, 64 * 16 + 100], dtype=torch.int64, device=DEV)
    pk.pa_reshape_and_cache(k, v, pool, slots)
    flags = pk.pa_get_device_error()
    assert flags == pk.PA_DEVERR_SLOT
    before[0, 0, :, 5] = k[2]
    before[0, 1, :, 5] = v[2]
    assert torch.equal(pool, before)
    assert pk.pa_get_device_error() == 0  # cleared by the read


def test_bad_block_id_and_bad_length_are_flagged():
    case = wl.custom_case("bad", 16, [40, 40, 40], 64, 8, 2, 128, "bf16", 4, 64)
    prep = prepare_decode_step(case)
    pool = case.make_pool(DEV)
    q = case.make_q(DEV)
    bt = torch.from_numpy(prep.block_tables).to(DEV)
    bt[1, 1] = 1 << 20            # past the pool
    bt[2, 0] = -5
    out = torch.empty_like(q)
    pk.pa_decode(out, q, pool, bt, torch.from_numpy(prep.seq_lens).to(DEV), case.scale, 64)
    assert pk.pa_get_device_error() & pk.PA_DEVERR_BLOCK
    sl = torch.tensor([40, 65, -1], dtype=torch.int32, device=DEV)   # 65 > max_seq_len
    pk.pa_decode(out, q, pool, torch.from_numpy(prep.block_tables).to(DEV), sl, case.scale, 64)
    assert pk.pa_get_device_error() == pk.PA_DEVERR_SEQLEN
    assert torch.all(out[1] == 0) and torch.all(out[2] == 0)


def test_bad_copy_pair_is_flagged_and_skipped():
    case = wl.tiny_case(0)
    pool = case.make_pool(DEV)
    before = pool.clone()
    src = torch.tensor([3, 70], dtype=torch.int32, device=DEV)
    dst = torch.tensor([9, 2], dtype=torch.int32, device=DEV)
    pk.pa_copy_blocks(pool, src, dst)
    assert pk.pa_get_device_error() == pk.PA_DEVERR_BLOCK
    before[9] = before[3]
    assert torch.equal(pool, before)
