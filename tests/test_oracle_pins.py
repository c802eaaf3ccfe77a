"""Pins of the oracle against what the pages and the mathematics fix (CPU only).

Each test checks the oracle against something other than itself: numbers the
pages print (tests/golden/page_arithmetic.json), closed forms, an independent
library routine (torch scaled_dot_product_attention, torch's bf16 conversion),
brute-force sums with math.fsum, and invariances.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle.block_manager import BMError, OracleBlockManager, blocks_for

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_arithmetic.json")


def golden():
    with open(GOLDEN) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# page arithmetic and the allocator: values printed on the pages
# ---------------------------------------------------------------------------
def test_blocks_for_tokens_golden():
    for row in golden()["blocks_for_tokens"]:
        assert blocks_for(row["tokens"]) == row["blocks"]
        bm = OracleBlockManager(4096)
        assert len(bm.allocate(7, row["tokens"])) == row["blocks"]


def test_page_size_golden():
    assert golden()["page_size"]["tokens_per_page"] == oa.BLOCK_SIZE == 16


def test_on_demand_growth_golden():
    g = golden()["on_demand_growth"]
    bm = OracleBlockManager(64)
    bm.allocate(1, g["start_tokens"])
    assert len(bm.table(1)) == g["start_pages"]
    # append tokens until the 1-based ordinal reaches each printed value
    ordinal = g["start_tokens"]
    while ordinal < g["token_ordinal_opening_new_page"]:
        before = len(bm.table(1))
        slot, cs, cd = bm.append_slot(1)
        ordinal += 1
        page_ordinal = bm.table(1).index(slot // 16) + 1
        if ordinal == g["token_ordinal_still_in_last_page"]:
            assert page_ordinal == g["page_ordinal_of_that_token"]
            assert len(bm.table(1)) == before
        if ordinal < g["token_ordinal_opening_new_page"]:
            assert len(bm.table(1)) == g["start_pages"]
        assert (cs, cd) == (-1, -1)
    assert ordinal == g["token_ordinal_opening_new_page"]
    assert len(bm.table(1)) == g["new_page_ordinal"]
    assert bm.table(1)[-1] * 16 == slot  # the new page's first row


def test_contiguous_waste_golden():
    g = golden()["contiguous_waste"]
    waste = 1.0 - g["used_tokens"] / g["reserved_tokens"]
    assert round(100 * waste) == g["waste_percent_rounded"]
    # paged: the same 500 tokens occupy ceil(500/16) pages, < 3% unused
    bm = OracleBlockManager(1024)
    bm.allocate(0, g["used_tokens"])
    assert 1.0 - g["used_tokens"] / (16 * len(bm.table(0))) < 0.03


def test_fresh_pool_first_allocation_golden():
    g = golden()["fresh_pool_first_allocation"]
    bm = OracleBlockManager(g["num_blocks"])
    assert bm.allocate(0, g["tokens"]) == g["blocks"]


def test_freed_blocks_return_and_are_reused():
    bm = OracleBlockManager(32)
    a = bm.allocate(0, 100)      # 7 blocks
    b = bm.allocate(1, 40)       # 3 blocks
    assert bm.num_free() == 22
    bm.free(0)
    assert bm.num_free() == 29
    assert list(bm.free_list)[-7:] == a  # tail, in table order
    bm.free(1)
    assert bm.num_free() == 32
    assert sorted(bm.free_list) == list(range(32))
    # exhaust the never-used blocks; the next allocation gets the freed ones
    bm.allocate(2, 22 * 16)
    assert bm.allocate(3, 16 * 10) == a + b


def test_allocation_is_all_or_nothing():
    bm = OracleBlockManager(4)
    bm.allocate(0, 40)
    before = (list(bm.free_list), dict(bm.tables), list(bm.refcount))
    with pytest.raises(BMError) as e:
        bm.allocate(1, 33)
    assert e.value.status == "NO_BLOCKS"
    assert (list(bm.free_list), dict(bm.tables), list(bm.refcount)) == before
    with pytest.raises(BMError):
        bm.allocate(0, 1)           # exists
    with pytest.raises(BMError):
        bm.free(9)                  # unknown
    with pytest.raises(BMError):
        bm.fork(9, 10)


def test_fork_shares_and_copy_on_write():
    bm = OracleBlockManager(16)
    bm.allocate(0, 20)             # pages [0, 1], last page holds 4 rows
    bm.fork(0, 1)
    bm.fork(0, 2)
    assert bm.table(1) == bm.table(2) == bm.table(0) == [0, 1]
    assert bm.refcount[0] == bm.refcount[1] == 3
    # first writer into the shared partial page copies it
    assert bm.append_slot(0) == (2 * 16 + 4, 1, 2)
    assert bm.table(0) == [0, 2] and bm.refcount[1] == 2 and bm.refcount[2] == 1
    assert bm.append_slot(1) == (3 * 16 + 4, 1, 3)
    # the last holder writes in place
    assert bm.append_slot(2) == (1 * 16 + 4, -1, -1)
    assert bm.refcount[1] == 1
    # shared full page: no copy, a fresh page
    bm2 = OracleBlockManager(8)
    bm2.allocate(0, 32)
    bm2.fork(0, 1)
    assert bm2.append_slot(1) == (2 * 16, -1, -1)
    assert bm2.table(1) == [0, 1, 2] and bm2.refcount[1] == 2
    # freeing a sharer only drops counts
    bm2.free(0)
    assert bm2.refcount[0] == 1 and 0 not in bm2.free_list


def test_block_manager_invariants_random_ops():
    rng = np.random.default_rng(7)
    N = 48
    bm = OracleBlockManager(N, rng.permutation(N))
    live = set()
    nxt = 0
    for _ in range(3000):
        op = rng.integers(0, 4)
        try:
            if op == 0:
                bm.allocate(nxt, int(rng.integers(0, 70)))
                live.add(nxt)
                nxt += 1
            elif op == 1 and live:
                bm.append_slot(int(rng.choice(sorted(live))))
            elif op == 2 and live:
                bm.fork(int(rng.choice(sorted(live))), nxt)
                live.add(nxt)
                nxt += 1
            elif op == 3 and live:
                s = int(rng.choice(sorted(live)))
                bm.free(s)
                live.discard(s)
        except BMError as e:
            assert e.status == "NO_BLOCKS"
        held = {}
        for s, tab in bm.tables.items():
            assert len(tab) == blocks_for(bm.lens[s])
            for blk in tab:
                held[blk] = held.get(blk, 0) + 1
        for blk in range(N):
            assert bm.refcount[blk] == held.get(blk, 0)
        assert not (set(bm.free_list) & set(held))
        assert len(bm.free_list) + len(held) == N


# ---------------------------------------------------------------------------
# bf16 decoding: checked against torch's own bf16 -> fp64 conversion
# ---------------------------------------------------------------------------
def test_bf16_decoding_matches_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oa.bf16_bits_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    finite = np.isfinite(ref)
    assert np.array_equal(ours[finite], ref[finite])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.array_equal(np.isinf(ours), np.isinf(ref))


# ---------------------------------------------------------------------------
# helpers: random paged inputs built independently of the oracle's gather
# ---------------------------------------------------------------------------
def scatter_logical(K, V, num_blocks, rng):
    """Place logical per-sequence K/V [L][Hkv][D] into a random pool; returns
    pool, tables. Written with its own loops so it shares nothing with the
    oracle's gather."""
    n_kv, d = K[0].shape[1], K[0].shape[2]
    pool = rng.standard_normal((num_blocks, 2, n_kv, 16, d))  # garbage elsewhere
    free = list(rng.permutation(num_blocks))
    tables = []
    for Kb, Vb in zip(K, V):
        L = Kb.shape[0]
        nb = -(-L // 16)
        tab = [int(free.pop()) for _ in range(nb)]
        for t in range(L):
            pool[tab[t // 16], 0, :, t % 16, :] = Kb[t]
            pool[tab[t // 16], 1, :, t % 16, :] = Vb[t]
        tables.append(tab + [-1] * 4)
    return pool, tables


def random_logical(rng, lens, n_kv, d):
    K = [rng.standard_normal((L, n_kv, d)) for L in lens]
    V = [rng.standard_normal((L, n_kv, d)) for L in lens]
    return K, V


# ---------------------------------------------------------------------------
# attention: closed forms
# ---------------------------------------------------------------------------
def test_single_token_returns_its_value_exactly():
    rng = np.random.default_rng(1)
    K, V = random_logical(rng, [1, 1], 2, 8)
    pool, tables = scatter_logical(K, V, 10, rng)
    q = rng.standard_normal((2, 4, 8))
    out = oa.paged_decode(q, pool, tables, [1, 1], 0.3, "f64")
    for b in range(2):
        for h in range(4):
            assert np.array_equal(out[b, h], V[b][0, h // 2])


def test_equal_keys_or_zero_query_give_mean_value():
    rng = np.random.default_rng(2)
    L = 37
    Krow = rng.standard_normal((1, 2, 8))
    K = [np.repeat(Krow, L, axis=0)]
    V = [rng.standard_normal((L, 2, 8))]
    pool, tables = scatter_logical(K, V, 8, rng)
    q = rng.standard_normal((1, 2, 8))
    out = oa.paged_decode(q, pool, tables, [L], 1.7, "f64")
    np.testing.assert_allclose(out[0], V[0].mean(axis=0), rtol=0, atol=1e-14)
    K2 = [rng.standard_normal((L, 2, 8))]
    pool2, tables2 = scatter_logical(K2, V, 8, rng)
    out0 = oa.paged_decode(np.zeros((1, 2, 8)), pool2, tables2, [L], 1.0, "f64")
    np.testing.assert_allclose(out0[0], V[0].mean(axis=0), rtol=0, atol=1e-14)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(3)
    L = 50
    K, V = random_logical(rng, [L], 1, 16)
    q = rng.standard_normal((1, 1, 16))
    star = 37                                   # third page, row 5
    K[0][star, 0] = 50.0 * q[0, 0] / np.linalg.norm(q[0, 0])
    pool, tables = scatter_logical(K, V, 9, rng)
    out = oa.paged_decode(q, pool, tables, [L], 1000.0, "f64")
    np.testing.assert_allclose(out[0, 0], V[0][star, 0], rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# attention: an independent library routine on the unpaged data
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("n_heads,n_kv", [(4, 4), (8, 2), (6, 1)])
def test_matches_contiguous_sdpa(n_heads, n_kv):
    rng = np.random.default_rng(4 + n_heads)
    lens = [1, 15, 16, 17, 40, 100]
    d = 32
    K, V = random_logical(rng, lens, n_kv, d)
    pool, tables = scatter_logical(K, V, 64, rng)
    q = rng.standard_normal((len(lens), n_heads, d))
    scale = d ** -0.5
    out = oa.paged_decode(q, pool, tables, lens, scale, "f64")
    G = n_heads // n_kv
    for b, L in enumerate(lens):
        kt = torch.from_numpy(K[b]).permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
        vt = torch.from_numpy(V[b]).permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
        qt = torch.from_numpy(q[b])[None, :, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
        np.testing.assert_allclose(out[b], ref[0, :, 0, :].numpy(), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# attention: brute force with exactly rounded sums
# ---------------------------------------------------------------------------
def test_brute_force_fsum_tiny():
    rng = np.random.default_rng(5)
    lens = [1, 3, 16, 17, 33]
    n_heads, n_kv, d = 4, 2, 4
    K, V = random_logical(rng, lens, n_kv, d)
    pool, tables = scatter_logical(K, V, 16, rng)
    q = rng.standard_normal((len(lens), n_heads, d))
    scale = 0.5
    out = oa.paged_decode(q, pool, tables, lens, scale, "f64")
    for b, L in enumerate(lens):
        for h in range(n_heads):
            g = h // (n_heads // n_kv)
            s = [scale * math.fsum(float(q[b, h, i]) * float(K[b][t, g, i]) for i in range(d))
                 for t in range(L)]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            z = math.fsum(e)
            for i in range(d):
                o = math.fsum(e[t] * float(V[b][t, g, i]) for t in range(L)) / z
                assert abs(o - out[b, h, i]) <= 1e-13 * max(1.0, abs(o))


# ---------------------------------------------------------------------------
# attention: invariance under physical placement; split-KV merge
# ---------------------------------------------------------------------------
def test_permutation_of_physical_blocks_is_bit_invariant():
    rng = np.random.default_rng(6)
    lens = [5, 16, 17, 33, 64]
    K, V = random_logical(rng, lens, 2, 8)
    pool, tables = scatter_logical(K, V, 40, rng)
    q = rng.standard_normal((len(lens), 4, 8))
    out = oa.paged_decode(q, pool, tables, lens, 0.4, "f64")
    perm = rng.permutation(40)
    pool2 = np.empty_like(pool)
    pool2[perm] = pool
    tables2 = [[int(perm[x]) if x >= 0 else -1 for x in t] for t in tables]
    out2 = oa.paged_decode(q, pool2, tables2, lens, 0.4, "f64")
    assert np.array_equal(out, out2)


@pytest.mark.parametrize("part", [16, 32, 48, 7, 1000])
def test_split_kv_merge_equals_unsplit(part):
    rng = np.random.default_rng(8)
    lens = [1, 16, 17, 100, 257]
    K, V = random_logical(rng, lens, 2, 16)
    pool, tables = scatter_logical(K, V, 64, rng)
    q = 3.0 * rng.standard_normal((len(lens), 4, 16))
    a = oa.paged_decode(q, pool, tables, lens, 0.25, "f64")
    b = oa.paged_decode_split(q, pool, tables, lens, 0.25, "f64", part)
    np.testing.assert_allclose(b, a, rtol=0, atol=1e-12)


def test_partition_state_closed_form():
    # two tokens: m = max(s0, s1), l = 1 + exp(min - max)
    q = np.array([1.0, 0.0])
    K = np.array([[2.0, 0.0], [-1.0, 5.0]])
    V = np.array([[1.0, 2.0], [3.0, 4.0]])
    m, l, acc = oa.partition_state(q, K, V, 0.5, 0, 2)
    assert m == 1.0
    assert l == pytest.approx(1.0 + math.exp(-1.5), abs=1e-15)
    np.testing.assert_allclose(acc, V[0] + math.exp(-1.5) * V[1], atol=1e-15)
    merged = oa.merge_partition_states([oa.partition_state(q, K, V, 0.5, 0, 1),
                                        oa.partition_state(q, K, V, 0.5, 1, 2)])
    np.testing.assert_allclose(merged, acc / l, atol=1e-15)


# ---------------------------------------------------------------------------
# cache append and block copy
# ---------------------------------------------------------------------------
def test_reshape_and_cache_round_trip_and_bounds():
    rng = np.random.default_rng(9)
    pool = rng.integers(-30000, 30000, size=(6, 2, 3, 16, 8)).astype(np.int16)
    orig = pool.copy()
    k = rng.integers(-30000, 30000, size=(4, 3, 8)).astype(np.int16)
    v = rng.integers(-30000, 30000, size=(4, 3, 8)).astype(np.int16)
    slots = np.array([5 * 16 + 15, -1, 96, 2 * 16 + 0])
    rejected = oa.reshape_and_cache(pool, k, v, slots)
    assert rejected == [2]
    assert np.array_equal(pool[5, 0, :, 15], k[0]) and np.array_equal(pool[5, 1, :, 15], v[0])
    assert np.array_equal(pool[2, 0, :, 0], k[3]) and np.array_equal(pool[2, 1, :, 0], v[3])
    mask = np.ones(pool.shape, bool)
    mask[5, :, :, 15] = False
    mask[2, :, :, 0] = False
    assert np.array_equal(pool[mask], orig[mask])
    # the appended token is the last token gathered through a table
    K, V = oa.gather_kv(pool, [4, 5], 32, "f64")
    assert np.array_equal(K[31], k[0].astype(np.float64))


def test_copy_blocks_bits_and_bounds():
    rng = np.random.default_rng(10)
    pool = rng.integers(0, 65535, size=(5, 2, 2, 16, 4)).astype(np.uint16)
    orig = pool.copy()
    rejected = oa.copy_blocks(pool, [1, 3, 7], [4, 0, 2])
    assert rejected == [2]
    assert np.array_equal(pool[4], orig[1]) and np.array_equal(pool[0], orig[3])
    assert np.array_equal(pool[[1, 2, 3]], orig[[1, 2, 3]])


# ---------------------------------------------------------------------------
# prefill (causal) oracle
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("n_heads,n_kv", [(4, 4), (8, 2)])
def test_prefill_matches_causal_sdpa(n_heads, n_kv):
    rng = np.random.default_rng(20 + n_heads)
    lens, qlens = [1, 17, 40, 70], [1, 17, 12, 33]     # full prompts and chunks after a context
    d = 16
    K, V = random_logical(rng, lens, n_kv, d)
    pool, tables = scatter_logical(K, V, 32, rng)
    q = rng.standard_normal((sum(qlens), n_heads, d))
    out = oa.paged_prefill(q, pool, tables, lens, qlens, 0.3, "f64")
    G = n_heads // n_kv
    row = 0
    for b, (L, n) in enumerate(zip(lens, qlens)):
        kt = torch.from_numpy(K[b]).permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
        vt = torch.from_numpy(V[b]).permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
        qt = torch.from_numpy(q[row:row + n]).permute(1, 0, 2)[None]
        # causal with the queries at the last n positions: mask[i, t] = t <= L - n + i
        mask = torch.arange(L)[None, :] <= (L - n + torch.arange(n))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=0.3)
        np.testing.assert_allclose(out[row:row + n], ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
        row += n


def test_prefill_last_row_is_decode_and_first_token_sees_itself():
    rng = np.random.default_rng(30)
    lens, qlens = [33], [33]
    K, V = random_logical(rng, lens, 2, 8)
    pool, tables = scatter_logical(K, V, 8, rng)
    q = rng.standard_normal((33, 4, 8))
    pre = oa.paged_prefill(q, pool, tables, lens, qlens, 0.5, "f64")
    dec = oa.paged_decode(q[-1:], pool, tables, lens, 0.5, "f64")
    assert np.array_equal(pre[-1], dec[0])
    for h in range(4):
        assert np.array_equal(pre[0, h], V[0][0, h // 2])


def test_prefill_brute_force_fsum_tiny():
    """Prefill oracle against sums written out with math.fsum: each new token at
    position p scores positions 0..p only, softmax-normalised, over its own KV
    head; chunks after cached context and GQA grouping included."""
    rng = np.random.default_rng(31)
    lens, qlens, n_heads, n_kv, d, scale = [9, 20], [9, 4], 4, 2, 4, 0.7
    K, V = random_logical(rng, lens, n_kv, d)
    pool, tables = scatter_logical(K, V, 8, rng)
    q = rng.standard_normal((sum(qlens), n_heads, d))
    out = oa.paged_prefill(q, pool, tables, lens, qlens, scale, "f64")
    G = n_heads // n_kv
    row = 0
    for b, (L, n) in enumerate(zip(lens, qlens)):
        for i in range(n):
            p = L - n + i
            for h in range(n_heads):
                g = h // G
                s = [scale * math.fsum(float(q[row + i, h, c]) * float(K[b][t, g, c]) for c in range(d))
                     for t in range(p + 1)]
                m = max(s)
                e = [math.exp(x - m) for x in s]
                z = math.fsum(e)
                for c in range(d):
                    o = math.fsum(e[t] * float(V[b][t, g, c]) for t in range(p + 1)) / z
                    assert abs(out[row + i, h, c] - o) <= 1e-12 * max(1.0, abs(o))
        row += n
