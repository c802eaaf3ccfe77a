"""Test helper: the oracle's view of one decode-step workload.

Replays the workload's block-manager script on the oracle block manager,
builds the oracle's pool from the workload generator (only the blocks it
needs), applies the oracle's copy-on-write copies and cache append, and runs
the fp64 oracle attention. Nothing here reads a value produced by the CUDA
path.
"""
from __future__ import annotations

import time
from dataclasses import dataclass

import numpy as np
import torch

from oracle import attention as oa
from oracle.block_manager import OracleBlockManager


@dataclass
class OracleStep:
    bm: OracleBlockManager
    slots: list
    cows: list
    tables: list        # per batch sequence
    lens: list


def oracle_indices(case) -> OracleStep:
    bm = OracleBlockManager(case.num_blocks, case.free_order)
    for op in case.ops:
        kind = op[0]
        if kind == "allocate":
            bm.allocate(op[1], op[2])
        elif kind == "fork":
            bm.fork(op[1], op[2])
        elif kind == "free":
            bm.free(op[1])
        else:
            bm.append_slot(op[1])
    slots, cows = [], []
    for s in case.batch:
        slot, a, b = bm.append_slot(s)
        slots.append(slot)
        if a >= 0:
            cows.append((a, b))
    return OracleStep(bm, slots, cows, [bm.table(s) for s in case.batch],
                      [bm.seq_len(s) for s in case.batch])


def storage_bits(t: torch.Tensor) -> np.ndarray:
    """Host numpy array of a CPU tensor's elements: float32 as-is, bf16 as bits."""
    t = t.cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def oracle_inputs(case, ost: OracleStep, sample):
    """Generator inputs for the oracle run on batch rows `sample`.

    The oracle pool holds only the blocks the sampled rows read plus the
    copy-on-write sources feeding them; block ids are relabelled to that
    compact pool (the oracle is invariant under relabelling, which its pins
    check). Returns a dict consumed by oracle_compute."""
    needed = set()
    for i in sample:
        needed.update(ost.tables[i])
    for a, b in ost.cows:
        if b in needed:
            needed.add(a)
    ids = sorted(needed)
    remap = {b: i for i, b in enumerate(ids)}
    k, v = case.make_kv_new("cpu")
    k, v = storage_bits(k), storage_bits(v)
    rows, slots = [], []
    for t, s in enumerate(ost.slots):
        if s // 16 in remap:
            rows.append(t)
            slots.append(remap[s // 16] * 16 + s % 16)
    return {
        "pool": storage_bits(case.pool_blocks(ids)),
        "cow_src": [remap[a] for a, b in ost.cows if b in remap],
        "cow_dst": [remap[b] for a, b in ost.cows if b in remap],
        "k": k[rows], "v": v[rows], "slots": slots,
        "q": storage_bits(case.make_q("cpu"))[list(sample)],
        "tables": [[remap[b] for b in ost.tables[i]] for i in sample],
        "lens": [ost.lens[i] for i in sample],
        "scale": case.scale, "dtype": case.dtype,
    }


def oracle_compute(x):
    """The oracle's step on prepared inputs: copy-on-write copies, cache
    append, fp64 attention. Modifies x["pool"] in place."""
    assert oa.copy_blocks(x["pool"], x["cow_src"], x["cow_dst"]) == []
    assert oa.reshape_and_cache(x["pool"], x["k"], x["v"], x["slots"]) == []
    return oa.paged_decode(x["q"], x["pool"], x["tables"], x["lens"], x["scale"], x["dtype"])


def oracle_outputs(case, ost: OracleStep, sample, chunk: int = 16):
    """fp64 oracle output for batch rows `sample` ([len(sample)][H][D]), built
    `chunk` rows at a time (each chunk's pool holds only its blocks)."""
    sample = list(sample)
    parts = [oracle_compute(oracle_inputs(case, ost, sample[i:i + chunk]))
             for i in range(0, len(sample), chunk)]
    return np.concatenate(parts) if parts else np.zeros((0, case.num_heads, case.head_dim))


def tolerance_ok(case, out_gpu: np.ndarray, ref: np.ndarray):
    """The stated bar: fp32 max|err| / max|ref| <= 2e-5; bf16 max|err| <= 1e-2."""
    err = np.abs(out_gpu.astype(np.float64) - ref)
    if case.dtype == "f32":
        rel = err.max() / max(np.abs(ref).max(), 1e-30)
        return rel <= 2e-5, rel
    return err.max() <= 1e-2, err.max()


# ---------------------------------------------------------------------------
# prefill
# ---------------------------------------------------------------------------
@dataclass
class OraclePrefill:
    bm: OracleBlockManager
    slots: list          # per new token, sequence order
    tables: list
    lens: list


def oracle_prefill_indices(case) -> OraclePrefill:
    bm = OracleBlockManager(case.num_blocks, case.free_order)
    for _, seq, n in case.ops:
        bm.allocate(seq, n)
    slots = []
    for b, (c, n) in enumerate(zip(case.ctx_lens, case.query_lens)):
        slots.extend(bm.slots(b, c, n))
    seqs = range(len(case.query_lens))
    return OraclePrefill(bm, slots, [bm.table(b) for b in seqs], [bm.seq_len(b) for b in seqs])


def oracle_prefill_rows(case, ost: OraclePrefill, picks):
    """fp64 oracle output for selected new-token rows. picks: list of
    (sequence b, index i of its new tokens). Row (b, i) sits at position
    p = ctx_b + i and attends to positions 0..p, so each pick is the oracle's
    prefill of a one-token query over the first p+1 positions of b (after the
    step's append). Returns [len(picks)][H][D]."""
    starts = np.concatenate([[0], np.cumsum(case.query_lens)]).astype(np.int64)
    seqs = sorted({b for b, _ in picks})
    ids = sorted({blk for b in seqs for blk in ost.tables[b]})
    remap = {blk: j for j, blk in enumerate(ids)}
    pool = storage_bits(case.pool_blocks(ids))
    k, v = case.make_kv_new("cpu")
    k, v = storage_bits(k), storage_bits(v)
    rows, slots = [], []
    for b in seqs:
        for i in range(case.query_lens[b]):
            t = int(starts[b]) + i
            s = ost.slots[t]
            rows.append(t)
            slots.append(remap[s // 16] * 16 + s % 16)
    assert oa.reshape_and_cache(pool, k[rows], v[rows], slots) == []
    q = storage_bits(case.make_q("cpu"))
    out = []
    for b, i in picks:
        p = case.ctx_lens[b] + i
        qrow = q[int(starts[b]) + i][None]
        table = [remap[blk] for blk in ost.tables[b]]
        out.append(oa.paged_prefill(qrow, pool, [table], [p + 1], [1], case.scale, case.dtype)[0])
    return np.stack(out) if out else np.zeros((0, case.num_heads, case.head_dim))


def oracle_prefill_all(case, ost: OraclePrefill):
    """fp64 oracle output for every new-token row ([T][H][D]), one prefill call
    over the whole step (small cases)."""
    pool = storage_bits(case.make_pool("cpu")).copy()
    k, v = case.make_kv_new("cpu")
    assert oa.reshape_and_cache(pool, storage_bits(k), storage_bits(v), ost.slots) == []
    q = storage_bits(case.make_q("cpu"))
    return oa.paged_prefill(q, pool, ost.tables, ost.lens, case.query_lens, case.scale, case.dtype), pool


def oracle_prefill_inputs(case, ost: OraclePrefill, seqs):
    """Generator inputs for the oracle's prefill of whole sequences `seqs`
    (their blocks relabelled into a compact pool). Consumed by
    oracle_prefill_compute."""
    starts = np.concatenate([[0], np.cumsum(case.query_lens)]).astype(np.int64)
    ids = sorted({blk for b in seqs for blk in ost.tables[b]})
    remap = {blk: j for j, blk in enumerate(ids)}
    k, v = case.make_kv_new("cpu")
    k, v = storage_bits(k), storage_bits(v)
    q = storage_bits(case.make_q("cpu"))
    rows = [int(starts[b]) + i for b in seqs for i in range(case.query_lens[b])]
    return {
        "pool": storage_bits(case.pool_blocks(ids)),
        "k": k[rows], "v": v[rows], "q": q[rows],
        "slots": [remap[ost.slots[t] // 16] * 16 + ost.slots[t] % 16 for t in rows],
        "tables": [[remap[blk] for blk in ost.tables[b]] for b in seqs],
        "lens": [ost.lens[b] for b in seqs], "query_lens": [case.query_lens[b] for b in seqs],
        "scale": case.scale, "dtype": case.dtype,
    }


def oracle_prefill_compute(x):
    """The oracle's prefill step: append the new tokens' K/V, then causal
    fp64 attention of the new tokens. Modifies x["pool"] in place."""
    assert oa.reshape_and_cache(x["pool"], x["k"], x["v"], x["slots"]) == []
    return oa.paged_prefill(x["q"], x["pool"], x["tables"], x["lens"], x["query_lens"], x["scale"], x["dtype"])


BF16_UNIT_ROUNDOFF = 2.0 ** -8


def prefill_tolerance_ok(got: np.ndarray, ref: np.ndarray):
    """bf16 bar for prefill: |err| <= 1e-2 + u |ref|, u = 2^-8 the bf16 unit
    roundoff. The 1e-2 absolute bar plus the rounding of the stored result:
    early prompt positions average only a few V rows, so outputs reach ~6 in
    magnitude, where one bf16 rounding alone can exceed 1e-2. Returns (ok,
    max|err|, max of err / bar)."""
    err = np.abs(got.astype(np.float64) - ref)
    bar = 1e-2 + BF16_UNIT_ROUNDOFF * np.abs(ref)
    return bool((err <= bar).all()), float(err.max(initial=0.0)), float((err / bar).max(initial=0.0))


# ---------------------------------------------------------------------------
# continuous-batching trace
# ---------------------------------------------------------------------------
def oracle_trace_row(trace, layer, step, req, table, length):
    """Oracle decode output of one request at (layer, step) of a trace: the
    request's K/V for positions 0..length-1 (generator values) are written
    through its own block table into a compact pool by the oracle's append,
    then gathered and attended in fp64. Returns ([H][D] output, seconds of
    oracle work: append + attention, input generation excluded)."""
    ids = sorted(set(table))
    remap = {b: i for i, b in enumerate(ids)}
    pool = np.zeros((len(ids), 2, trace.num_kv_heads, 16, trace.head_dim), dtype=np.uint16)
    k, v = trace.kv_values(layer, [req] * length, np.arange(length), "cpu")
    k, v = storage_bits(k), storage_bits(v)
    q = storage_bits(trace.q_values(layer, step, [req], "cpu"))
    slots = [remap[table[p // 16]] * 16 + p % 16 for p in range(length)]
    tab = [[remap[b] for b in table]]
    t0 = time.perf_counter()
    assert oa.reshape_and_cache(pool, k, v, slots) == []
    out = oa.paged_decode(q, pool, tab, [length], trace.scale, "bf16")[0]
    return out, time.perf_counter() - t0
