"""Test helper: the oracle's view of one decode-step workload.

Replays the workload's block-manager script on the oracle block manager,
builds the oracle's pool from the workload generator (only the blocks it
needs), applies the oracle's copy-on-write copies and cache append, and runs
the fp64 oracle attention. Nothing here reads a value produced by the CUDA
path.
"""
from __future__ import annotations

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


def oracle_outputs(case, ost: OracleStep, sample):
    """fp64 oracle output for batch rows `sample` ([len(sample)][H][D])."""
    return oracle_compute(oracle_inputs(case, ost, sample))


def tolerance_ok(case, out_gpu: np.ndarray, ref: np.ndarray):
    """The stated bar: fp32 max|err| / max|ref| <= 2e-5; bf16 max|err| <= 1e-2."""
    err = np.abs(out_gpu.astype(np.float64) - ref)
    if case.dtype == "f32":
        rel = err.max() / max(np.abs(ref).max(), 1e-30)
        return rel <= 2e-5, rel
    return err.max() <= 1e-2, err.max()
