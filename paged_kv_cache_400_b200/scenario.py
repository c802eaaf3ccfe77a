"""Host-side set-up of one decode step through the library's block manager.

Replays a workload's block-manager script (allocate / fork / free / append)
on a pa_bm handle, then appends one slot for every sequence of the decode
batch, collecting the copy-on-write pairs, and packs the batch's block tables
and lengths with pa_bm_pack. Everything it computes comes from C-ABI calls.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .binding import BlockManager


@dataclass
class PreparedStep:
    bm: BlockManager
    slot_mapping: np.ndarray     # int64 [B]: slot of each batch sequence's new token
    cow_src: np.ndarray          # int32 [n]
    cow_dst: np.ndarray          # int32 [n]
    block_tables: np.ndarray     # int32 [B][table_width]
    seq_lens: np.ndarray         # int32 [B]


def replay_ops(bm: BlockManager, ops) -> None:
    for op in ops:
        kind = op[0]
        if kind == "allocate":
            bm.allocate(op[1], op[2])
        elif kind == "fork":
            bm.fork(op[1], op[2])
        elif kind == "free":
            bm.free(op[1])
        elif kind == "append":
            bm.append_slot(op[1])
        else:
            raise ValueError(f"unknown op {kind!r}")


def prepare_decode_step(case) -> PreparedStep:
    bm = BlockManager(case.num_blocks, case.free_order)
    replay_ops(bm, case.ops)
    slots, cs, cd = [], [], []
    for seq in case.batch:
        s, a, b = bm.append_slot(seq)
        slots.append(s)
        if a >= 0:
            cs.append(a)
            cd.append(b)
    bt, sl, _ = bm.pack(case.batch, case.table_width)
    return PreparedStep(bm, np.asarray(slots, np.int64), np.asarray(cs, np.int32),
                        np.asarray(cd, np.int32), bt, sl)


@dataclass
class PreparedPrefill:
    bm: BlockManager
    slot_mapping: np.ndarray     # int64 [T]: slot of each new token (sequence order)
    block_tables: np.ndarray     # int32 [B][table_width]
    seq_lens: np.ndarray         # int32 [B]: KV length, new tokens included
    query_start: np.ndarray      # int32 [B+1]: first new-token row of each sequence


def prepare_prefill_step(case) -> PreparedPrefill:
    """Allocates every sequence's full length, then takes the slots of its new
    positions ctx .. ctx+n-1 and packs the tables (all through the C ABI)."""
    bm = BlockManager(case.num_blocks, case.free_order)
    replay_ops(bm, case.ops)
    seqs = list(range(len(case.query_lens)))
    slots = [bm.slots(b, int(c), int(n)) for b, (c, n) in enumerate(zip(case.ctx_lens, case.query_lens))]
    slot_mapping = np.concatenate(slots).astype(np.int64) if slots else np.zeros(0, np.int64)
    bt, sl, _ = bm.pack(seqs, case.table_width)
    qs = np.zeros(len(seqs) + 1, np.int32)
    qs[1:] = np.cumsum(np.asarray(case.query_lens, np.int64))
    return PreparedPrefill(bm, slot_mapping, bt, sl, qs)
