"""Continuous-batching decode loop over per-layer paged KV pools.

Each step the host scheduler (pa_sched_step, C++) decides which requests run,
which are admitted (their prompt K/V are (re)written: recompute), which grow a
block, which are preempted or finish; then, for every layer, the step's device
work runs through the C ABI: copy-on-write block copies, the prompt-token
append, then the decode-token append and paged decode over the running batch
in one call (pa_append_decode)
("vLLM 原理：PagedAttention 和 Continuous Batching" / "vLLM 的调度 / 调度流程";
"大模型推理性能优化：PagedAttention与Continuous Batching原理与实践" §2.3).

The model around attention is out of scope: the caller supplies the K/V of
(layer, request, position) and the query of (layer, step, request), e.g. the
seeded synthetic values of workloads.TraceCase.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

from . import binding as bd


@dataclass
class StepRecord:
    step: int
    num_running: int
    num_prompt_tokens: int
    admitted: int
    preempted: int
    finished: int
    num_free_blocks: int
    kernel_ms: float = 0.0     # device time of the layer loop (CUDA events)
    host_ms: float = 0.0       # pa_sched_step + index packing


@dataclass
class StepIndices:
    """Host copies of one step's index arrays (from pa_step_out)."""
    step: int
    running: np.ndarray
    seq_lens: np.ndarray
    block_tables: np.ndarray
    decode_slots: np.ndarray
    prompt_seqs: np.ndarray
    prompt_lens: np.ndarray
    prompt_starts: np.ndarray
    prompt_slots: np.ndarray
    cow_src: np.ndarray
    cow_dst: np.ndarray
    swap_out: np.ndarray       # [n][2] (device block, host block)
    swap_in: np.ndarray        # [n][2] (host block, device block)
    done: bool
    record: StepRecord = field(default=None)


class DecodeEngine:
    def __init__(self, num_blocks, num_layers, num_heads, num_kv_heads, head_dim, arrival_step,
                 prompt_len, output_len, table_width, scale, device, dtype=torch.bfloat16,
                 max_seq_len=None, prompt_tokens=None, swap_host_blocks=0):
        """prompt_tokens: per-request prompt token ids to turn on automatic
        prefix caching (admission reuses cached prompt blocks and only the KV
        after the cached prefix is written). swap_host_blocks: pinned host
        blocks per layer for swap-mode preemption (0: recompute only)."""
        self.device = torch.device(device)
        self.num_layers = num_layers
        self.num_heads = num_heads
        self.num_kv_heads = num_kv_heads
        self.head_dim = head_dim
        self.scale = scale
        self.table_width = table_width
        self.max_seq_len = max_seq_len or table_width * bd.BLOCK_SIZE
        self.bm = bd.BlockManager(num_blocks)
        if prompt_tokens is not None:
            self.bm.set_prefix_caching(True)
        self.sched = bd.Scheduler(self.bm, arrival_step, prompt_len, output_len, table_width)
        if prompt_tokens is not None:
            self.sched.set_prompt_tokens(prompt_tokens)
        self.host_pools = []
        if swap_host_blocks > 0:
            self.sched.set_swap(swap_host_blocks)
        shape = (num_blocks, 2, num_kv_heads, bd.BLOCK_SIZE, head_dim)
        self.pools = [torch.empty(shape, dtype=dtype, device=self.device) for _ in range(num_layers)]
        if swap_host_blocks > 0:
            hshape = (swap_host_blocks,) + shape[1:]
            self.host_pools = [torch.empty(hshape, dtype=dtype, pin_memory=True) for _ in range(num_layers)]
        self._ws = None
        self._ws_bytes = 0
        self.prefill_out = None

    def close(self):
        self.sched.close()
        self.bm.close()

    # ---- host side -----------------------------------------------------------
    def schedule(self) -> StepIndices:
        import time
        t0 = time.perf_counter()
        o = self.sched.step_raw()
        n = o.num_running

        def arr(ptr, count, dt, shape=None):
            if count == 0:
                return np.empty(shape if shape else 0, dtype=dt)
            a = np.ctypeslib.as_array(ptr, shape=(count,)).copy()
            return a.reshape(shape) if shape else a

        idx = StepIndices(
            step=o.step,
            running=arr(o.running, n, np.int64),
            seq_lens=arr(o.seq_lens, n, np.int32),
            block_tables=arr(o.block_tables, n * o.max_blocks_per_seq, np.int32,
                             (n, o.max_blocks_per_seq)),
            decode_slots=arr(o.decode_slots, n, np.int64),
            prompt_seqs=arr(o.prompt_seqs, o.num_prompt_seqs, np.int64),
            prompt_lens=arr(o.prompt_lens, o.num_prompt_seqs, np.int32),
            prompt_starts=arr(o.prompt_starts, o.num_prompt_seqs, np.int32),
            prompt_slots=arr(o.prompt_slots, o.num_prompt_tokens, np.int64),
            cow_src=arr(o.cow_src, o.num_cow, np.int32),
            cow_dst=arr(o.cow_dst, o.num_cow, np.int32),
            swap_out=np.stack([arr(o.swap_out_src, o.num_swap_out, np.int32),
                               arr(o.swap_out_dst, o.num_swap_out, np.int32)], axis=1),
            swap_in=np.stack([arr(o.swap_in_src, o.num_swap_in, np.int32),
                              arr(o.swap_in_dst, o.num_swap_in, np.int32)], axis=1),
            done=bool(o.done),
        )
        idx.record = StepRecord(o.step, n, o.num_prompt_tokens, o.num_admitted, o.num_preempted,
                                o.num_finished, o.num_free_blocks,
                                host_ms=1e3 * (time.perf_counter() - t0))
        return idx

    @staticmethod
    def prompt_positions(idx: StepIndices):
        """(request, position) of every prompt slot, in prompt_slots order
        (positions start..len-1 of each admitted request)."""
        counts = idx.prompt_lens - idx.prompt_starts
        reqs = np.repeat(idx.prompt_seqs, counts)
        pos = np.concatenate([np.arange(a, n) for a, n in zip(idx.prompt_starts, idx.prompt_lens)]) \
            if len(idx.prompt_lens) else np.empty(0, np.int64)
        return reqs, pos

    def prefill_indices(self, idx: StepIndices):
        """Device index arrays of the step's prefill: the admitted prompts'
        block tables (their rows of the step's tables), KV lengths (prompt
        lengths: the decode token comes after), query_start over the new
        positions prompt_starts .. prompt_lens - 1, and the longest run."""
        dev = self.device
        row = {int(r): i for i, r in enumerate(idx.running)}
        rows = np.asarray([row[int(r)] for r in idx.prompt_seqs], np.int64)
        counts = (idx.prompt_lens - idx.prompt_starts).astype(np.int64)
        qs = np.zeros(len(rows) + 1, np.int32)
        qs[1:] = np.cumsum(counts)
        bt = torch.from_numpy(np.ascontiguousarray(idx.block_tables[rows])).to(dev)
        sl = torch.from_numpy(idx.prompt_lens.astype(np.int32)).to(dev)
        return bt, sl, torch.from_numpy(qs).to(dev), int(counts.max()) if len(counts) else 0

    # ---- device side -------------------------------------------------------------
    def workspace(self, batch):
        """A workspace large enough for `batch` sequences (grown on demand: the
        partition size, hence the bytes needed, depends on the batch)."""
        need = bd.pa_decode_workspace_size(batch, self.num_heads, self.pools[0], self.max_seq_len)
        if need == 0:
            return None
        if self._ws is None or need > self._ws_bytes:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
            self._ws_bytes = need
        return self._ws

    def run_swaps(self, idx: StepIndices):
        """This step's swap copies, every layer: swap-out (device -> host) before
        swap-in (host -> device), both before any other write of the step."""
        if not len(idx.swap_out) and not len(idx.swap_in):
            return
        dev = self.device
        pairs = [(idx.swap_out, False), (idx.swap_in, True)]
        for arr, to_device in pairs:
            if not len(arr):
                continue
            src = torch.from_numpy(np.ascontiguousarray(arr[:, 0])).to(dev)
            dst = torch.from_numpy(np.ascontiguousarray(arr[:, 1])).to(dev)
            for pool, host in zip(self.pools, self.host_pools):
                if to_device:
                    bd.pa_copy_blocks_between(pool, host, src, dst)
                else:
                    bd.pa_copy_blocks_between(host, pool, src, dst)

    def run_layers(self, idx: StepIndices, inputs, out=None):
        """Device work of one step over all layers.

        inputs: per layer l, a dict with "q" [n][H][D], "k_dec", "v_dec" [n][Hkv][D]
        (the new token of each running request) and "k_prompt", "v_prompt"
        [T][Hkv][D] (the prompt K/V in prompt_slots order), all on the device;
        with "q_prompt" [T][H][D] (prompt queries, same order) the admitted
        prompts' causal prefill attention runs too (pa_prefill, after the prompt
        append), its outputs kept in self.prefill_out[l].
        Returns the attention outputs per layer ([n][H][D] each)."""
        dev = self.device
        n = len(idx.running)
        if n == 0:
            return []
        bt = torch.from_numpy(idx.block_tables).to(dev, non_blocking=True)
        sl = torch.from_numpy(idx.seq_lens).to(dev, non_blocking=True)
        ds = torch.from_numpy(idx.decode_slots).to(dev, non_blocking=True)
        ps = torch.from_numpy(idx.prompt_slots).to(dev, non_blocking=True) if len(idx.prompt_slots) else None
        cs = torch.from_numpy(idx.cow_src).to(dev) if len(idx.cow_src) else None
        cd = torch.from_numpy(idx.cow_dst).to(dev) if len(idx.cow_dst) else None
        ws = self.workspace(n)
        self.run_swaps(idx)
        pf = self.prefill_indices(idx) if (ps is not None and "q_prompt" in inputs[0]) else None
        self.prefill_out = [] if pf is not None else None
        outs = out if out is not None else [torch.empty(n, self.num_heads, self.head_dim,
                                                         dtype=self.pools[0].dtype, device=dev)
                                             for _ in range(self.num_layers)]
        for l, pool in enumerate(self.pools):
            x = inputs[l]
            if cs is not None:
                bd.pa_copy_blocks(pool, cs, cd)
            if ps is not None:
                bd.pa_reshape_and_cache(x["k_prompt"], x["v_prompt"], pool, ps)
            if pf is not None:
                # the admitted prompts' new positions attend causally over their KV
                pbt, psl, pqs, pmax = pf
                po = torch.empty_like(x["q_prompt"])
                bd.pa_prefill(po, x["q_prompt"], pool, pbt, psl, pqs, self.scale, pmax)
                self.prefill_out.append(po)
            # each running request's new token appended and attended in one call
            bd.pa_append_decode(outs[l], x["q"], x["k_dec"], x["v_dec"], pool, ds, bt, sl, self.scale,
                                self.max_seq_len, ws)
        return outs


class GraphedLayers:
    """The decode part of a step over all layers (each running request's new
    token appended and attended: pa_append_decode per layer) replayed as one
    CUDA graph per batch-size bucket (prompt appends, prefill attention and
    copy-on-write copies, whose sizes vary every step, run eagerly first).

    Padded rows have length 0 and slot -1: they append nothing and their
    output rows are zeros, so a bucket's graph serves any batch up to its size.
    Index arrays and per-layer inputs are copied into the graph's static
    buffers before each replay; prompt appends and copy-on-write copies (their
    sizes vary every step) run eagerly before it. Capture happens on first use
    of a bucket, after an eager warm-up of the same calls.
    """

    def __init__(self, engine: "DecodeEngine", max_batch: int, bucket: int = 64):
        self.eng = engine
        self.bucket = bucket
        self.max_batch = ((max_batch + bucket - 1) // bucket) * bucket
        dev, L = engine.device, engine.num_layers
        H, Hkv, D, W = engine.num_heads, engine.num_kv_heads, engine.head_dim, engine.table_width
        dt = engine.pools[0].dtype
        B = self.max_batch
        self.q = torch.zeros(L, B, H, D, dtype=dt, device=dev)
        self.k = torch.zeros(L, B, Hkv, D, dtype=dt, device=dev)
        self.v = torch.zeros(L, B, Hkv, D, dtype=dt, device=dev)
        self.out = torch.zeros(L, B, H, D, dtype=dt, device=dev)
        self.bt = torch.full((B, W), -1, dtype=torch.int32, device=dev)
        self.sl = torch.zeros(B, dtype=torch.int32, device=dev)
        self.slots = torch.full((B,), -1, dtype=torch.int64, device=dev)
        need = max(bd.pa_decode_workspace_size(n, H, engine.pools[0], engine.max_seq_len)
                   for n in range(bucket, B + 1, bucket))
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        self.graphs = {}

    def _calls(self, n):
        e = self.eng
        for l, pool in enumerate(e.pools):
            bd.pa_append_decode(self.out[l, :n], self.q[l, :n], self.k[l, :n], self.v[l, :n], pool,
                                self.slots[:n], self.bt[:n], self.sl[:n], e.scale, e.max_seq_len, self.ws)

    def _graph(self, n):
        g = self.graphs.get(n)
        if g is None:
            # eager warm-up (kernel attributes are set outside capture) on inert
            # rows only: length 0 and slot -1 append and read nothing
            self.sl[:n].zero_()
            self.slots[:n].fill_(-1)
            self._calls(n)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._calls(n)
            self.graphs[n] = g
        return g

    def run(self, idx: StepIndices, inputs, stacked=None):
        """inputs as for DecodeEngine.run_layers; `stacked` = (q [L][n][H][D],
        k [L][n][Hkv][D], v [L][n][Hkv][D]) of the decode tokens, when the
        caller has them in one tensor each (one copy each instead of per layer)."""
        e = self.eng
        dev = e.device
        n = len(idx.running)
        if n == 0:
            return []
        if n > self.max_batch:
            raise ValueError(f"batch {n} above the graphed maximum {self.max_batch}")
        nb = ((n + self.bucket - 1) // self.bucket) * self.bucket
        graph = self._graph(nb)  # captured on first use, before the rows are filled
        # eager, variable-size work first
        e.run_swaps(idx)
        cs = torch.from_numpy(idx.cow_src).to(dev) if len(idx.cow_src) else None
        cd = torch.from_numpy(idx.cow_dst).to(dev) if len(idx.cow_dst) else None
        ps = torch.from_numpy(idx.prompt_slots).to(dev, non_blocking=True) if len(idx.prompt_slots) else None
        pf = e.prefill_indices(idx) if (ps is not None and "q_prompt" in inputs[0]) else None
        e.prefill_out = [] if pf is not None else None
        for l, pool in enumerate(e.pools):
            if cs is not None:
                bd.pa_copy_blocks(pool, cs, cd)
            if ps is not None:
                bd.pa_reshape_and_cache(inputs[l]["k_prompt"], inputs[l]["v_prompt"], pool, ps)
            if pf is not None:
                po = torch.empty_like(inputs[l]["q_prompt"])
                bd.pa_prefill(po, inputs[l]["q_prompt"], pool, pf[0], pf[1], pf[2], e.scale, pf[3])
                e.prefill_out.append(po)
        # static buffers: this step's rows, then inert padding up to the bucket
        self.bt[:n].copy_(torch.from_numpy(idx.block_tables), non_blocking=True)
        self.sl[:n].copy_(torch.from_numpy(idx.seq_lens), non_blocking=True)
        self.slots[:n].copy_(torch.from_numpy(idx.decode_slots), non_blocking=True)
        if nb > n:
            self.bt[n:nb].fill_(-1)
            self.sl[n:nb].zero_()
            self.slots[n:nb].fill_(-1)
        if stacked is not None:
            self.q[:, :n].copy_(stacked[0])
            self.k[:, :n].copy_(stacked[1])
            self.v[:, :n].copy_(stacked[2])
        else:
            for l in range(e.num_layers):
                self.q[l, :n].copy_(inputs[l]["q"])
                self.k[l, :n].copy_(inputs[l]["k_dec"])
                self.v[l, :n].copy_(inputs[l]["v_dec"])
        graph.replay()
        return [self.out[l, :n] for l in range(e.num_layers)]
