"""Benchmark: paged decode attention + cache append on the Llama-3-8B-shaped GQA
decode step (32 query / 8 KV heads, head_dim 128, bf16, block 16, batch 256,
lognormal lengths median 1000 sigma 0.8 clipped to [16, 8192], random block
placement in a 32768-block pool).

One step = one pass of the hot path over the batch: append the batch's new
K/V into their slots (pa_reshape_and_cache), then split-KV paged decode with
its partition reduce (pa_decode). Inputs are resident in HBM before timing;
the KV read per step (~1.5 GB) is far larger than L2, so no flush is needed.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs its own independent batch (seed = rank): the
path has no exchange step, so ranks share nothing but the barrier and the
max-over-ranks timing ("weak" scaling). --impl reference times the fp64 CPU
oracle on a bounded sample of the same workload (rank 0 only).

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode-attn tokens/s; KV-read HBM GB/s as fraction of ~8 TB/s peak"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "pa_decode_gqa_b256.json")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--workload", choices=["gqa", "mha", "prefix", "trace", "prefix_trace", "prefill",
                                           "chunked_prefill"], default="gqa",
                    help="gqa is the benchmark line; the others are extra measurements")
    ap.add_argument("--trace-layers", type=int, default=32)
    ap.add_argument("--trace-requests", type=int, default=2000)
    ap.add_argument("--swap-host-blocks", type=int, default=0,
                    help="trace: pinned host blocks per layer for swap-mode preemption (0: recompute)")
    ap.add_argument("--no-prefix-cache", action="store_true",
                    help="prefix_trace: run without automatic prefix caching (for comparison)")
    ap.add_argument("--prefill", action="store_true",
                    help="trace: also run the admitted prompts' causal prefill attention (pa_prefill) per layer")
    ap.add_argument("--prefill-kernel", choices=["tcgen05", "mma_sync"], default="tcgen05",
                    help="prefill workloads: the product kernel, or a comparison build's kernel")
    ap.add_argument("--graphs", action="store_true",
                    help="trace: replay each step's decode over all layers as a CUDA graph")
    ap.add_argument("--batch", type=int, default=256,
                    help="sequences per GPU (256 is the workload; smaller only for profiling captures)")
    ap.add_argument("--prefill-batch", type=int, default=64,
                    help="prefill workloads: sequences per GPU (64 is the workload; smaller for captures)")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="bounded oracle sample for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-cpu-seconds", type=float, default=4.0,
                    help="bounded oracle sample of the chunked-prefill leg")
    ap.add_argument("--no-prefill-leg", action="store_true",
                    help="gqa: skip the prefill measurements added to the line (chunked, whole prompts)")
    ap.add_argument("--kv-util-jsonl", default=None,
                    help="trace: write each step's KV-cache utilisation record to this file")
    return ap.parse_args()


WORKLOAD_TEXT = {
    "gqa_llama3_8b": "gqa_llama3_8b_decode: 32 q / 8 kv heads, head_dim 128, bf16, block_size 16, "
                     "batch {B}, seq_lens lognormal(median 1000, sigma 0.8) clipped [16, 8192], "
                     "32768-block pool, random placement; step = cache append + split-KV decode",
    "mha_llama2_7b": "mha_llama2_7b_decode: 32 q = 32 kv heads, head_dim 128, bf16, block_size 16, "
                     "batch {B}, seq_lens uniform [128, 2048], 16384-block pool, random placement; "
                     "step = cache append + split-KV decode",
    "shared_prefix": "shared_prefix_decode: 32 seqs sharing a 1536-token prefix + suffixes U[0,512], "
                     "8 prompts x 4 samples forking at a partial block (copy-on-write); 32/8 heads, "
                     "head_dim 128, bf16, 4096-block pool; step = COW block copy + append + decode",
}


def workload_description(case, seq_lens):
    lens = np.asarray(seq_lens)
    return {
        "workload": WORKLOAD_TEXT[case.name].format(B=len(case.batch)),
        "global_batch": None,
        "seq_len_mean": float(lens.mean()),
        "seq_len_max": int(lens.max()),
        "tokens_in_cache": int(lens.sum()),
        "l2": "no flush: inputs larger than L2 (KV read per step %.2f GB vs 126 MB L2)"
              % (lens.sum() * 2 * case.num_kv_heads * case.head_dim * 2 / 1e9),
    }


def rank_case(seed: int, rank: int, batch: int, workload: str = "gqa"):
    """The batch a rank owns: an independent decode batch (seed + rank)."""
    from paged_kv_cache_400_b200 import workloads as wl
    if workload == "mha":
        return wl.mha_case(seed + rank)
    if workload == "prefix":
        return wl.prefix_case(seed + rank)
    return wl.gqa_case(seed + rank, batch=batch)


def max_over_ranks(value: float, dist, device) -> float:
    """Largest value over all ranks (the job's time is its slowest rank's)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def algorithmic_bytes(case, prep, partitions_per_seq, max_partitions):
    """Bytes the step must move at minimum (the kernel's roofline traffic)."""
    elt = 2
    lens = prep.seq_lens.astype(np.int64)
    B, H, Hkv, D = len(lens), case.num_heads, case.num_kv_heads, case.head_dim
    kv = int(lens.sum()) * 2 * Hkv * D * elt                       # K and V rows read
    qo = 2 * B * H * D * elt                                       # q read, out written
    tables = int(((lens + 15) // 16).sum()) * 4 + B * 4            # table entries + lengths
    split = int(sum(p for p in partitions_per_seq if p > 1)) * H * (D + 2) * 4 * 2  # partials w+r
    append = 2 * 2 * B * Hkv * D * elt + B * 8                     # k/v read + written, slots
    return {"kv": kv, "decode": kv + qo + tables + split, "append": append,
            "step": kv + qo + tables + split + append}


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every 10 ms."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int):
        self.samples = []
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - reported in the JSON
            self.err = repr(e)
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        p = self.nvml
        while not self._stop.is_set():
            try:
                mhz = p.nvmlDeviceGetClockInfo(self.h, p.NVML_CLOCK_SM)
                rs = p.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.01)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self, t0, t1, timed=None):
        """Clocks over the window [t0, t1] (the timed region plus the loops
        measured right after it on the same data); `timed` = (start, end) of
        the timed region itself, whose own sample count is reported too."""
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        note = ("sampled every 10 ms from the start of the timed region to the end of the "
                "comparison and end-to-end loops that follow it")
        if not inside:
            inside = self.samples[-5:]
            note = "window shorter than the sampling period: last samples before its end"
        reasons = set()
        for _, _, rs in inside:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        out = {"sm_mhz": statistics.median(m for _, m, _ in inside) if inside else None,
               "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
               "samples": len(inside), "window_s": t1 - t0, "note": note}
        if timed is not None:
            tin = [s for s in self.samples if timed[0] <= s[0] <= timed[1]]
            out["timed_region_samples"] = len(tin)
            if tin:
                out["timed_region_sm_mhz"] = statistics.median(m for _, m, _ in tin)
        return out


DECODE_KERNEL_SOURCES = ("common.cuh", "decode_common.cuh", "decode_staged.cuh", "ptx.cuh")


PREFILL_KERNEL_SOURCES = ("common.cuh", "ptx.cuh", "tcgen05.cuh", "decode_common.cuh", "decode_staged.cuh",
                          "prefill_common.cuh", "prefill_tc.cuh")


def kernel_source_digest(sources=None):
    """Digest of the sources a kernel is compiled from (default: the staged
    decode kernel's)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_400_b200", "csrc", "device")
    for n in (sources or DECODE_KERNEL_SOURCES):
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(n.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(path=None, sources=None):
    """ncu DRAM bytes per launch recorded in profiles/<kernel>_<workload>.json
    (beside the summary of the same capture), if taken on this source."""
    try:
        with open(path or TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None, "no ncu record"
    if "kernel_source_digest" not in rec or "dram_bytes_per_launch" not in rec:
        return None, "record lacks digest or traffic"
    if rec["kernel_source_digest"] != kernel_source_digest(sources):
        return None, "kernel changed since the ncu capture"
    return int(rec["dram_bytes_per_launch"]), "ncu capture (%s)" % rec.get("captured", "?")


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_sample(case, seconds, rng_seed=0):
    """Times the oracle (as it stands) on whole sequences of the batch, one at a
    time in random order, for about `seconds` of oracle work: its copy-on-write
    copies, cache append and fp64 attention. Input generation (the generator's
    pool blocks, q, k, v) and the oracle block-manager replay are outside the
    timed part. Returns (sequences done, oracle seconds)."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle_side import oracle_compute, oracle_indices, oracle_inputs
    ost = oracle_indices(case)
    order = np.random.default_rng(rng_seed).permutation(len(case.batch))
    done, busy = 0, 0.0
    while done < len(order) and busy < seconds:
        x = oracle_inputs(case, ost, [int(order[done])])
        t0 = time.perf_counter()
        oracle_compute(x)
        busy += time.perf_counter() - t0
        done += 1
    return done, busy


def run_reference(args, rank, world):
    from paged_kv_cache_400_b200 import workloads as wl
    if rank != 0:
        return
    case = wl.gqa_case(args.seed)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle_side import oracle_compute, oracle_indices, oracle_inputs
    ost = oracle_indices(case)
    rng = np.random.default_rng(1)
    per_step = 2  # sequences per step: a bounded sample of the batch
    times = []
    for i in range(args.warmup + args.steps):
        rows = [int(x) for x in rng.choice(len(case.batch), size=per_step, replace=False)]
        x = oracle_inputs(case, ost, rows)
        t0 = time.perf_counter()
        oracle_compute(x)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = per_step * len(times) / total
    cfg = workload_description(case, ost.lens)
    cfg["global_batch"] = per_step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{per_step} random sequences of the batch per step (their KV "
                                   "gathered through the oracle block manager's tables), fp64"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def timed_loop(K, stream, phases):
    """Runs K steps; each step runs the callables of `phases` in order, with a
    CUDA event between phases. Returns (total ms, per-phase ms lists)."""
    import torch
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(phases) + 1)] for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(K):
        ev[i][0].record(stream)
        for j, fn in enumerate(phases):
            fn()
            ev[i][j + 1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    per = [[e[j].elapsed_time(e[j + 1]) for e in ev] for j in range(len(phases))]
    return t0.elapsed_time(t1), per


def packed_buffers(templates, dev):
    """One pinned host buffer and one device buffer laid out alike, holding
    tensors of the templates' shapes and dtypes at 256-byte aligned offsets, so
    that a step's inputs cross to the device in one copy. Returns (host,
    device, host views, device views); the host views start as copies of the
    templates."""
    import torch
    offs, n = [], 0
    for t in templates:
        offs.append(n)
        n += (t.numel() * t.element_size() + 255) // 256 * 256
    host = torch.empty(n, dtype=torch.uint8).pin_memory()
    devb = torch.empty(n, dtype=torch.uint8, device=dev)
    hv, dv = [], []
    for t, o in zip(templates, offs):
        nb = t.numel() * t.element_size()
        hv.append(host[o:o + nb].view(t.dtype).view(t.shape))
        dv.append(devb[o:o + nb].view(t.dtype).view(t.shape))
    for h, t in zip(hv, templates):
        h.copy_(t)
    return host, devb, hv, dv


def run_ours(args, rank, world, dist):
    import torch

    import paged_kv_cache_400_b200 as pk
    from paged_kv_cache_400_b200.scenario import prepare_decode_step

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    case = rank_case(args.seed, rank, args.batch, args.workload)
    prep = prepare_decode_step(case)
    B, H, D = len(case.batch), case.num_heads, case.head_dim
    pool = case.make_pool(dev)
    q = case.make_q(dev)
    k, v = case.make_kv_new(dev)
    slots = torch.from_numpy(prep.slot_mapping).to(dev)
    bt = torch.from_numpy(prep.block_tables).to(dev)
    sl = torch.from_numpy(prep.seq_lens).to(dev)
    out = torch.empty_like(q)
    ws = pk.alloc_workspace(B, H, pool, case.max_seq_len)
    S = pk.pa_decode_partition_tokens(B, H, pool, case.max_seq_len)
    parts = [(int(n) + S - 1) // S for n in prep.seq_lens]
    max_parts = (case.max_seq_len + S - 1) // S   # partitions the launch is sized for
    nbytes = algorithmic_bytes(case, prep, parts, max(parts))
    stream = torch.cuda.current_stream()
    cow_src = torch.from_numpy(prep.cow_src).to(dev) if len(prep.cow_src) else None
    cow_dst = torch.from_numpy(prep.cow_dst).to(dev) if len(prep.cow_dst) else None

    def cow():
        # the step's copy-on-write copies (shared-prefix workload) come first
        if cow_src is not None:
            pk.pa_copy_blocks(pool, cow_src, cow_dst)

    def append_decode():   # the step as one call: append folded into decode
        pk.pa_append_decode(out, q, k, v, pool, slots, bt, sl, case.scale, case.max_seq_len, ws)

    def append():
        pk.pa_reshape_and_cache(k, v, pool, slots)

    def decode():
        pk.pa_decode(out, q, pool, bt, sl, case.scale, case.max_seq_len, ws)

    for _ in range(max(args.warmup, 3)):
        cow()
        append_decode()
        cow()
        append()
        decode()
    assert pk.pa_get_device_error() == 0

    K = args.steps
    sampler = ClockSampler(local)
    sampler.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    total_ms, (cow_ms, step_ms) = timed_loop(K, stream, [cow, append_decode])
    wall1 = time.perf_counter()
    if dist is not None:
        dist.barrier()
    # the same step as separate calls, for comparison
    total_sep, (_, app_ms, dec_ms) = timed_loop(K, stream, [cow, append, decode])
    assert pk.pa_get_device_error() == 0

    total_ms = max_over_ranks(total_ms, dist, dev)
    total_sep = max_over_ranks(total_sep, dist, dev)
    ms_per_step = total_ms / K
    value = world * B / (ms_per_step / 1e3)

    # ---- e2e: host buffers through the public API, copies inside the region
    E = args.e2e_steps or min(K, 100)
    pin = lambda t: t.cpu().pin_memory()
    h_q, h_k, h_v = pin(q), pin(k), pin(v)
    h_slots = pin(slots)
    h_bt, h_sl = pin(bt), pin(sl)
    h_out = torch.empty_like(out, device="cpu").pin_memory()
    bt_np, sl_np = h_bt.numpy(), h_sl.numpy()
    batch = np.asarray(case.batch, np.int64)
    h2d = sum(t.numel() * t.element_size() for t in (h_q, h_k, h_v, h_slots, h_bt, h_sl))
    d2h = h_out.numel() * h_out.element_size()
    for i in range(3 + E):
        if i == 3:
            if dist is not None:
                dist.barrier()
            torch.cuda.synchronize()
            e0 = time.perf_counter()
        prep.bm.pack(batch, case.table_width, bt_np, sl_np, None)   # host tables (C ABI)
        q.copy_(h_q, non_blocking=True)
        k.copy_(h_k, non_blocking=True)
        v.copy_(h_v, non_blocking=True)
        slots.copy_(h_slots, non_blocking=True)
        bt.copy_(h_bt, non_blocking=True)
        sl.copy_(h_sl, non_blocking=True)
        cow()
        append_decode()
        h_out.copy_(out, non_blocking=True)
        stream.synchronize()
    e1 = time.perf_counter()
    e2e_serial_s = max_over_ranks((e1 - e0) / E, dist, dev)

    # ---- e2e, pipelined: the same per-step work (host table packing, H2D of
    # every input, the step, D2H of its output), with later steps' uploads and
    # earlier steps' downloads on copy streams while step i computes (NB
    # buffer sets; a set is reused only after the step NB back has released
    # it, so the host runs up to NB - 1 steps ahead of the device). A set's
    # inputs sit in one pinned buffer and cross in one copy.
    NB = 3
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    sets = [packed_buffers((h_q, h_k, h_v, h_slots, h_bt, h_sl), dev) for _ in range(NB)]
    tables_np = [(hv[4].numpy(), hv[5].numpy()) for _, _, hv, _ in sets]
    h2d_packed = sets[0][0].numel()
    douts = [out] + [torch.empty_like(out) for _ in range(NB - 1)]
    houts = [h_out] + [torch.empty_like(out, device="cpu").pin_memory() for _ in range(NB - 1)]
    hout_bits = [h.view(torch.int16).numpy() for h in houts]
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev() for _ in range(NB)], [ev() for _ in range(NB)], [ev() for _ in range(NB)]
    checksum = 0
    W0 = NB + 1  # untimed steps: the pipeline is full when the timer starts
    for i in range(W0 + E):
        b = i % NB
        host_in, dev_in, _, (dq, dk, dv, dslots, dbt, dsl) = sets[b]
        if i == W0:
            torch.cuda.synchronize()
            if dist is not None:
                dist.barrier()
            p0 = time.perf_counter()
        if i >= NB:
            in_done[b].synchronize()      # inputs of step i-NB uploaded: host buffer free
            out_done[b].synchronize()     # result of step i-NB is on the host
            checksum += int(hout_bits[b][0, 0, 0])
        prep.bm.pack(batch, case.table_width, tables_np[b][0], tables_np[b][1], None)
        with torch.cuda.stream(s_in):
            if i >= NB:
                s_in.wait_event(comp_done[b])   # step i-NB no longer reads device buffers b
            dev_in.copy_(host_in, non_blocking=True)
            in_done[b].record(s_in)
        stream.wait_event(in_done[b])
        if i >= NB:
            stream.wait_event(out_done[b])      # step i-NB's output was downloaded
        cow()
        pk.pa_append_decode(douts[b], dq, dk, dv, pool, dslots, dbt, dsl, case.scale, case.max_seq_len, ws)
        comp_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            houts[b].copy_(douts[b], non_blocking=True)
            out_done[b].record(s_out)
    torch.cuda.synchronize()
    p1 = time.perf_counter()
    sampler.stop()
    e2e_s = max_over_ranks((p1 - p0) / E, dist, dev)
    assert pk.pa_get_device_error() == 0

    # the prefill legs (the step on the other side of decode): chunked prefill
    # and whole prompts, every rank
    prefill_line = prompts_line = None
    if args.workload == "gqa" and not args.no_prefill_leg:
        prefill_line = measure_prefill(args, rank, world, dist, True, max(K, 10), args.warmup,
                                       None if args.no_cpu_baseline else args.prefill_cpu_seconds)
        prompts_line = measure_prefill(args, rank, world, dist, False, max(K, 10), args.warmup,
                                       None if args.no_cpu_baseline else args.prefill_cpu_seconds)

    if rank != 0:
        return
    peak, peak_src = measured_peak()
    step_avg = sum(step_ms) / K
    fused_bytes = nbytes["decode"] + nbytes["append"]
    achieved = fused_bytes / (step_avg / 1e3) / 1e9
    # the ncu record is of the batch-256 GQA launch (seed 0); other decode
    # workloads carry none
    if args.workload == "gqa" and args.batch == 256 and args.seed + rank == 0:
        traffic, traffic_src = recorded_traffic()
    else:
        traffic, traffic_src = None, "captured for the batch-256 GQA workload only"
    kv_gbs = nbytes["kv"] / (ms_per_step / 1e3) / 1e9
    cfg = workload_description(case, prep.seq_lens)
    cfg["global_batch"] = B * world
    cfg["parallelism"] = f"dp{world} independent replicas (no exchange step)"
    cfg["partition_tokens"] = S
    cfg["step"] = ("pa_append_decode (cache append folded into the split-KV decode kernel)"
                   + (" after pa_copy_blocks" if cow_src is not None else ""))
    dec_avg = sum(dec_ms) / K
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": cfg,
        "tokens_per_s_32_layer_equiv": value / 32,
        "kv_read_gbs": kv_gbs, "kv_frac_of_8tbs": kv_gbs / NOMINAL_HBM_GBS,
        "kv_frac_of_measured": kv_gbs / peak,
        "roofline": {"kernel": "decode_staged_kernel with fused append (pa_append_decode; partition "
                               "reduce launch included)",
                     "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_src,
                     "traffic": traffic, "traffic_source": traffic_src,
                     "algorithmic_bytes_per_launch": fused_bytes, "avg_launch_ms": step_avg},
        "separate_calls": {"ms_per_step": total_sep / K, "append_avg_ms": sum(app_ms) / K,
                           "decode_avg_ms": dec_avg,
                           "decode_frac_of_measured": nbytes["decode"] / (dec_avg / 1e3) / 1e9 / peak,
                           "value": world * B / (total_sep / K / 1e3)},
        # per step: the decode kernel, the partition merge when the bound
        # allows several partitions, the plan kernel from 4 partitions on (the
        # work-list path), and the copy-on-write copy when there are pairs
        "gpu_launches": K * (1 + (1 if max_parts > 1 else 0) + (1 if max_parts >= 4 else 0)
                             + (1 if cow_src is not None else 0)),
        "clocks": sampler.summary(wall0, p1, timed=(wall0, wall1)),
        "e2e": {"value": world * B / e2e_s, "unit": "tokens/s", "h2d_bytes_per_step": h2d_packed,
                "d2h_bytes_per_step": d2h,
                "note": "per step: host table packing (pa_bm_pack) into a pinned buffer holding all of "
                        "the step's inputs (q/k/v/slots/tables/lens, 256-byte aligned), one H2D copy of "
                        "it, pa_append_decode, D2H of out; uploads and downloads on copy streams "
                        "overlapping the neighbouring steps' compute (three buffer sets: the host packs "
                        "and uploads up to two steps ahead)"},
        "e2e_serial": {"value": world * B / e2e_serial_s, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                       "note": "the same per-step work with each input copied separately and a stream "
                               "sync after every step"},
        "library": os.path.relpath(pk.library_path(), ROOT),
    }
    if case.name == "shared_prefix":
        uniq = len({int(x) for row, n in zip(prep.block_tables, prep.seq_lens)
                    for x in row[:(int(n) + 15) // 16]})
        ub = uniq * 2 * case.num_kv_heads * 16 * D * 2
        line["unique_kv_bytes"] = ub
        line["unique_kv_gbs"] = ub / (ms_per_step / 1e3) / 1e9
    if prefill_line is not None:
        line["chunked_prefill"] = prefill_line
    if prompts_line is not None:
        line["prompts_prefill"] = prompts_line
    if not args.no_cpu_baseline and world == 1:
        done, el = oracle_sample(case, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": done / el, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{done} of {B} sequences (random order), one decode token each: oracle "
                      f"copy-on-write + append + gather through its own block tables + fp64 "
                      f"attention, {el:.1f} s of oracle time"}
        try:
            from threadpoolctl import threadpool_limits
            with threadpool_limits(1):
                d1, e1 = oracle_sample(case, args.cpu_seconds / 3, rng_seed=1)
            line["cpu_baseline"]["one_core_value"] = d1 / e1
        except Exception as e:  # pragma: no cover
            line["cpu_baseline"]["one_core_value"] = None
            line["cpu_baseline"]["one_core_error"] = repr(e)
    print(json.dumps(line), flush=True)


def trace_oracle_scheduler(tr, caching, swap_host_blocks):
    """The oracle scheduler over the trace's requests, configured as the run."""
    sys.path.insert(0, ROOT)
    from oracle.block_manager import OracleBlockManager
    from oracle.scheduler import OracleScheduler
    bm = OracleBlockManager(tr.num_blocks)
    if caching:
        bm.set_prefix_caching(True)
    sch = OracleScheduler(bm, tr.arrival_step, tr.prompt_len, tr.output_len, tr.table_width)
    if caching:
        sch.set_prompt_tokens(tr.prompt_tokens)
    if swap_host_blocks:
        sch.set_swap(swap_host_blocks)
    return sch


def trace_oracle_plan(tr, caching, swap_host_blocks, n_samples, rows_per_sample, seed):
    """The oracle's side of the trace measurement. Replays the whole trace on
    the oracle scheduler (timed: the integer half of the oracle, in full), then
    picks `n_samples` seeded (step, layer) samples and, per sample, up to
    `rows_per_sample` running requests, and replays once more (untimed) to keep
    those steps' requests, lengths and block tables. Returns (replay seconds,
    steps, {step: (layer, [(row, request, length, table)])})."""
    t0 = time.perf_counter()
    sch = trace_oracle_scheduler(tr, caching, swap_host_blocks)
    running = []
    while True:
        o = sch.step()
        running.append(len(o["running"]))
        if o["done"]:
            break
    replay_s = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    busy = [i for i, n in enumerate(running) if n > 0]
    steps = sorted(int(x) for x in rng.choice(busy, size=min(n_samples, len(busy)), replace=False))
    plan = {st: int(rng.integers(tr.num_layers)) for st in steps}
    picks = {}
    sch = trace_oracle_scheduler(tr, caching, swap_host_blocks)
    while True:
        o = sch.step()
        st = o["step"]
        if st in plan:
            n = len(o["running"])
            rows = sorted(int(x) for x in rng.choice(n, size=min(rows_per_sample, n), replace=False))
            picks[st] = (plan[st], [(i, o["running"][i], o["seq_lens"][i],
                                     o["block_tables"][i][:(o["seq_lens"][i] + 15) // 16]) for i in rows])
        if o["done"]:
            break
    return replay_s, len(running), picks


def run_trace(args, rank, world):
    """The 2000-request arrival trace through the C++ scheduler and the kernels:
    per step, pa_sched_step, then for each of the layers the prompt append, the
    decode-token append and paged decode. Inputs (the synthetic stand-in for the
    model's K/V/Q projections) are generated on the device before each step's
    layer loop and are outside every timed region. Reports generated tokens per
    second of device time of the layer loops, and end to end (scheduler + index
    copies + layer loops, wall clock, excluding input generation)."""
    import torch

    import paged_kv_cache_400_b200 as pk
    from paged_kv_cache_400_b200 import workloads as wl
    from paged_kv_cache_400_b200.engine import DecodeEngine

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    shared = args.workload == "prefix_trace"
    if shared:
        tr = wl.prefix_trace_case(args.seed + rank, n_requests=args.trace_requests,
                                  num_layers=args.trace_layers)
    else:
        tr = wl.trace_case(args.seed + rank, n_requests=args.trace_requests, num_layers=args.trace_layers)
    caching = shared and not args.no_prefix_cache
    eng = DecodeEngine(tr.num_blocks, tr.num_layers, tr.num_heads, tr.num_kv_heads, tr.head_dim,
                       tr.arrival_step, tr.prompt_len, tr.output_len, tr.table_width, tr.scale, dev,
                       prompt_tokens=tr.prompt_tokens if caching else None,
                       swap_host_blocks=args.swap_host_blocks)
    graphed = None
    if args.graphs:
        from paged_kv_cache_400_b200.engine import GraphedLayers
        graphed = GraphedLayers(eng, max_batch=1280)
    stream = torch.cuda.current_stream()
    # the oracle's half: full scheduler replay (timed) and the sampled steps
    oracle_on = not args.no_cpu_baseline and world == 1
    if oracle_on:
        replay_s, oracle_steps, picks = trace_oracle_plan(tr, caching, args.swap_host_blocks, 20, 2,
                                                          args.seed + 17)
    else:
        picks = {}
    got_rows = {}
    util_log = open(args.kv_util_jsonl, "w") if args.kv_util_jsonl else None
    utils, occupancy = [], []
    slots_held = 0
    events = []
    tokens = kv_tokens = prompt_tokens = steps = preempted = cached_tokens = peak_batch = 0
    swap_blocks = 0
    host_s = e2e_s = 0.0
    sampler = ClockSampler(local)
    sampler.start()
    wall0 = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        idx = eng.schedule()
        t1 = time.perf_counter()
        host_s += t1 - t0
        n = len(idx.running)
        if n:
            reqs_p, pos_p = eng.prompt_positions(idx)
            inputs, stacked = tr.step_inputs(idx.step, idx.running, idx.seq_lens, reqs_p, pos_p, dev,
                                             stacked=True, prefill=args.prefill)
            if graphed is not None:
                graphed._graph(((n + graphed.bucket - 1) // graphed.bucket) * graphed.bucket)
            torch.cuda.synchronize()
            t2 = time.perf_counter()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            if graphed is not None:
                outs = graphed.run(idx, inputs, stacked)
            else:
                outs = eng.run_layers(idx, inputs)
            e1.record(stream)
            torch.cuda.synchronize()
            e2e_s += (t1 - t0) + (time.perf_counter() - t2)
            events.append((e0, e1))
            if idx.step in picks:
                layer, rows = picks[idx.step]
                got_rows[idx.step] = outs[layer][[r for r, _, _, _ in rows]].float().cpu().numpy()
            tokens += n
            lens_sum = int(idx.seq_lens.astype(np.int64).sum())
            kv_tokens += lens_sum
            prompt_tokens += len(idx.prompt_slots)
            # KV-cache utilisation: token slots holding a running request's KV
            # over the slots of the distinct blocks those requests hold
            held = np.unique(idx.block_tables[idx.block_tables >= 0])
            util = lens_sum / (16.0 * len(held))
            occ = (tr.num_blocks - idx.record.num_free_blocks) / tr.num_blocks
            utils.append(util)
            occupancy.append(occ)
            slots_held += 16 * len(held)
            if util_log is not None:
                util_log.write(json.dumps({"step": int(idx.step), "running": n, "kv_tokens": lens_sum,
                                           "blocks_held": int(len(held)), "kv_util": util,
                                           "pool_occupancy": occ}) + "\n")
        steps += 1
        preempted += idx.record.preempted
        cached_tokens += int(idx.prompt_starts.sum())
        swap_blocks += len(idx.swap_out) + len(idx.swap_in)
        peak_batch = max(peak_batch, n)
        if idx.done:
            break
    wall1 = time.perf_counter()
    sampler.stop()
    if util_log is not None:
        util_log.close()
    assert pk.pa_get_device_error() == 0
    gpu_s = sum(a.elapsed_time(b) for a, b in events) / 1e3
    eng.close()
    kv_bytes = kv_tokens * 2 * tr.num_kv_heads * tr.head_dim * 2 * tr.num_layers
    prompts = ("8 shared system prompts U[256,1024] + user tokens U[16,512]" if shared
               else "prompts U[16,1024]")
    line = {
        "graphs": bool(args.graphs),
        "prefill_attention": bool(args.prefill),
        "prefix_caching": caching,
        "workload": f"continuous-batching trace: {args.trace_requests} requests, Poisson(50) arrivals/step, "
                    f"{prompts}, outputs geometric mean 200 cap 2048, 40000-block pools, "
                    f"{tr.num_layers} layers x (prompt append + "
                    + ("causal prefill attention of the new prompt positions + " if args.prefill else "")
                    + "decode-token append + paged decode), "
                    "32/8 heads, head_dim 128, bf16",
        "prompt_tokens_cached": cached_tokens, "peak_batch": peak_batch,
        "swap_host_blocks": args.swap_host_blocks,
        "swap_bytes": swap_blocks * 2 * tr.num_kv_heads * 16 * tr.head_dim * 2 * tr.num_layers,
        "metric": "generated tokens/s (device time of the layer loops)", "value": tokens / gpu_s,
        "unit": "tokens/s", "steps": steps, "generated_tokens": tokens, "prompt_tokens_written": prompt_tokens,
        "preemptions": preempted, "gpu_s": gpu_s, "host_scheduler_s": host_s,
        "kv_read_tb": kv_bytes / 1e12, "kv_read_gbs": kv_bytes / gpu_s / 1e9,
        "kv_read_note": ("logical bytes: blocks shared by many sequences are read through L2"
                         if caching else "every sequence's own blocks"),
        "e2e": {"value": tokens / e2e_s, "unit": "tokens/s",
                "note": "pa_sched_step + index H2D + layer loops, wall clock; input generation excluded"},
        "wall_s": wall1 - wall0, "clocks": sampler.summary(wall0, wall1),
        "kv_util": {"mean": float(np.mean(utils)), "min": float(np.min(utils)),
                    "over_all_steps": kv_tokens / max(1, slots_held),
                    "pool_occupancy_mean": float(np.mean(occupancy)),
                    "definition": "per step: KV tokens of the running requests / (16 x distinct blocks "
                                  "they hold); pool_occupancy = blocks held / pool blocks",
                    "per_step_jsonl": args.kv_util_jsonl},
    }
    if oracle_on:
        # parity and timing of the oracle's attention on the sampled rows
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        from oracle_side import oracle_trace_row
        att_s, att_tokens, max_err, n_rows = 0.0, 0, 0.0, 0
        for st, (layer, rows) in picks.items():
            for j, (_, req, length, table) in enumerate(rows):
                ref, dt = oracle_trace_row(tr, layer, st, req, table, length)
                max_err = max(max_err, float(np.abs(got_rows[st][j] - ref).max()))
                att_s += dt
                att_tokens += length
                n_rows += 1
        assert max_err <= 1e-2, f"trace: sampled decode rows differ from the oracle by {max_err}"
        # oracle time of the whole run: the replay (measured in full) plus the
        # attention of every (step, layer, request), extrapolated from the
        # sampled rows by their KV tokens
        att_total = att_s / att_tokens * (kv_tokens * tr.num_layers)
        line["parity"] = {"sampled_steps": len(picks), "rows": n_rows, "max_abs_err": max_err, "bar": 1e-2,
                          "oracle": "fp64 append + gather through the oracle scheduler's own tables"}
        line["cpu_baseline"] = {
            "value": tokens / (replay_s + att_total), "unit": "tokens/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"oracle scheduler replay of the whole trace timed in full ({replay_s:.2f} s, "
                      f"{oracle_steps} steps); fp64 attention timed on {n_rows} rows of {len(picks)} seeded "
                      f"(step, layer) samples ({att_s:.2f} s for {att_tokens} KV tokens) and extrapolated "
                      f"by KV tokens to every request of every step and layer ({att_total:.0f} s)",
            "replay_s": replay_s, "attention_s_extrapolated": att_total}
    print(json.dumps(line), flush=True)


def prefill_flops(case):
    """Algorithmic FLOPs of causal prefill attention: a new token at position p
    scores p + 1 keys and sums p + 1 values, 2 x 128 FLOPs each, per query head."""
    f = 0
    for c, n in zip(case.ctx_lens, case.query_lens):
        # sum over p = c .. c+n-1 of (p + 1)
        f += n * c + n * (n + 1) // 2
    return 4 * case.head_dim * case.num_heads * f


def measured_tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
    except Exception:
        return 1590.0, "fallback 1.59 PFLOP/s"


def oracle_prefill_sample(case, seconds, rng_seed=0):
    """The oracle (as it stands) on whole sequences of the step in random
    order, for about `seconds`: append of the new tokens' K/V, then causal fp64
    attention. Input generation is outside the timed part. Returns (new tokens
    done, sequences done, oracle seconds)."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle_side import oracle_prefill_compute, oracle_prefill_indices, oracle_prefill_inputs
    ost = oracle_prefill_indices(case)
    order = np.random.default_rng(rng_seed).permutation(len(case.query_lens))
    toks = done = 0
    busy = 0.0
    while done < len(order) and busy < seconds:
        b = int(order[done])
        x = oracle_prefill_inputs(case, ost, [b])
        t0 = time.perf_counter()
        oracle_prefill_compute(x)
        busy += time.perf_counter() - t0
        toks += case.query_lens[b]
        done += 1
    return toks, done, busy


def run_prefill(args, rank, world, dist):
    """The prefill workloads as the benchmark line (see measure_prefill)."""
    line = measure_prefill(args, rank, world, dist, args.workload == "chunked_prefill", args.steps,
                           args.warmup, None if args.no_cpu_baseline else args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)


def measure_prefill(args, rank, world, dist, chunked, K, warmup, cpu_seconds):
    """One prefill step per iteration: append every new token's K/V into its
    slot (pa_reshape_and_cache), then causal paged attention of the new tokens
    (pa_prefill). Returns (on rank 0; None elsewhere) the line: new tokens per
    second, the attention kernel's TFLOP/s against the measured bf16 tensor
    peak, the end-to-end rate from host buffers and, with cpu_seconds, the
    oracle on a bounded sample."""
    import torch

    import paged_kv_cache_400_b200 as pk
    from paged_kv_cache_400_b200 import workloads as wl
    from paged_kv_cache_400_b200.scenario import prepare_prefill_step

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pb = args.prefill_batch
    case = (wl.chunked_prefill_case(args.seed + rank, batch=pb) if chunked
            else wl.prefill_case(args.seed + rank, batch=pb))
    prep = prepare_prefill_step(case)
    T = case.num_tokens
    pool = case.make_pool(dev)
    q = case.make_q(dev)
    k, v = case.make_kv_new(dev)
    slots = torch.from_numpy(prep.slot_mapping).to(dev)
    bt = torch.from_numpy(prep.block_tables).to(dev)
    sl = torch.from_numpy(prep.seq_lens).to(dev)
    qs = torch.from_numpy(prep.query_start).to(dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    mq = case.max_query_len

    def append():
        pk.pa_reshape_and_cache(k, v, pool, slots)

    def attend():
        pk.pa_prefill(out, q, pool, bt, sl, qs, case.scale, mq)

    for _ in range(max(warmup, 3)):
        append()
        attend()
    assert pk.pa_get_device_error() == 0
    sampler = ClockSampler(local)
    sampler.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    total_ms, (app_ms, att_ms) = timed_loop(K, stream, [append, attend])
    wall1 = time.perf_counter()
    if dist is not None:
        dist.barrier()
    assert pk.pa_get_device_error() == 0
    total_ms = max_over_ranks(total_ms, dist, dev)
    ms_per_step = total_ms / K
    value = world * T / (ms_per_step / 1e3)

    E = args.e2e_steps or min(K, 50)
    pin = lambda t: t.cpu().pin_memory()
    hs = [pin(t) for t in (q, k, v, slots, bt, sl, qs)]
    h_out = torch.empty_like(out, device="cpu").pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in hs)
    d2h = h_out.numel() * h_out.element_size()
    for i in range(3 + E):
        if i == 3:
            if dist is not None:
                dist.barrier()
            torch.cuda.synchronize()
            e0 = time.perf_counter()
        for d_, h_ in zip((q, k, v, slots, bt, sl, qs), hs):
            d_.copy_(h_, non_blocking=True)
        append()
        attend()
        h_out.copy_(out, non_blocking=True)
        stream.synchronize()
    e2e_serial_s = max_over_ranks((time.perf_counter() - e0) / E, dist, dev)

    # pipelined: step i+1's uploads and step i-1's download on copy streams
    # while step i computes (two buffer sets: the prefill step is bound by
    # its host copies, not by the host running ahead)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dsets = [(q, k, v, slots, bt, sl, qs), tuple(t.clone() for t in (q, k, v, slots, bt, sl, qs))]
    douts = [out, torch.empty_like(out)]
    houts = [h_out, torch.empty_like(out, device="cpu").pin_memory()]
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    checksum = 0.0
    for i in range(3 + E):
        b = i & 1
        if i == 3:
            torch.cuda.synchronize()
            if dist is not None:
                dist.barrier()
            p0 = time.perf_counter()
        if i >= 2:
            out_done[b].synchronize()
            checksum += float(houts[b][0, 0, 0])
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[b])
            for d_, h_ in zip(dsets[b], hs):
                d_.copy_(h_, non_blocking=True)
            in_done[b].record(s_in)
        stream.wait_event(in_done[b])
        if i >= 2:
            stream.wait_event(out_done[b])
        dq_, dk_, dv_, dslots_, dbt_, dsl_, dqs_ = dsets[b]
        pk.pa_reshape_and_cache(dk_, dv_, pool, dslots_)
        pk.pa_prefill(douts[b], dq_, pool, dbt_, dsl_, dqs_, case.scale, mq)
        comp_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            houts[b].copy_(douts[b], non_blocking=True)
            out_done[b].record(s_out)
    torch.cuda.synchronize()
    wall2 = time.perf_counter()
    sampler.stop()
    e2e_s = max_over_ranks((wall2 - p0) / E, dist, dev)
    assert pk.pa_get_device_error() == 0
    if rank != 0:
        return None
    flops = prefill_flops(case)
    mma_sync = args.prefill_kernel == "mma_sync"
    att_avg = sum(att_ms) / K
    peak, peak_src = measured_tensor_peak()
    achieved = flops / (att_avg / 1e3) / 1e12
    kv_bytes = int(sum(int(c) + int(n) for c, n in zip(case.ctx_lens, case.query_lens))) * 2 * \
        case.num_kv_heads * case.head_dim * 2
    traffic, traffic_src = None, ("mma.sync kernel: not captured" if mma_sync else
                                  "captured at 64 sequences (seed 0) only")
    if args.prefill_kernel == "tcgen05" and pb == 64 and args.seed + rank == 0:
        traffic, traffic_src = recorded_traffic(
            os.path.join(ROOT, "profiles", f"prefill_tc_{'chunked' if chunked else 'prompts'}_b64.json"),
            PREFILL_KERNEL_SOURCES)
    desc = (f"chunked_prefill_gqa: {pb} sequences, cached context U[0,3072] + a 512-token chunk"
            if chunked else f"prefill_gqa: {pb} whole prompts, lengths U[16,1024]")
    line = {
        "metric": "paged prefill new tokens/s (append + causal paged attention)", "value": value,
        "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": desc + "; 32 q / 8 kv heads, head_dim 128, bf16, block_size 16, random "
                                      "placement; step = pa_reshape_and_cache + pa_prefill",
                   "global_batch": len(case.query_lens) * world, "new_tokens": T,
                   "max_query_len": mq, "kv_tokens": int(prep.seq_lens.sum()),
                   "parallelism": f"dp{world} independent replicas (no exchange step)",
                   "l2": "no flush: K/V read %.2f GB per step (> 126 MB L2), q/out %.2f GB"
                         % (kv_bytes / 1e9, 2 * T * case.num_heads * case.head_dim * 2 / 1e9)},
        "roofline": {"kernel": ("prefill_kernel (mma.sync m16n8k16; comparison build)" if mma_sync else
                                "prefill_tc_kernel (tcgen05.mma, accumulators in tensor memory)"),
                     "bound": "tensor", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "peak_source": peak_src,
                     "traffic": traffic, "traffic_source": traffic_src,
                     "algorithmic_kv_bytes": kv_bytes,
                     "algorithmic_flops_per_launch": flops, "avg_launch_ms": att_avg},
        "append_avg_ms": sum(app_ms) / K,
        "gpu_launches": 2 * K,
        "clocks": sampler.summary(wall0, wall2, timed=(wall0, wall1)),
        "e2e": {"value": world * T / e2e_s, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": "per step: H2D of q/k/v/slots/tables/lens/query_start from pinned memory, "
                        "append, prefill, D2H of out; copies on copy streams overlapping the "
                        "neighbouring steps' compute (two buffer sets)"},
        "e2e_serial": {"value": world * T / e2e_serial_s, "unit": "tokens/s",
                       "note": "the same per-step work with a stream sync after every step"},
        "library": os.path.relpath(pk.library_path(), ROOT),
    }
    if cpu_seconds is not None and world == 1:
        toks, done, el = oracle_prefill_sample(case, cpu_seconds)
        line["cpu_baseline"] = {
            "value": toks / el, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{done} of {len(case.query_lens)} sequences ({toks} new tokens, random order): oracle "
                      f"append + fp64 causal attention through its own block tables, {el:.1f} s"}
    return line


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if args.impl == "reference" and rank != 0:
        return  # the CPU oracle runs on rank 0 only
    if world > 1 and args.impl == "ours":
        import datetime

        import torch
        import torch.distributed as dist_mod
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_mod
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.workload in ("trace", "prefix_trace"):
            run_trace(args, rank, world)
        elif args.workload in ("prefill", "chunked_prefill"):
            from paged_kv_cache_400_b200 import binding as bd
            variant = {"tcgen05": None, "mma_sync": "prefill_mma_sync"}[args.prefill_kernel]
            with bd.use_variant(variant):
                run_prefill(args, rank, world, dist)
        else:
            run_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
