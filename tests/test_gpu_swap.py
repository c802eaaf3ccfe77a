"""Swap-mode preemption on the GPU: block copies between the device pool and
pinned host memory are bit-exact, memory the GPU cannot address is refused
before any launch, and a trace whose victims are swapped out and back in
matches the fp64 oracle (restored K/V must equal what was written)."""
import numpy as np
import pytest
import torch

import paged_kv_cache_400_b200 as pk
from oracle.block_manager import OracleBlockManager
from oracle.scheduler import OracleScheduler
from paged_kv_cache_400_b200 import workloads as wl
from paged_kv_cache_400_b200.engine import DecodeEngine

from test_gpu_trace import layer_inputs, oracle_attention

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_block_copies_to_host_and_back_are_bit_exact():
    case = wl.custom_case("swap_rt", 41, [100, 700], 256, 32, 8, 128, "bf16", 64, 1024)
    pool = case.make_pool(DEV)
    orig = pool.clone()
    host = torch.empty((64,) + tuple(pool.shape[1:]), dtype=pool.dtype, pin_memory=True)
    src = torch.tensor([3, 200, 17, 255], dtype=torch.int32, device=DEV)
    hst = torch.tensor([0, 63, 5, 6], dtype=torch.int32, device=DEV)
    pk.pa_copy_blocks_between(host, pool, src, hst)
    torch.cuda.synchronize()
    assert torch.equal(host[hst.long().cpu()], orig[src.long()].cpu())
    back = torch.tensor([10, 11, 12, 13], dtype=torch.int32, device=DEV)
    pk.pa_copy_blocks_between(pool, host, hst, back)
    assert pk.pa_get_device_error() == 0
    assert torch.equal(pool[back.long()], orig[src.long()])
    untouched = [b for b in range(256) if b not in (10, 11, 12, 13)]
    assert torch.equal(pool[untouched], orig[untouched])
    # an id past the host pool: skipped and flagged
    pk.pa_copy_blocks_between(pool, host, torch.tensor([64], dtype=torch.int32, device=DEV),
                              torch.tensor([20], dtype=torch.int32, device=DEV))
    assert pk.pa_get_device_error() == pk.PA_DEVERR_BLOCK
    assert torch.equal(pool[20], orig[20])


def test_unaddressable_host_memory_is_refused():
    case = wl.custom_case("swap_bad", 42, [5], 16, 4, 2, 64, "bf16", 4, 64)
    pool = case.make_pool(DEV)
    pageable = torch.empty((4,) + tuple(pool.shape[1:]), dtype=pool.dtype)   # not pinned
    idx = torch.zeros(1, dtype=torch.int32, device=DEV)
    from paged_kv_cache_400_b200 import binding as bd
    with pytest.raises(bd.PagedKVError) as e:
        rc = bd.lib().pa_copy_blocks_between(
            bd.C.c_void_p(pageable.data_ptr()), 4, bd.C.c_void_p(pool.data_ptr()), 16,
            bd.C.c_void_p(idx.data_ptr()), bd.C.c_void_p(idx.data_ptr()), 1, bd.pool_desc(pool), None)
        bd._check("pa_copy_blocks_between", rc)
    assert e.value.status == "INVALID_ARG"
    assert pk.pa_get_device_error() == 0


def test_swap_mode_trace_matches_oracle():
    trace = wl.trace_case(seed=8, n_requests=240, rate=16.0, num_blocks=1800, num_layers=2, output_cap=300)
    eng = DecodeEngine(trace.num_blocks, trace.num_layers, trace.num_heads, trace.num_kv_heads,
                       trace.head_dim, trace.arrival_step, trace.prompt_len, trace.output_len,
                       trace.table_width, trace.scale, DEV, swap_host_blocks=700)
    obm = OracleBlockManager(trace.num_blocks)
    osch = OracleScheduler(obm, trace.arrival_step, trace.prompt_len, trace.output_len, trace.table_width)
    osch.set_swap(700)
    rng = np.random.default_rng(3)
    swapped_in_live = set()
    checked = restored_checked = swaps = 0
    while True:
        idx = eng.schedule()
        o = osch.step()
        assert idx.swap_out.tolist() == [list(x) for x in o["swap_out"]]
        assert idx.swap_in.tolist() == [list(x) for x in o["swap_in"]]
        assert idx.prompt_slots.tolist() == o["prompt_slots"]
        swaps += len(o["swapped_out"])
        swapped_in_live.update(o["swapped_in"])
        if len(idx.running):
            inputs = [layer_inputs(trace, eng, idx, l, DEV) for l in range(trace.num_layers)]
            outs = eng.run_layers(idx, inputs)
            restored = [i for i, r in enumerate(idx.running) if int(r) in swapped_in_live]
            if (restored and restored_checked < 25) or (idx.step % 20 == 0 and checked < 40):
                layer = int(rng.integers(0, trace.num_layers))
                got = outs[layer].float().cpu().numpy()
                rows = restored[:3] if restored else list(rng.choice(len(idx.running),
                                                                     size=min(3, len(idx.running)),
                                                                     replace=False))
                for i in rows:
                    r = int(idx.running[i])
                    ref = oracle_attention(trace, layer, idx.step, r,
                                           o["block_tables"][i][:(o["seq_lens"][i] + 15) // 16],
                                           o["seq_lens"][i])
                    assert float(np.abs(got[i] - ref).max()) <= 1e-2, (idx.step, r)
                    checked += 1
                    restored_checked += r in swapped_in_live
                swapped_in_live -= {int(idx.running[i]) for i in rows}
        if idx.done:
            break
    assert pk.pa_get_device_error() == 0
    assert swaps > 0 and restored_checked >= 5, (swaps, restored_checked)
    eng.close()
