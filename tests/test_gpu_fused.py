"""pa_append_decode (append folded into the decode kernel) against the two
calls it replaces, pa_reshape_and_cache then pa_decode: identical outputs and
identical pools, bit for bit; and against the fp64 oracle."""
import numpy as np
import pytest
import torch

import paged_kv_cache_400_b200 as pk
from paged_kv_cache_400_b200 import workloads as wl
from paged_kv_cache_400_b200.scenario import prepare_decode_step

from oracle_side import oracle_indices, oracle_outputs, tolerance_ok

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_both(case):
    prep = prepare_decode_step(case)
    q = case.make_q(DEV)
    k, v = case.make_kv_new(DEV)
    slots = torch.from_numpy(prep.slot_mapping).to(DEV)
    bt = torch.from_numpy(prep.block_tables).to(DEV)
    sl = torch.from_numpy(prep.seq_lens).to(DEV)
    ws = pk.alloc_workspace(len(case.batch), case.num_heads, bd_pool(case), case.max_seq_len)
    results = []
    for fused in (False, True):
        pool = case.make_pool(DEV)
        if len(prep.cow_src):
            pk.pa_copy_blocks(pool, torch.from_numpy(prep.cow_src).to(DEV),
                              torch.from_numpy(prep.cow_dst).to(DEV))
        out = torch.empty_like(q)
        if fused:
            pk.pa_append_decode(out, q, k, v, pool, slots, bt, sl, case.scale, case.max_seq_len, ws)
        else:
            pk.pa_reshape_and_cache(k, v, pool, slots)
            pk.pa_decode(out, q, pool, bt, sl, case.scale, case.max_seq_len, ws)
        assert pk.pa_get_device_error() == 0
        results.append((out, pool))
    return prep, results


def bd_pool(case):
    return torch.empty((1, 2, case.num_kv_heads, 16, case.head_dim), dtype=wl.TORCH_DTYPE[case.dtype],
                       device=DEV).expand(case.num_blocks, -1, -1, -1, -1)


CASES = {
    "gqa": lambda: wl.custom_case("f_gqa", 31, [1, 15, 16, 17, 300, 511, 512, 513, 2000, 4096], 1024, 32, 8,
                                  128, "bf16", 256, 4096),
    "mha": lambda: wl.custom_case("f_mha", 32, [1, 16, 33, 700, 1500], 512, 32, 32, 128, "bf16", 128, 2048),
    "g16": lambda: wl.custom_case("f_g16", 33, [5, 90, 1000], 256, 16, 1, 128, "bf16", 64, 1024),
    "prefix": lambda: wl.prefix_case(1),
    "tiny_fp32": lambda: wl.tiny_case(3),
}


@pytest.mark.parametrize("name", list(CASES))
def test_fused_equals_two_calls_bitwise(name):
    case = CASES[name]()
    prep, ((o1, p1), (o2, p2)) = run_both(case)
    assert torch.equal(o1.view(torch.int16) if o1.dtype == torch.bfloat16 else o1,
                       o2.view(torch.int16) if o2.dtype == torch.bfloat16 else o2)
    assert torch.equal(p1, p2)
    ost = oracle_indices(case)
    sample = list(range(min(len(case.batch), 12)))
    ref = oracle_outputs(case, ost, sample)
    ok, err = tolerance_ok(case, o2[sample].float().cpu().numpy().astype(np.float64), ref)
    assert ok, err


def test_fused_rejects_a_slot_that_is_not_the_new_position():
    case = CASES["gqa"]()
    prep = prepare_decode_step(case)
    pool = case.make_pool(DEV)
    before = pool.clone()
    q = case.make_q(DEV)
    k, v = case.make_kv_new(DEV)
    slots = prep.slot_mapping.copy()
    slots[3] = slots[4]        # wrong position for sequence 3
    slots[5] = -1              # padding: not appended, not an error
    bt = torch.from_numpy(prep.block_tables).to(DEV)
    sl = torch.from_numpy(prep.seq_lens).to(DEV)
    out = torch.empty_like(q)
    ws = pk.alloc_workspace(len(case.batch), case.num_heads, pool, case.max_seq_len)
    pk.pa_append_decode(out, q, k, v, pool, torch.from_numpy(slots).to(DEV), bt, sl, case.scale,
                        case.max_seq_len, ws)
    assert pk.pa_get_device_error() == pk.PA_DEVERR_SLOT
    s3, s5 = int(prep.slot_mapping[3]), int(prep.slot_mapping[5])
    for s in (s3, s5):
        assert torch.equal(pool[s // 16, :, :, s % 16], before[s // 16, :, :, s % 16])
    s4 = int(prep.slot_mapping[4])
    assert torch.equal(pool[s4 // 16, 0, :, s4 % 16], k[4])
