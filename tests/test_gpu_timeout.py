"""The timeout path every kernel's waits share: a wait on staged data that
never completes gives up after its limit, sets PA_DEVERR_TIMEOUT and returns,
so the context stays usable. pa_selftest_timeout makes one such wait run out
on a barrier nothing arrives at (a short limit, not the kernels' 2 s); no GPU
fault, trap or hang is involved."""
import pytest
import torch

import paged_kv_cache_400_b200 as pk
from paged_kv_cache_400_b200 import binding as bd
from paged_kv_cache_400_b200 import workloads as wl
from paged_kv_cache_400_b200.scenario import prepare_decode_step

from oracle_side import oracle_indices, oracle_outputs, tolerance_ok

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_a_wait_that_runs_out_sets_the_bit_and_the_context_stays_usable():
    assert pk.pa_get_device_error() == 0
    pk.pa_selftest_timeout(20_000_000)          # 20 ms
    assert pk.pa_get_device_error() == pk.PA_DEVERR_TIMEOUT
    assert pk.pa_get_device_error() == 0        # read and cleared
    # the same context runs a decode step correctly afterwards
    case = wl.tiny_case()
    prep = prepare_decode_step(case)
    pool = case.make_pool(DEV)
    k, v = case.make_kv_new(DEV)
    pk.pa_reshape_and_cache(k, v, pool, torch.from_numpy(prep.slot_mapping).to(DEV))
    q = case.make_q(DEV)
    out = torch.empty_like(q)
    ws = pk.alloc_workspace(len(case.batch), case.num_heads, pool, case.max_seq_len)
    pk.pa_decode(out, q, pool, torch.from_numpy(prep.block_tables).to(DEV),
                 torch.from_numpy(prep.seq_lens).to(DEV), case.scale, case.max_seq_len, ws)
    assert pk.pa_get_device_error() == 0
    ost = oracle_indices(case)
    ok, err = tolerance_ok(case, out.float().cpu().numpy().astype("float64"),
                           oracle_outputs(case, ost, range(len(case.batch))))
    assert ok, err


def test_limit_out_of_range_rejected():
    for bad in (0, 2_000_000_000):
        with pytest.raises(bd.PagedKVError):
            pk.pa_selftest_timeout(bad)
