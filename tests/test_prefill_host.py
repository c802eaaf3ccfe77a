"""Host side of the prefill step (no GPU): the library block manager's tables
and new-token slots for the prefill workloads are bit-exact with the oracle
block manager's, and the oracle's one-row sampling used at full size agrees
with its whole-step prefill."""
import numpy as np

from paged_kv_cache_400_b200 import workloads as wl
from paged_kv_cache_400_b200.scenario import prepare_prefill_step

from oracle_side import oracle_prefill_all, oracle_prefill_indices, oracle_prefill_rows


def _same(case):
    prep = prepare_prefill_step(case)
    ost = oracle_prefill_indices(case)
    assert prep.slot_mapping.tolist() == ost.slots
    assert prep.seq_lens.tolist() == ost.lens
    for b, tab in enumerate(ost.tables):
        assert prep.block_tables[b, :len(tab)].tolist() == tab
    assert prep.query_start[0] == 0 and prep.query_start[-1] == case.num_tokens
    assert np.all(np.diff(prep.query_start) == np.asarray(case.query_lens))


def test_prefill_indices_bit_exact():
    _same(wl.prefill_case(0))
    _same(wl.chunked_prefill_case(0))
    _same(wl.prefill_custom("c", 1, [0, 5, 16, 33], [7, 64, 1, 0], 32, 8))


def test_row_sampling_matches_whole_step():
    case = wl.prefill_custom("s", 2, [0, 19, 3], [21, 17, 5], 4, 2)
    ost = oracle_prefill_indices(case)
    whole, _ = oracle_prefill_all(case, ost)
    picks = [(b, i) for b in range(3) for i in range(case.query_lens[b])]
    rows = oracle_prefill_rows(case, ost, picks)
    assert np.allclose(rows, whole, rtol=0, atol=1e-12)
