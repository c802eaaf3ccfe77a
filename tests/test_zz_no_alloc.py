"""pa_decode_noalloc: decode for callers that cannot allocate device memory
(for example a plugin whose host engine owns all device memory, or a decode
loop that may not call cudaMalloc/cudaFree between steps because they can
synchronise the device). Its split-KV partial results live in the library's
fixed per-device array instead of a caller workspace.

Checked through the C ABI against pa_decode with a caller workspace. Both run
the same kernels with the same partition count on the same inputs, so the
outputs must be bit-identical; any difference would mean the shared array
leaked state between calls. Between two calls of one shape, a call of a larger
shape (more partitions per sequence, the work-list path) overwrites the array
with other partial results. One call is also compared with the fp64 oracle.
Collected last so that a failure here leaves every other test run.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_400_b200 as pk
from paged_kv_cache_400_b200 import binding as bd
from paged_kv_cache_400_b200 import workloads as wl
from paged_kv_cache_400_b200.scenario import prepare_decode_step

from oracle_side import oracle_indices, oracle_outputs, tolerance_ok

pytestmark = pytest.mark.gpu
DEV = "cuda"
SCRATCH = 32 << 20   # PA_DECODE_NOALLOC_SCRATCH_BYTES


def _inputs(case):
    prep = prepare_decode_step(case)
    pool = case.make_pool(DEV)
    k, v = case.make_kv_new(DEV)
    pk.pa_reshape_and_cache(k, v, pool, torch.from_numpy(prep.slot_mapping).to(DEV))
    return (pool, case.make_q(DEV), torch.from_numpy(prep.block_tables).to(DEV),
            torch.from_numpy(prep.seq_lens).to(DEV))


def _with_workspace(case, pool, q, bt, sl):
    ref = torch.empty_like(q)
    ws = pk.alloc_workspace(len(case.batch), case.num_heads, pool, case.max_seq_len)
    pk.pa_decode(ref, q, pool, bt, sl, case.scale, case.max_seq_len, ws)
    assert pk.pa_get_device_error() == 0
    return ref


def _noalloc(case, pool, q, bt, sl):
    out = torch.full_like(q, float("nan"))
    bd.pa_decode_noalloc(out, q, pool, bt, sl, case.scale, case.max_seq_len)
    assert pk.pa_get_device_error() == 0
    return out


def _bits(t):
    return t.view(torch.int16)


@pytest.mark.parametrize("heads,kv_heads", [(32, 8), (32, 32)])
def test_noalloc_is_bit_identical_to_workspace_decode(heads, kv_heads):
    lens = [4096, 3000, 1, 17, 513, 2048, 777, 4000]
    small = wl.custom_case(f"noalloc_{heads}_{kv_heads}", 21, lens, 2048, heads, kv_heads, 128, "bf16",
                           256, 4096)
    s_in = _inputs(small)
    assert 0 < pk.pa_decode_workspace_size(len(lens), heads, s_in[0], small.max_seq_len) <= SCRATCH
    ref = _with_workspace(small, *s_in)

    # a larger shape: 48 sequences of up to 16k tokens, 8 partitions each (the
    # persistent work-list path), partial results spread over the array
    rng = np.random.default_rng(5)
    big_lens = [int(x) for x in rng.integers(4096, 16384, size=48, endpoint=True)]
    big = wl.custom_case(f"noalloc_big_{heads}_{kv_heads}", 23, big_lens, 48 * 1024 + 64, heads, kv_heads,
                         128, "bf16", 1024, 16384)
    b_in = _inputs(big)
    need_big = pk.pa_decode_workspace_size(len(big_lens), heads, b_in[0], big.max_seq_len)
    assert pk.pa_decode_workspace_size(len(lens), heads, s_in[0], small.max_seq_len) < need_big <= SCRATCH
    big_ref = _with_workspace(big, *b_in)

    first = _noalloc(small, *s_in)
    assert torch.equal(_bits(first), _bits(ref))
    got_big = _noalloc(big, *b_in)
    assert torch.equal(_bits(got_big), _bits(big_ref))
    second = _noalloc(small, *s_in)
    assert torch.equal(_bits(second), _bits(ref))

    # and one call against the fp64 oracle (the bf16 bar of the parity tests)
    expect = oracle_outputs(small, oracle_indices(small), range(len(lens)))
    ok, err = tolerance_ok(small, second.float().cpu().numpy().astype(np.float64), expect)
    assert ok, err


def test_noalloc_rejects_shapes_beyond_its_array():
    case = wl.custom_case("noalloc_reject", 22, [16] * 4, 64, 32, 8, 128, "bf16", 4, 64)
    pool, q, bt, sl = _inputs(case)
    B, max_len = 1024, 32768   # 1024 sequences of up to 32k tokens: partials beyond 32 MiB
    q_big = torch.empty(B, 32, 128, dtype=torch.bfloat16, device=DEV)
    need = pk.pa_decode_workspace_size(B, 32, pool, max_len)
    assert need > SCRATCH
    with pytest.raises(bd.PagedKVError) as e:
        bd.pa_decode_noalloc(q_big.clone(), q_big, pool,
                             torch.zeros(B, max_len // 16, dtype=torch.int32, device=DEV),
                             torch.zeros(B, dtype=torch.int32, device=DEV), 0.1, max_len)
    assert e.value.status == "WORKSPACE"
