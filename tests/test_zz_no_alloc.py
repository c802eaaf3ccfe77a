"""pa_decode_noalloc: decode for callers that cannot allocate device memory
(for example a plugin whose host engine owns all device memory, or a decode
loop that may not call cudaMalloc/cudaFree between steps because they can
synchronise the device). Its split-KV partial results live in the library's
fixed per-device array instead of a caller workspace.

Checked through the C ABI against pa_decode with a caller workspace, within
the tolerance the parity tests use (bf16: max |diff| <= 1e-2), on two calls in
a row, for shapes that use the partial results (several partitions per
sequence). Collected last so that a failure here leaves every other test run.
"""
import pytest
import torch

import paged_kv_cache_400_b200 as pk
from paged_kv_cache_400_b200 import binding as bd
from paged_kv_cache_400_b200 import workloads as wl
from paged_kv_cache_400_b200.scenario import prepare_decode_step

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 1e-2


def _inputs(case):
    prep = prepare_decode_step(case)
    pool = case.make_pool(DEV)
    k, v = case.make_kv_new(DEV)
    pk.pa_reshape_and_cache(k, v, pool, torch.from_numpy(prep.slot_mapping).to(DEV))
    return (pool, case.make_q(DEV), torch.from_numpy(prep.block_tables).to(DEV),
            torch.from_numpy(prep.seq_lens).to(DEV))


@pytest.mark.parametrize("heads,kv_heads", [(32, 8), (32, 32)])
def test_noalloc_matches_workspace_decode_twice(heads, kv_heads):
    lens = [4096, 3000, 1, 17, 513, 2048, 777, 4000]
    case = wl.custom_case(f"noalloc_{heads}_{kv_heads}", 21, lens, 2048, heads, kv_heads, 128, "bf16",
                          256, 4096)
    pool, q, bt, sl = _inputs(case)
    B = len(lens)
    need = pk.pa_decode_workspace_size(B, heads, pool, case.max_seq_len)
    assert 0 < need <= (32 << 20)  # uses the partial results, within the fixed array
    ref = torch.empty_like(q)
    ws = pk.alloc_workspace(B, heads, pool, case.max_seq_len)
    pk.pa_decode(ref, q, pool, bt, sl, case.scale, case.max_seq_len, ws)
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        bd.pa_decode_noalloc(out, q, pool, bt, sl, case.scale, case.max_seq_len)
        assert pk.pa_get_device_error() == 0
        diff = (out.float() - ref.float()).abs().max().item()
        assert diff <= TOL, diff


def test_noalloc_rejects_shapes_beyond_its_array():
    case = wl.custom_case("noalloc_big", 22, [16] * 4, 64, 32, 8, 128, "bf16", 4, 64)
    pool, q, bt, sl = _inputs(case)
    B, max_len = 1024, 32768   # 1024 sequences of up to 32k tokens: partials beyond 32 MiB
    q_big = torch.empty(B, 32, 128, dtype=torch.bfloat16, device=DEV)
    need = pk.pa_decode_workspace_size(B, 32, pool, max_len)
    assert need > (32 << 20)
    with pytest.raises(bd.PagedKVError) as e:
        bd.pa_decode_noalloc(q_big.clone(), q_big, pool,
                             torch.zeros(B, max_len // 16, dtype=torch.int32, device=DEV),
                             torch.zeros(B, dtype=torch.int32, device=DEV), 0.1, max_len)
    assert e.value.status == "WORKSPACE"
