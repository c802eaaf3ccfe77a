"""The C-ABI library loads and exports every entry point include/pagedkv.h
declares; host-side argument checks reject bad input before any device work
(these calls never reach the GPU, so they run without one)."""
import ctypes as C
import os
import re

import pytest

from paged_kv_cache_400_b200 import binding as bd

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "pagedkv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("pa_reshape_and_cache", "pa_decode", "pa_decode_workspace_size",
                 "pa_copy_blocks", "pa_get_device_error", "pa_bm_create", "pa_sched_step"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = C.CDLL(bd.lib()._name)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert missing == []


def test_status_strings():
    for code in range(10):
        s = bd.lib().pa_status_string(code)
        assert s and s != b"unknown status"


def pool(num_blocks=8, heads=2, dim=128, dtype=bd.PA_BF16, bs=16):
    return bd.pa_pool_desc(num_blocks, heads, dim, bs, dtype)


def test_decode_rejects_bad_arguments_on_host():
    L = bd.lib()
    p = pool()
    vp = C.c_void_p(16)  # never dereferenced: rejected before use
    cases = [
        (pool(dim=96), 2, 1),     # unsupported head_dim
        (pool(bs=32), 2, 1),      # block size must be 16
        (pool(heads=3), 4, 1),    # H not a multiple of Hkv
        (pool(heads=1), 17, 1),   # group of 17
    ]
    for desc, H, want in cases:
        st = L.pa_decode(vp, vp, vp, vp, 4, vp, 1, H, 0.1, desc, None, 0, 16, None)
        assert st in (1, 2), (desc.head_dim, H, st)
    # max_seq_len beyond the table width
    assert L.pa_decode(vp, vp, vp, vp, 1, vp, 1, 2, 0.1, p, None, 0, 17, None) == 1
    # NaN scale
    assert L.pa_decode(vp, vp, vp, vp, 4, vp, 1, 2, float("nan"), p, None, 0, 16, None) == 1
    # long sequences need a workspace
    assert L.pa_decode(vp, vp, vp, vp, 512, vp, 64, 2, 0.1, p, None, 0, 8192, None) == 9
    # misaligned pointers
    odd = C.c_void_p(18)
    assert L.pa_decode(odd, vp, vp, vp, 4, vp, 1, 2, 0.1, p, None, 0, 16, None) == 1
    assert b"aligned" in L.pa_last_error()
    # empty batch is a no-op
    assert L.pa_decode(None, None, None, None, 4, None, 0, 2, 0.1, p, None, 0, 16, None) == 0


def test_decode_rejects_more_partitions_than_a_work_item_holds():
    # the persistent decode keeps a partition index in 16 bits: a bound that
    # needs more than 65535 partitions is refused on the host (status 2),
    # before the workspace is looked at; 65535 itself passes that check
    L = bd.lib()
    vp = C.c_void_p(16)  # never dereferenced: rejected before use
    p = pool(num_blocks=1 << 20, heads=8)
    S = L.pa_decode_partition_tokens(1, 32, p, 140_000_000)
    assert S == 2048
    too_long = 65536 * S - 100
    assert L.pa_decode(vp, vp, vp, vp, too_long // 16 + 1, vp, 1, 32, 0.1, p, None, 0, too_long, None) == 2
    assert b"partitions" in L.pa_last_error()
    assert L.pa_append_decode(vp, vp, vp, vp, vp, vp, vp, too_long // 16 + 1, vp, 1, 32, 0.1, p, None, 0,
                              too_long, None) == 2
    fits = 65535 * S
    # the largest bound that fits: the next check (the missing workspace) answers
    assert L.pa_decode(vp, vp, vp, vp, fits // 16, vp, 1, 32, 0.1, p, None, 0, fits, None) == 9


def test_noalloc_reports_argument_errors_before_its_size_limit():
    """pa_decode_noalloc returns pa_decode's own argument errors even for a
    shape beyond its fixed array; only valid arguments reach the size check."""
    L = bd.lib()
    vp = C.c_void_p(16)  # never dereferenced: rejected before use
    big = pool(num_blocks=1 << 20, heads=8)
    B, width, max_len = 1024, 2048, 32768   # partials far beyond the fixed array
    assert L.pa_decode_workspace_size(B, 32, big, max_len) > (32 << 20)
    call = lambda H, desc=big, mb=width, ml=max_len, scale=0.1: L.pa_decode_noalloc(
        vp, vp, vp, vp, mb, vp, B, H, scale, desc, ml, None)
    assert call(36) == 1                          # num_heads not a multiple of num_kv_heads
    assert call(8 * 32) == 2                      # head group 32
    assert call(32, mb=1024) == 1                 # max_seq_len beyond max_blocks * 16
    assert call(32, scale=float("nan")) == 1
    assert call(32, desc=pool(num_blocks=1 << 20, heads=8, dim=96)) == 2
    assert call(32) == 9                          # valid arguments: the size limit
    assert b"fixed array" in L.pa_last_error()
    assert L.pa_decode_noalloc(None, None, None, None, 4, None, 0, 2, 0.1, pool(), 16, None) == 0


def test_prefill_rejects_bad_arguments_on_host():
    L = bd.lib()
    vp = C.c_void_p(16)  # never dereferenced: rejected before use
    p = pool(heads=8)
    # (out, q, pool, tables, max_blocks, seq_lens, query_start, num_seqs, num_tokens, H, scale, desc, max_q)
    ok_args = (vp, vp, vp, vp, 4, vp, vp, 2, 64, 32, 0.1, p, 40, None)
    def call(**kw):
        a = list(ok_args)
        names = ["out", "q", "kv", "bt", "mb", "sl", "qs", "ns", "nt", "H", "scale", "desc", "mq", "st"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return L.pa_prefill(*a)
    assert call(desc=pool(heads=8, dtype=bd.PA_F32)) == 2     # only bf16
    assert call(desc=pool(heads=8, dim=64)) == 2              # only head_dim 128
    assert call(H=24) == 2                                    # group of 3: not a power of two
    assert call(H=36) == 1                                    # H not a multiple of Hkv
    assert call(H=256) == 2                                   # group of 32
    assert call(mq=65) == 1                                   # longer than the tokens given
    assert call(mq=80, nt=100) == 1                           # beyond max_blocks * 16
    assert call(scale=float("inf")) == 1
    assert call(q=None) == 1
    assert call(out=C.c_void_p(24)) == 1                      # misaligned
    assert call(ns=-1) == 1
    assert call(ns=0) == 0                                    # nothing to do
    assert call(mq=0, nt=0) == 0
    assert call(desc=pool(heads=8, bs=32)) == 2               # block size must be 16


def test_append_and_copy_reject_bad_arguments_on_host():
    L = bd.lib()
    vp = C.c_void_p(16)
    assert L.pa_reshape_and_cache(vp, vp, vp, vp, -1, pool(), None) == 1
    assert L.pa_reshape_and_cache(None, None, None, None, 0, pool(), None) == 0
    assert L.pa_reshape_and_cache(vp, vp, vp, vp, 3, pool(dtype=7), None) == 2
    assert L.pa_copy_blocks(vp, vp, vp, -2, pool(), None) == 1
    assert L.pa_copy_blocks(None, None, None, 0, pool(), None) == 0


def test_workspace_size_is_deterministic_and_zero_for_one_partition():
    p = pool(num_blocks=32768, heads=8)
    assert bd.lib().pa_decode_workspace_size(256, 32, p, 8192) == \
        bd.lib().pa_decode_workspace_size(256, 32, p, 8192) > 0
    S = bd.lib().pa_decode_partition_tokens(256, 32, p, 8192)
    assert S % 16 == 0 and S >= 128
    # a bound within the smallest partition (128 tokens) needs no workspace
    assert bd.lib().pa_decode_workspace_size(4, 2, pool(heads=2), 128) == 0
    assert bd.lib().pa_decode_workspace_size(0, 2, p, 100) == 0


@pytest.mark.parametrize("B,H,Hkv,D,max_len", [
    (256, 32, 8, 128, 8192), (64, 32, 32, 128, 8192), (3, 32, 8, 128, 65536), (7, 12, 3, 64, 20000),
    (1, 32, 8, 128, 131072), (1000, 16, 16, 128, 4096),
])
def test_workspace_covers_every_region_the_kernels_write(B, H, Hkv, D, max_len):
    # the split-KV partial accumulators [B][H][P][D] fp32 and (m, l) pairs
    # [B][H][P][2] fp32, and from 4 partitions on the work list [B][P] int32 and
    # its counters: a workspace of the reported size must hold all of them
    p = pool(num_blocks=4096, heads=Hkv, dim=D)
    S = bd.lib().pa_decode_partition_tokens(B, H, p, max_len)
    assert S % 16 == 0 and 128 <= S <= 2048
    P = (max_len + S - 1) // S
    need = B * H * P * D * 4 + B * H * P * 2 * 4 + (B * P * 4 + 2 * 4 if P >= 4 else 0)
    size = bd.lib().pa_decode_workspace_size(B, H, p, max_len)
    assert (size == 0) == (P <= 1)
    assert size >= need


def test_bm_errors_are_statuses():
    bm = bd.BlockManager(4)
    with pytest.raises(bd.PagedKVError) as e:
        bm.allocate(0, 100)
    assert e.value.status == "NO_BLOCKS" and bm.num_free() == 4
    bm.allocate(0, 10)
    with pytest.raises(bd.PagedKVError) as e:
        bm.allocate(0, 1)
    assert e.value.status == "SEQ_EXISTS"
    with pytest.raises(bd.PagedKVError) as e:
        bm.free(5)
    assert e.value.status == "UNKNOWN_SEQ"
    with pytest.raises(bd.PagedKVError):
        bd.BlockManager(4, [0, 1, 1, 2])
    with pytest.raises(bd.PagedKVError) as e:
        bd._check("pa_bm_create", bd.lib().pa_bm_create(4, 32, None, C.byref(C.c_void_p())))
    assert e.value.status == "UNSUPPORTED"
