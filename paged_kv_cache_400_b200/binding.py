"""ctypes binding of libpagedkv.so: argument marshalling only.

Every function keeps the name of its C entry point (include/pagedkv.h). Device
calls take torch CUDA tensors, pass their data pointers and the current CUDA
stream, and raise PagedKVError on a non-OK status. No computation happens
here: each step of the path runs in the library's kernels or host C++ code.
If the library cannot be loaded (not built, nvcc missing) every call raises.
"""
from __future__ import annotations

import contextlib
import ctypes as C
import os
import threading

import numpy as np
import torch

from . import build as _build

PA_OK = 0
STATUS_NAMES = {
    0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "NO_BLOCKS",
    5: "UNKNOWN_SEQ", 6: "DEVICE_BOUNDS", 7: "SEQ_EXISTS", 8: "CAPACITY", 9: "WORKSPACE",
}
PA_F32, PA_BF16 = 0, 1
PA_DEVERR_SLOT, PA_DEVERR_BLOCK, PA_DEVERR_SEQLEN, PA_DEVERR_TIMEOUT = 1, 2, 4, 8
BLOCK_SIZE = 16


class PagedKVError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str):
        self.status = STATUS_NAMES.get(status, str(status))
        self.code = status
        super().__init__(f"{fn}: {self.status}: {detail}")


class pa_pool_desc(C.Structure):
    _fields_ = [("num_blocks", C.c_int32), ("num_kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("block_size", C.c_int32), ("dtype", C.c_int32)]


_P64 = C.POINTER(C.c_int64)
_P32 = C.POINTER(C.c_int32)


class pa_step_out(C.Structure):
    _fields_ = [
        ("step", C.c_int32), ("done", C.c_int32), ("num_running", C.c_int32),
        ("max_blocks_per_seq", C.c_int32),
        ("running", _P64), ("seq_lens", _P32), ("block_tables", _P32), ("decode_slots", _P64),
        ("num_prompt_seqs", C.c_int32), ("num_prompt_tokens", C.c_int32),
        ("prompt_seqs", _P64), ("prompt_lens", _P32), ("prompt_slots", _P64),
        ("num_cow", C.c_int32), ("cow_src", _P32), ("cow_dst", _P32),
        ("num_admitted", C.c_int32), ("admitted", _P64),
        ("num_preempted", C.c_int32), ("preempted", _P64),
        ("num_finished", C.c_int32), ("finished", _P64),
        ("num_waiting", C.c_int32), ("num_free_blocks", C.c_int32),
        ("prompt_starts", _P32), ("num_cached_tokens", C.c_int32),
        ("num_swap_out", C.c_int32), ("swap_out_src", _P32), ("swap_out_dst", _P32),
        ("num_swap_in", C.c_int32), ("swap_in_src", _P32), ("swap_in_dst", _P32),
        ("num_swapped_out", C.c_int32), ("swapped_out", _P64),
        ("num_swapped_in", C.c_int32), ("swapped_in", _P64),
    ]


_lib = None
_lock = threading.Lock()


def _declare(lib):
    vp, i32, i64, f32, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_size_t
    sigs = {
        "pa_reshape_and_cache": (i32, [vp, vp, vp, vp, i32, pa_pool_desc, vp]),
        "pa_decode_workspace_size": (sz, [i32, i32, pa_pool_desc, i32]),
        "pa_decode_partition_tokens": (i32, [i32, i32, pa_pool_desc, i32]),
        "pa_decode": (i32, [vp, vp, vp, vp, i32, vp, i32, i32, f32, pa_pool_desc, vp, sz, i32, vp]),
        "pa_copy_blocks": (i32, [vp, vp, vp, i32, pa_pool_desc, vp]),
        "pa_append_decode": (i32, [vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32, f32, pa_pool_desc, vp, sz,
                                   i32, vp]),
        "pa_get_device_error": (i32, [C.POINTER(C.c_uint32), vp]),
        "pa_selftest_timeout": (i32, [C.c_uint64, vp]),
        "pa_status_string": (C.c_char_p, [i32]),
        "pa_last_error": (C.c_char_p, []),
        "pa_bm_create": (i32, [i32, i32, _P32, C.POINTER(vp)]),
        "pa_bm_destroy": (None, [vp]),
        "pa_bm_allocate": (i32, [vp, i64, i32]),
        "pa_bm_append_slot": (i32, [vp, i64, _P64, _P32, _P32]),
        "pa_bm_fork": (i32, [vp, i64, i64]),
        "pa_bm_free": (i32, [vp, i64]),
        "pa_bm_num_free": (i32, [vp]),
        "pa_bm_num_blocks": (i32, [vp]),
        "pa_bm_seq_len": (i32, [vp, i64, _P32]),
        "pa_bm_refcount": (i32, [vp, i32, _P32]),
        "pa_bm_block_table": (i32, [vp, i64, _P32, i32, _P32]),
        "pa_bm_free_list": (i32, [vp, _P32, i32, _P32]),
        "pa_bm_slots": (i32, [vp, i64, i32, i32, _P64]),
        "pa_bm_pack": (i32, [vp, _P64, i32, i32, _P32, _P32, _P64]),
        "pa_sched_create": (i32, [vp, _P32, _P32, _P32, i32, i32, C.POINTER(vp)]),
        "pa_sched_step": (i32, [vp, C.POINTER(pa_step_out)]),
        "pa_sched_destroy": (None, [vp]),
        "pa_sched_set_prompt_tokens": (i32, [vp, _P32, _P64]),
        "pa_sched_set_swap": (i32, [vp, i32]),
        "pa_copy_blocks_between": (i32, [vp, i32, vp, i32, vp, vp, i32, pa_pool_desc, vp]),
        "pa_bm_set_prefix_caching": (i32, [vp, i32]),
        "pa_bm_allocate_prefix": (i32, [vp, i64, _P32, i32, i32, _P32]),
        "pa_bm_mark_written": (i32, [vp, i64]),
        "pa_bm_evictable_list": (i32, [vp, _P32, i32, _P32]),
        "pa_bm_num_cached": (i32, [vp]),
        "pa_prefill": (i32, [vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, f32, pa_pool_desc, i32, vp]),
        "pa_decode_noalloc": (i32, [vp, vp, vp, vp, i32, vp, i32, i32, f32, pa_pool_desc, i32, vp]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_variant = None       # name of the comparison build in use, None for the product library
_variant_libs = {}


def lib():
    """The loaded library (built first if missing or stale): the product
    library, or the comparison build selected by use_variant()."""
    global _lib
    if _variant is not None:
        return _variant_libs[_variant]
    if _lib is None:
        with _lock:
            if _lib is None:
                path = _build.build()
                _lib = _declare(C.CDLL(path))
    return _lib


@contextlib.contextmanager
def use_variant(name):
    """Routes every call of this module to a comparison build of the library
    (build.VARIANTS, e.g. "prefill_mma_sync") until the block exits; None keeps
    the product library. For comparisons and their tests only; not
    thread-safe."""
    global _variant
    if name is not None and name not in _variant_libs:
        with _lock:
            if name not in _variant_libs:
                _variant_libs[name] = _declare(C.CDLL(_build.build(variant=name)))
    prev = _variant
    _variant = name
    try:
        yield
    finally:
        _variant = prev


def library_path() -> str:
    return _build.lib_path(_variant)


def _check(fn: str, status: int):
    if status != PA_OK:
        detail = lib().pa_last_error().decode(errors="replace")
        raise PagedKVError(fn, status, detail)


# ---------------------------------------------------------------------------
# device calls
# ---------------------------------------------------------------------------
def _stream(stream):
    if stream is None:
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return C.c_void_p(stream.cuda_stream)
    return C.c_void_p(int(stream))


def pool_desc(kv_pool: torch.Tensor) -> pa_pool_desc:
    if kv_pool.dim() != 5 or kv_pool.shape[1] != 2 or kv_pool.shape[3] != BLOCK_SIZE:
        raise ValueError("kv_pool must be [num_blocks][2][num_kv_heads][16][head_dim]")
    dt = {torch.float32: PA_F32, torch.bfloat16: PA_BF16}.get(kv_pool.dtype)
    if dt is None:
        raise ValueError(f"kv_pool dtype {kv_pool.dtype} not supported")
    return pa_pool_desc(kv_pool.shape[0], kv_pool.shape[2], kv_pool.shape[4], BLOCK_SIZE, dt)


def _dev(t: torch.Tensor, name: str, dtype=None) -> C.c_void_p:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return C.c_void_p(t.data_ptr())


def pa_reshape_and_cache(k, v, kv_pool, slot_mapping, stream=None):
    desc = pool_desc(kv_pool)
    n = slot_mapping.numel()
    if k.shape != (n, desc.num_kv_heads, desc.head_dim) or v.shape != k.shape:
        raise ValueError("k, v must be [num_tokens][num_kv_heads][head_dim]")
    if n == 0:
        return
    _check("pa_reshape_and_cache", lib().pa_reshape_and_cache(
        _dev(k, "k", kv_pool.dtype), _dev(v, "v", kv_pool.dtype), _dev(kv_pool, "kv_pool"),
        _dev(slot_mapping, "slot_mapping", torch.int64), n, desc, _stream(stream)))


def pa_decode_workspace_size(num_seqs, num_heads, kv_pool, max_seq_len) -> int:
    desc = kv_pool if isinstance(kv_pool, pa_pool_desc) else pool_desc(kv_pool)
    return int(lib().pa_decode_workspace_size(num_seqs, num_heads, desc, max_seq_len))


def pa_decode_partition_tokens(num_seqs, num_heads, kv_pool, max_seq_len) -> int:
    desc = kv_pool if isinstance(kv_pool, pa_pool_desc) else pool_desc(kv_pool)
    return int(lib().pa_decode_partition_tokens(num_seqs, num_heads, desc, max_seq_len))


def alloc_workspace(num_seqs, num_heads, kv_pool, max_seq_len):
    """Device workspace for pa_decode (None when none is needed)."""
    n = pa_decode_workspace_size(num_seqs, num_heads, kv_pool, max_seq_len)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=kv_pool.device)


def pa_decode(out, q, kv_pool, block_tables, seq_lens, scale, max_seq_len, workspace=None,
              stream=None):
    desc = pool_desc(kv_pool)
    B, H, D = q.shape
    if out.shape != q.shape or D != desc.head_dim:
        raise ValueError("q, out must be [num_seqs][num_heads][head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.shape != (B,):
        raise ValueError("block_tables must be [num_seqs][max_blocks], seq_lens [num_seqs]")
    ws_ptr, ws_bytes = C.c_void_p(0), 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    _check("pa_decode", lib().pa_decode(
        _dev(out, "out", kv_pool.dtype), _dev(q, "q", kv_pool.dtype), _dev(kv_pool, "kv_pool"),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(seq_lens, "seq_lens", torch.int32), B, H, float(scale), desc, ws_ptr, ws_bytes,
        int(max_seq_len), _stream(stream)))


def pa_append_decode(out, q, k_new, v_new, kv_pool, slot_mapping, block_tables, seq_lens, scale,
                     max_seq_len, workspace=None, stream=None):
    """pa_reshape_and_cache of each sequence's new token followed by pa_decode,
    in one call (one kernel for bf16 / head_dim 128)."""
    desc = pool_desc(kv_pool)
    B, H, D = q.shape
    if out.shape != q.shape or D != desc.head_dim:
        raise ValueError("q, out must be [num_seqs][num_heads][head_dim]")
    if k_new.shape != (B, desc.num_kv_heads, D) or v_new.shape != k_new.shape:
        raise ValueError("k_new, v_new must be [num_seqs][num_kv_heads][head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.shape != (B,) \
            or slot_mapping.shape != (B,):
        raise ValueError("block_tables [num_seqs][max_blocks], seq_lens and slot_mapping [num_seqs]")
    ws_ptr, ws_bytes = C.c_void_p(0), 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    _check("pa_append_decode", lib().pa_append_decode(
        _dev(out, "out", kv_pool.dtype), _dev(q, "q", kv_pool.dtype), _dev(k_new, "k_new", kv_pool.dtype),
        _dev(v_new, "v_new", kv_pool.dtype), _dev(kv_pool, "kv_pool"),
        _dev(slot_mapping, "slot_mapping", torch.int64), _dev(block_tables, "block_tables", torch.int32),
        block_tables.shape[1], _dev(seq_lens, "seq_lens", torch.int32), B, H, float(scale), desc, ws_ptr,
        ws_bytes, int(max_seq_len), _stream(stream)))


def pa_prefill(out, q, kv_pool, block_tables, seq_lens, query_start, scale, max_query_len, stream=None):
    """Causal attention of each sequence's new tokens (the last
    query_start[b+1] - query_start[b] positions of seq_lens[b]) over its paged
    KV; q, out: [total new tokens][num_heads][128] bf16."""
    desc = pool_desc(kv_pool)
    T, H, D = q.shape
    B = seq_lens.shape[0]
    if out.shape != q.shape or D != desc.head_dim:
        raise ValueError("q, out must be [num_tokens][num_heads][head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.shape != (B,) \
            or query_start.shape != (B + 1,):
        raise ValueError("block_tables [num_seqs][max_blocks], seq_lens [num_seqs], query_start [num_seqs+1]")
    _check("pa_prefill", lib().pa_prefill(
        _dev(out, "out", kv_pool.dtype), _dev(q, "q", kv_pool.dtype), _dev(kv_pool, "kv_pool"),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(seq_lens, "seq_lens", torch.int32), _dev(query_start, "query_start", torch.int32), B, T, H,
        float(scale), desc, int(max_query_len), _stream(stream)))


def pa_decode_noalloc(out, q, kv_pool, block_tables, seq_lens, scale, max_seq_len, stream=None):
    """pa_decode without a workspace, for callers that cannot allocate device
    memory: the split-KV partial results go to the library's fixed per-device
    array (PA_DECODE_NOALLOC_SCRATCH_BYTES). Shapes that need more are rejected
    (PagedKVError WORKSPACE). Calls overlapping on the GPU share that array and
    race."""
    fn = lib().pa_decode_noalloc
    desc = pool_desc(kv_pool)
    B, H, D = q.shape
    if out.shape != q.shape or D != desc.head_dim:
        raise ValueError("q, out must be [num_seqs][num_heads][head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.shape != (B,):
        raise ValueError("block_tables must be [num_seqs][max_blocks], seq_lens [num_seqs]")
    _check("pa_decode_noalloc", fn(
        _dev(out, "out", kv_pool.dtype), _dev(q, "q", kv_pool.dtype), _dev(kv_pool, "kv_pool"),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(seq_lens, "seq_lens", torch.int32), B, H, float(scale), desc, int(max_seq_len),
        _stream(stream)))


def pa_copy_blocks(kv_pool, src, dst, stream=None):
    desc = pool_desc(kv_pool)
    n = src.numel()
    if dst.numel() != n:
        raise ValueError("src and dst differ in length")
    if n == 0:
        return
    _check("pa_copy_blocks", lib().pa_copy_blocks(
        _dev(kv_pool, "kv_pool"), _dev(src, "src", torch.int32), _dev(dst, "dst", torch.int32),
        n, desc, _stream(stream)))


def pa_copy_blocks_between(dst_pool, src_pool, src, dst, stream=None):
    """Block copy between two pools of one block shape (device or pinned host)."""
    desc = pool_desc(dst_pool)
    if pool_desc(src_pool).num_kv_heads != desc.num_kv_heads or src_pool.shape[1:] != dst_pool.shape[1:] \
            or src_pool.dtype != dst_pool.dtype:
        raise ValueError("pools differ in block shape")
    n = src.numel()
    if dst.numel() != n:
        raise ValueError("src and dst differ in length")
    if n == 0:
        return
    for t, name in ((dst_pool, "dst_pool"), (src_pool, "src_pool"), (src, "src"), (dst, "dst")):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if not (t.is_cuda or t.is_pinned()):
            raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")
    if src.dtype != torch.int32 or dst.dtype != torch.int32:
        raise ValueError("src and dst must be int32")
    _check("pa_copy_blocks_between", lib().pa_copy_blocks_between(
        C.c_void_p(dst_pool.data_ptr()), dst_pool.shape[0], C.c_void_p(src_pool.data_ptr()), src_pool.shape[0],
        C.c_void_p(src.data_ptr()), C.c_void_p(dst.data_ptr()), n, desc, _stream(stream)))


def pa_selftest_timeout(limit_ns: int, stream=None):
    """One thread waits on a barrier nothing arrives at until its bounded
    wait gives up after limit_ns, then sets PA_DEVERR_TIMEOUT."""
    _check("pa_selftest_timeout", lib().pa_selftest_timeout(C.c_uint64(int(limit_ns)), _stream(stream)))


def pa_get_device_error(stream=None) -> int:
    """Synchronises the stream, returns and clears the device error bits."""
    flags = C.c_uint32(0)
    st = lib().pa_get_device_error(C.byref(flags), _stream(stream))
    if st not in (PA_OK, 6):
        _check("pa_get_device_error", st)
    return int(flags.value)


# ---------------------------------------------------------------------------
# host block manager and scheduler
# ---------------------------------------------------------------------------
def _i32p(a: np.ndarray):
    return a.ctypes.data_as(_P32)


def _i64p(a: np.ndarray):
    return a.ctypes.data_as(_P64)


class BlockManager:
    """pa_bm_* handle."""

    def __init__(self, num_blocks: int, initial_free_order=None):
        h = C.c_void_p()
        order = None
        if initial_free_order is not None:
            self._order = np.ascontiguousarray(initial_free_order, dtype=np.int32)
            order = _i32p(self._order)
        _check("pa_bm_create", lib().pa_bm_create(num_blocks, BLOCK_SIZE, order, C.byref(h)))
        self.handle = h
        self.num_blocks = num_blocks

    def close(self):
        if getattr(self, "handle", None):
            lib().pa_bm_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def allocate(self, seq: int, num_tokens: int):
        _check("pa_bm_allocate", lib().pa_bm_allocate(self.handle, seq, num_tokens))

    def append_slot(self, seq: int):
        slot, cs, cd = C.c_int64(), C.c_int32(), C.c_int32()
        _check("pa_bm_append_slot", lib().pa_bm_append_slot(
            self.handle, seq, C.byref(slot), C.byref(cs), C.byref(cd)))
        return slot.value, cs.value, cd.value

    def fork(self, parent: int, child: int):
        _check("pa_bm_fork", lib().pa_bm_fork(self.handle, parent, child))

    def free(self, seq: int):
        _check("pa_bm_free", lib().pa_bm_free(self.handle, seq))

    def num_free(self) -> int:
        return int(lib().pa_bm_num_free(self.handle))

    def seq_len(self, seq: int) -> int:
        n = C.c_int32()
        _check("pa_bm_seq_len", lib().pa_bm_seq_len(self.handle, seq, C.byref(n)))
        return n.value

    def refcount(self, block: int) -> int:
        n = C.c_int32()
        _check("pa_bm_refcount", lib().pa_bm_refcount(self.handle, block, C.byref(n)))
        return n.value

    def block_table(self, seq: int) -> list:
        n = C.c_int32()
        cap = 64
        while True:
            buf = np.empty(cap, dtype=np.int32)
            st = lib().pa_bm_block_table(self.handle, seq, _i32p(buf), cap, C.byref(n))
            if st == 8 and n.value > cap:
                cap = n.value
                continue
            _check("pa_bm_block_table", st)
            return buf[: n.value].tolist()

    def free_list(self) -> list:
        n = C.c_int32()
        buf = np.empty(self.num_blocks, dtype=np.int32)
        _check("pa_bm_free_list", lib().pa_bm_free_list(self.handle, _i32p(buf), self.num_blocks, C.byref(n)))
        return buf[: n.value].tolist()

    def set_prefix_caching(self, enable: bool):
        _check("pa_bm_set_prefix_caching", lib().pa_bm_set_prefix_caching(self.handle, int(bool(enable))))

    def allocate_prefix(self, seq: int, prompt_tokens, num_tokens: int) -> int:
        """Allocation sharing cached prompt blocks; returns the cached tokens."""
        toks = np.ascontiguousarray(prompt_tokens, dtype=np.int32)
        cached = C.c_int32()
        _check("pa_bm_allocate_prefix", lib().pa_bm_allocate_prefix(
            self.handle, seq, _i32p(toks), len(toks), num_tokens, C.byref(cached)))
        return cached.value

    def mark_written(self, seq: int):
        _check("pa_bm_mark_written", lib().pa_bm_mark_written(self.handle, seq))

    def evictable_list(self) -> list:
        n = C.c_int32()
        buf = np.empty(self.num_blocks, dtype=np.int32)
        _check("pa_bm_evictable_list", lib().pa_bm_evictable_list(self.handle, _i32p(buf), self.num_blocks,
                                                                  C.byref(n)))
        return buf[: n.value].tolist()

    def num_cached(self) -> int:
        return int(lib().pa_bm_num_cached(self.handle))

    def slots(self, seq: int, start: int, count: int) -> np.ndarray:
        out = np.empty(count, dtype=np.int64)
        _check("pa_bm_slots", lib().pa_bm_slots(self.handle, seq, start, count, _i64p(out)))
        return out

    def pack(self, seqs, max_blocks: int, block_tables=None, seq_lens=None, last_slots=None):
        """Packs a decode batch into host arrays (optionally caller-provided,
        e.g. pinned numpy views). Returns (block_tables, seq_lens, last_slots)."""
        seqs = np.ascontiguousarray(seqs, dtype=np.int64)
        n = len(seqs)
        bt = np.empty((n, max_blocks), np.int32) if block_tables is None else block_tables
        sl = np.empty(n, np.int32) if seq_lens is None else seq_lens
        ls = np.empty(n, np.int64) if last_slots is None else last_slots
        _check("pa_bm_pack", lib().pa_bm_pack(self.handle, _i64p(seqs), n, max_blocks,
                                                _i32p(bt), _i32p(sl), _i64p(ls)))
        return bt, sl, ls


class Scheduler:
    """pa_sched_* handle over a BlockManager; step() returns numpy copies."""

    def __init__(self, bm: BlockManager, arrival_step, prompt_len, output_len, max_blocks_per_seq):
        self.bm = bm
        a = np.ascontiguousarray(arrival_step, dtype=np.int32)
        p = np.ascontiguousarray(prompt_len, dtype=np.int32)
        o = np.ascontiguousarray(output_len, dtype=np.int32)
        h = C.c_void_p()
        _check("pa_sched_create", lib().pa_sched_create(bm.handle, _i32p(a), _i32p(p), _i32p(o), len(a),
                                                        max_blocks_per_seq, C.byref(h)))
        self.handle = h
        self._out = pa_step_out()

    def close(self):
        if getattr(self, "handle", None):
            lib().pa_sched_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_prompt_tokens(self, tokens):
        """Per-request prompt token ids (prefix-cached admission)."""
        lens = [len(t) for t in tokens]
        flat = np.ascontiguousarray(np.concatenate([np.asarray(t, np.int32) for t in tokens])
                                    if tokens else np.zeros(0, np.int32), dtype=np.int32)
        offs = np.ascontiguousarray(np.concatenate([[0], np.cumsum(lens)[:-1]]), dtype=np.int64)
        _check("pa_sched_set_prompt_tokens", lib().pa_sched_set_prompt_tokens(self.handle, _i32p(flat),
                                                                              _i64p(offs)))

    def set_swap(self, num_host_blocks: int):
        """Swap-mode preemption with this many host blocks (0: recompute only)."""
        _check("pa_sched_set_swap", lib().pa_sched_set_swap(self.handle, int(num_host_blocks)))

    def step_raw(self) -> pa_step_out:
        """Runs one step; the returned struct's arrays are valid until the next."""
        _check("pa_sched_step", lib().pa_sched_step(self.handle, C.byref(self._out)))
        return self._out

    def step(self) -> dict:
        o = self.step_raw()

        def arr(ptr, n, dt):
            if n == 0:
                return np.empty(0, dtype=dt)
            return np.ctypeslib.as_array(ptr, shape=(n,)).copy()

        nr = o.num_running
        tables = (np.ctypeslib.as_array(o.block_tables, shape=(nr * o.max_blocks_per_seq,)).copy()
                  .reshape(nr, o.max_blocks_per_seq) if nr else np.empty((0, o.max_blocks_per_seq), np.int32))
        return {
            "step": o.step, "done": o.done,
            "running": arr(o.running, nr, np.int64),
            "seq_lens": arr(o.seq_lens, nr, np.int32),
            "block_tables": tables,
            "decode_slots": arr(o.decode_slots, nr, np.int64),
            "prompt_seqs": arr(o.prompt_seqs, o.num_prompt_seqs, np.int64),
            "prompt_lens": arr(o.prompt_lens, o.num_prompt_seqs, np.int32),
            "prompt_slots": arr(o.prompt_slots, o.num_prompt_tokens, np.int64),
            "cow": list(zip(arr(o.cow_src, o.num_cow, np.int32).tolist(),
                            arr(o.cow_dst, o.num_cow, np.int32).tolist())),
            "admitted": arr(o.admitted, o.num_admitted, np.int64),
            "preempted": arr(o.preempted, o.num_preempted, np.int64),
            "finished": arr(o.finished, o.num_finished, np.int64),
            "num_waiting": o.num_waiting, "num_free_blocks": o.num_free_blocks,
            "prompt_starts": arr(o.prompt_starts, o.num_prompt_seqs, np.int32),
            "num_cached_tokens": o.num_cached_tokens,
            "swap_out": list(zip(arr(o.swap_out_src, o.num_swap_out, np.int32).tolist(),
                                 arr(o.swap_out_dst, o.num_swap_out, np.int32).tolist())),
            "swap_in": list(zip(arr(o.swap_in_src, o.num_swap_in, np.int32).tolist(),
                                arr(o.swap_in_dst, o.num_swap_in, np.int32).tolist())),
            "swapped_out": arr(o.swapped_out, o.num_swapped_out, np.int64),
            "swapped_in": arr(o.swapped_in, o.num_swapped_in, np.int64),
        }


def loaded_library_file() -> str:
    """Path of the shared object this process loaded (for provenance)."""
    return os.path.realpath(_build.LIB)
