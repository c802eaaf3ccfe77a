"""B200-native paged KV cache: cache append, split-KV paged decode attention and
block copy as sm_100a CUDA kernels behind a C ABI (libpagedkv.so), with a host
C++ block manager and continuous-batching scheduler. This package holds the
kernels and host sources (csrc/), the in-tree build, the ctypes binding and the
seeded synthetic workloads."""
from .binding import (  # noqa: F401
    BLOCK_SIZE, PA_DEVERR_BLOCK, PA_DEVERR_SEQLEN, PA_DEVERR_SLOT, PA_DEVERR_TIMEOUT, BlockManager,
    PagedKVError, Scheduler, alloc_workspace, lib, library_path, pa_append_decode, pa_copy_blocks,
    pa_copy_blocks_between, pa_decode, pa_decode_partition_tokens, pa_decode_workspace_size,
    pa_get_device_error, pa_prefill, pa_reshape_and_cache, pa_selftest_timeout, pool_desc,
)
