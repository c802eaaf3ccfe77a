"""Seeded synthetic workloads shared by the tests, the benchmark and the oracle checks.

This module only produces inputs: random values, sequence lengths, pool
placements, block-manager scripts and request traces. It holds none of the
method's arithmetic (no page counts, slots, tables or attention); the product
path and the oracle each derive those from what is generated here.

Values. Every tensor element is drawn from one counter-based generator, so any
element can be rebuilt on any device from its coordinates alone:
    h_n  = mix(key + n * 0x9E3779B97F4A7C15)      (SplitMix64, Steele, Lea and
           Flood, "Fast Splittable Pseudorandom Number Generators", OOPSLA 2014,
           whose output function is Stafford's "Mix13" 64-bit finaliser)
    x_c  = (sum of the 8 bytes of h_2c and the low 4 bytes of h_2c+1 + 6) / 256 - 6
x_c is an Irwin-Hall(12) variate: mean 0, variance ~1, in [-6, 6), an exact
multiple of 1/256, so it is the same fp32 number on CPU and GPU and rounds to
the same bf16 number. It stands in for the N(0, 1) draws the workloads ask for.
Those values carry at most 11 significant bits, so fp32 products of two of them
are exact. Cases with full_mantissa=True use y_c = fp32(x_c * 1.05) instead
(the product formed in fp64, one rounding to fp32: the same number on every
device), whose fp32 significands are full.

Workloads (sizes follow the decode configurations they are named after):
  tiny      fp32, 4 sequences of length {5, 16, 17, 33} after the append,
            2 query = 2 KV heads, head_dim 64, 64-block pool, scale 1/8.
  mha       Llama-2-7B-shaped: 32 = 32 heads, head_dim 128, bf16, batch 64,
            lengths uniform in [128, 2048], 16384-block pool.
  gqa       Llama-3-8B-shaped: 32 query / 8 KV heads, head_dim 128, bf16,
            batch 256, lengths lognormal (median 1000, sigma 0.8) rounded and
            clipped to [16, 8192], 32768-block pool.
  prefix    32 sequences sharing a 1536-token prefix plus private suffixes
            uniform in [0, 512]; 8 prompts (length uniform in [16, 1024], not a
            multiple of 16) x 4 samples forking at a partial block;
            32/8 heads, head_dim 128, bf16, 4096-block pool.
  trace     2000 requests, Poisson(50) arrivals per step, prompts uniform in
            [16, 1024], outputs geometric with mean 200 capped at 2048,
            40000-block pool, 32/8 heads, head_dim 128, bf16.
  prefill   64 whole prompts, lengths uniform in [16, 1024]; 32/8 heads,
            head_dim 128, bf16, 16384-block pool.
  chunked   64 sequences, cached context uniform in [0, 3072] plus a
            512-token chunk; 32/8 heads, head_dim 128, bf16, 32768 blocks.
Physical placement is random: the block manager's initial free list is a
seeded permutation of the pool.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

# ---------------------------------------------------------------------------
# counter-based value generator (SplitMix64 output stream, Irwin-Hall sum)
# ---------------------------------------------------------------------------
_U64 = 1 << 64


def _s64(x: int) -> int:
    """Unsigned 64-bit constant as the int64 with the same bits."""
    x &= _U64 - 1
    return x - _U64 if x >= (1 << 63) else x


_GAMMA = _s64(0x9E3779B97F4A7C15)
_M1 = _s64(0xBF58476D1CE4E5B9)
_M2 = _s64(0x94D049BB133111EB)


def _shr(z: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _shr(z, 30)) * _M1
    z = (z ^ _shr(z, 27)) * _M2
    return z ^ _shr(z, 31)


def _mix_int(z: int) -> int:
    z &= _U64 - 1
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & (_U64 - 1)
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & (_U64 - 1)
    return z ^ (z >> 31)


def stream_key(*coords: int) -> int:
    """Key of a value stream named by small non-negative integers."""
    k = 0x243F6A8885A308D3
    for c in coords:
        k = _mix_int(k ^ (int(c) & (_U64 - 1)))
    return _s64(k)


FULL_MANTISSA_SCALE = 1.05   # not a dyadic rational: x * 1.05 fills the fp32 significand


def values(key, counters: torch.Tensor, full_mantissa: bool = False) -> torch.Tensor:
    """Irwin-Hall(12) values (fp32) at the given int64 counters of stream `key`
    (an int, or an int64 tensor of keys broadcast against the counters);
    with full_mantissa, each value times 1.05 rounded once to fp32."""
    n = counters.to(torch.int64) * 2
    h1 = _mix(n * _GAMMA + key)
    h2 = _mix((n + 1) * _GAMMA + key)
    shape = h1.shape
    # the 8 bytes of h1 and the low 4 bytes of h2 (little-endian byte views)
    b1 = h1.reshape(-1).contiguous().view(torch.uint8).view(-1, 8)
    b2 = h2.reshape(-1).contiguous().view(torch.uint8).view(-1, 8)[:, :4]
    s = (b1.sum(dim=1, dtype=torch.int32) + b2.sum(dim=1, dtype=torch.int32)).reshape(shape)
    x = (s.to(torch.float32) + 6.0) / 256.0 - 6.0
    if full_mantissa:
        x = (x.to(torch.float64) * FULL_MANTISSA_SCALE).to(torch.float32)
    return x


def value_block(key: int, shape, offset: int = 0, device="cpu",
                dtype=torch.float32, full_mantissa: bool = False) -> torch.Tensor:
    """Values at counters offset .. offset+prod(shape)-1, row-major in `shape`."""
    n = int(np.prod(shape))
    c = torch.arange(offset, offset + n, dtype=torch.int64, device=device)
    return values(key, c, full_mantissa).to(dtype).reshape(shape)


TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}

# value-stream tags
TAG_POOL, TAG_Q, TAG_K, TAG_V = 1, 2, 3, 4
TAG_TRACE_KV, TAG_TRACE_Q, TAG_TRACE_PQ = 5, 6, 7


# ---------------------------------------------------------------------------
# single-step decode workloads
# ---------------------------------------------------------------------------
@dataclass
class DecodeCase:
    """One decode step over a pool prepared by a block-manager script.

    ops: block-manager operations run in order before the step:
         ("allocate", seq, num_tokens), ("fork", parent, child), ("free", seq),
         ("append", seq) (a token whose K/V is already in the pool).
    batch: the decode batch, in order; each sequence appends one token (its
         K/V are k_new[i], v_new[i]) and then attends over its whole length.
    table_width: columns of the packed block tables.
    """
    name: str
    seed: int
    num_blocks: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str
    scale: float
    free_order: np.ndarray
    ops: list
    batch: list
    table_width: int
    max_seq_len: int
    info: dict = field(default_factory=dict)
    full_mantissa: bool = False   # values x * 1.05 (full fp32 significands)

    @property
    def pool_shape(self):
        return (self.num_blocks, 2, self.num_kv_heads, 16, self.head_dim)

    def make_pool(self, device="cpu", chunk_blocks: int = 1024) -> torch.Tensor:
        """Initial pool contents (every slot holds a value, used or not)."""
        pool = torch.empty(self.pool_shape, dtype=TORCH_DTYPE[self.dtype], device=device)
        per_block = int(np.prod(self.pool_shape[1:]))
        key = stream_key(self.seed, TAG_POOL)
        for b0 in range(0, self.num_blocks, chunk_blocks):
            b1 = min(b0 + chunk_blocks, self.num_blocks)
            pool[b0:b1] = value_block(key, (b1 - b0,) + self.pool_shape[1:],
                                      offset=b0 * per_block, device=device,
                                      dtype=pool.dtype, full_mantissa=self.full_mantissa)
        return pool

    def pool_blocks(self, block_ids, device="cpu") -> torch.Tensor:
        """Initial contents of selected blocks only, [n][2][Hkv][16][D]."""
        per_block = int(np.prod(self.pool_shape[1:]))
        key = stream_key(self.seed, TAG_POOL)
        ids = torch.as_tensor(np.asarray(block_ids, dtype=np.int64), device=device)
        c = ids[:, None] * per_block + torch.arange(per_block, device=device)[None, :]
        return values(key, c, self.full_mantissa).to(TORCH_DTYPE[self.dtype]).reshape(
            (len(block_ids),) + self.pool_shape[1:])

    def make_q(self, device="cpu") -> torch.Tensor:
        return value_block(stream_key(self.seed, TAG_Q),
                           (len(self.batch), self.num_heads, self.head_dim),
                           device=device, dtype=TORCH_DTYPE[self.dtype],
                           full_mantissa=self.full_mantissa)

    def make_kv_new(self, device="cpu"):
        shape = (len(self.batch), self.num_kv_heads, self.head_dim)
        k = value_block(stream_key(self.seed, TAG_K), shape, device=device,
                        dtype=TORCH_DTYPE[self.dtype], full_mantissa=self.full_mantissa)
        v = value_block(stream_key(self.seed, TAG_V), shape, device=device,
                        dtype=TORCH_DTYPE[self.dtype], full_mantissa=self.full_mantissa)
        return k, v


def _decode_case_from_lens(name, seed, lens_after, num_blocks, num_heads, num_kv_heads,
                           head_dim, dtype, scale, table_width, max_seq_len, rng):
    """Sequences 0..B-1 hold len-1 tokens of cached context, then append one."""
    free_order = rng.permutation(num_blocks).astype(np.int32)
    ops = [("allocate", b, int(n) - 1) for b, n in enumerate(lens_after)]
    return DecodeCase(name=name, seed=seed, num_blocks=num_blocks, num_heads=num_heads,
                      num_kv_heads=num_kv_heads, head_dim=head_dim, dtype=dtype,
                      scale=scale, free_order=free_order, ops=ops,
                      batch=list(range(len(lens_after))), table_width=table_width,
                      max_seq_len=max_seq_len,
                      info={"seq_lens_after_append": [int(x) for x in lens_after]})


def tiny_case(seed: int = 0, full_mantissa: bool = False) -> DecodeCase:
    rng = np.random.default_rng(seed)
    case = _decode_case_from_lens("tiny_fp32_full" if full_mantissa else "tiny_fp32", seed,
                                  [5, 16, 17, 33], 64, 2, 2, 64, "f32", 1.0 / 8.0, 4, 64, rng)
    case.full_mantissa = full_mantissa
    return case


def mha_case(seed: int = 0, batch: int = 64) -> DecodeCase:
    rng = np.random.default_rng(seed + 101)
    lens = rng.integers(128, 2048, size=batch, endpoint=True)
    return _decode_case_from_lens("mha_llama2_7b", seed, lens, 16384, 32, 32, 128,
                                  "bf16", 128 ** -0.5, 128, 2048, rng)


def gqa_lens(rng, batch: int):
    x = rng.lognormal(mean=np.log(1000.0), sigma=0.8, size=batch)
    return np.clip(np.round(x), 16, 8192).astype(np.int64)


def gqa_case(seed: int = 0, batch: int = 256) -> DecodeCase:
    rng = np.random.default_rng(seed + 202)
    lens = gqa_lens(rng, batch)
    return _decode_case_from_lens("gqa_llama3_8b", seed, lens, 32768, 32, 8, 128,
                                  "bf16", 128 ** -0.5, 512, 8192, rng)


def custom_case(name, seed, lens_after, num_blocks, num_heads, num_kv_heads, head_dim,
                dtype, table_width, max_seq_len, scale=None, full_mantissa=False) -> DecodeCase:
    """A decode step with caller-chosen lengths (edge cases, small variants)."""
    rng = np.random.default_rng(seed + 303)
    if scale is None:
        scale = head_dim ** -0.5
    case = _decode_case_from_lens(name, seed, list(lens_after), num_blocks, num_heads,
                                  num_kv_heads, head_dim, dtype, scale, table_width,
                                  max_seq_len, rng)
    case.full_mantissa = full_mantissa
    return case


def prefix_case(seed: int = 0) -> DecodeCase:
    """Shared prefix + parallel sampling (copy-on-write at a partial block)."""
    rng = np.random.default_rng(seed + 404)
    num_blocks = 4096
    free_order = rng.permutation(num_blocks).astype(np.int32)
    ops = []
    # (i) one 1536-token prefix held by seq 10000, forked to 32 sequences, each
    #     of which then grows a private suffix; the holder is released.
    holder = 10000
    ops.append(("allocate", holder, 1536))
    for i in range(32):
        ops.append(("fork", holder, i))
    ops.append(("free", holder))
    suffix = rng.integers(0, 512, size=32, endpoint=True)
    for i in range(32):
        ops.extend([("append", i)] * int(suffix[i]))
    # (ii) 8 prompts of length not a multiple of 16, each sampled 4 times
    #      (the prompt sequence is sample 0, forked three times).
    plens = []
    while len(plens) < 8:
        n = int(rng.integers(16, 1024, endpoint=True))
        if n % 16 != 0:
            plens.append(n)
    batch = list(range(32))
    for j, n in enumerate(plens):
        p = 100 + j
        ops.append(("allocate", p, n))
        batch.append(p)
        for s in range(1, 4):
            c = 200 + 4 * j + s
            ops.append(("fork", p, c))
            batch.append(c)
    return DecodeCase(name="shared_prefix", seed=seed, num_blocks=num_blocks,
                      num_heads=32, num_kv_heads=8, head_dim=128, dtype="bf16",
                      scale=128 ** -0.5, free_order=free_order, ops=ops, batch=batch,
                      table_width=136, max_seq_len=2176,
                      info={"prefix_len": 1536, "suffix_lens": [int(x) for x in suffix],
                            "prompt_lens": plens, "samples": 4})


# ---------------------------------------------------------------------------
# prefill / chunked-prefill workloads
# ---------------------------------------------------------------------------
@dataclass
class PrefillCase:
    """One prefill step: sequence b holds ctx_lens[b] tokens of cached KV (from
    the initial pool) and brings query_lens[b] new tokens, whose K/V
    (k_new/v_new rows, in sequence order) are appended first; each new token
    then attends causally over its sequence. The block manager allocates every
    sequence's full length (ops) before the step."""
    name: str
    seed: int
    num_blocks: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str
    scale: float
    free_order: np.ndarray
    ctx_lens: list
    query_lens: list
    table_width: int
    info: dict = field(default_factory=dict)
    full_mantissa: bool = False   # prefill inputs are bf16: the short values round the same

    pool_shape = DecodeCase.pool_shape
    make_pool = DecodeCase.make_pool
    pool_blocks = DecodeCase.pool_blocks

    @property
    def ops(self):
        return [("allocate", b, int(c) + int(n))
                for b, (c, n) in enumerate(zip(self.ctx_lens, self.query_lens))]

    @property
    def num_tokens(self) -> int:
        return int(sum(self.query_lens))

    @property
    def max_query_len(self) -> int:
        return int(max(self.query_lens)) if len(self.query_lens) else 0

    def make_q(self, device="cpu") -> torch.Tensor:
        return value_block(stream_key(self.seed, TAG_Q), (self.num_tokens, self.num_heads, self.head_dim),
                           device=device, dtype=TORCH_DTYPE[self.dtype])

    def make_kv_new(self, device="cpu"):
        shape = (self.num_tokens, self.num_kv_heads, self.head_dim)
        k = value_block(stream_key(self.seed, TAG_K), shape, device=device, dtype=TORCH_DTYPE[self.dtype])
        v = value_block(stream_key(self.seed, TAG_V), shape, device=device, dtype=TORCH_DTYPE[self.dtype])
        return k, v


def prefill_custom(name, seed, ctx_lens, query_lens, num_heads=32, num_kv_heads=8,
                   num_blocks=None, table_width=None) -> PrefillCase:
    """A prefill step with caller-chosen lengths (bf16, head_dim 128)."""
    rng = np.random.default_rng(seed + 707)
    totals = [int(c) + int(n) for c, n in zip(ctx_lens, query_lens)]
    need = sum((t + 15) // 16 for t in totals)
    if num_blocks is None:
        num_blocks = max(64, 2 * need)
    if table_width is None:
        table_width = max(1, max((t + 15) // 16 for t in totals) if totals else 1)
    return PrefillCase(name=name, seed=seed, num_blocks=num_blocks, num_heads=num_heads,
                       num_kv_heads=num_kv_heads, head_dim=128, dtype="bf16", scale=128 ** -0.5,
                       free_order=rng.permutation(num_blocks).astype(np.int32),
                       ctx_lens=[int(c) for c in ctx_lens], query_lens=[int(n) for n in query_lens],
                       table_width=table_width)


def prefill_case(seed: int = 0, batch: int = 64) -> PrefillCase:
    """Whole prompts: `batch` prompts with lengths uniform in [16, 1024] (the
    trace's prompt distribution), Llama-3-8B-shaped heads (32 / 8, head_dim
    128, bf16), random placement in a 256 x batch-block pool (16384 at 64)."""
    rng = np.random.default_rng(seed + 808)
    n = rng.integers(16, 1024, size=batch, endpoint=True)
    nb = 256 * batch
    return PrefillCase(name="prefill_gqa", seed=seed, num_blocks=nb, num_heads=32, num_kv_heads=8,
                       head_dim=128, dtype="bf16", scale=128 ** -0.5,
                       free_order=rng.permutation(nb).astype(np.int32),
                       ctx_lens=[0] * batch, query_lens=[int(x) for x in n], table_width=64)


def chunked_prefill_case(seed: int = 0, batch: int = 64, chunk: int = 512) -> PrefillCase:
    """Chunked prefill: `batch` sequences with cached context uniform in
    [0, 3072] each bring a chunk of `chunk` new prompt tokens; heads as
    prefill_case, a 512 x batch-block pool (32768 at 64)."""
    rng = np.random.default_rng(seed + 909)
    ctx = rng.integers(0, 3072, size=batch, endpoint=True)
    nb = 512 * batch
    return PrefillCase(name="chunked_prefill_gqa", seed=seed, num_blocks=nb, num_heads=32,
                       num_kv_heads=8, head_dim=128, dtype="bf16", scale=128 ** -0.5,
                       free_order=rng.permutation(nb).astype(np.int32),
                       ctx_lens=[int(x) for x in ctx], query_lens=[chunk] * batch,
                       table_width=(3072 + chunk + 15) // 16)


# ---------------------------------------------------------------------------
# continuous-batching trace
# ---------------------------------------------------------------------------
TRACE_MAX_POS = 4096    # positions per request in the K/V value space
TRACE_MAX_REQ = 1 << 16
TRACE_MAX_STEP = 1 << 20


@dataclass
class TraceCase:
    seed: int
    arrival_step: np.ndarray
    prompt_len: np.ndarray
    output_len: np.ndarray
    num_blocks: int
    num_layers: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str
    scale: float
    table_width: int
    # shared-prompt traces: prompt token ids per request, and which of the
    # system prompts (sys_id) covers its first sys_len tokens
    prompt_tokens: list = None
    sys_id: np.ndarray = None
    sys_len: np.ndarray = None

    def _owner(self, reqs: torch.Tensor, pos: torch.Tensor) -> torch.Tensor:
        """Value stream of each (request, position): a system prompt's own
        stream inside it (identical prefixes hold identical K/V, as a model's
        would), the request's stream elsewhere."""
        if self.sys_len is None:
            return reqs
        dev = reqs.device
        sl = torch.as_tensor(self.sys_len, dtype=torch.int64, device=dev)[reqs]
        sid = torch.as_tensor(self.sys_id, dtype=torch.int64, device=dev)[reqs]
        return torch.where(pos < sl, TRACE_MAX_REQ + sid, reqs)

    def kv_values(self, layer: int, reqs, positions, device="cpu"):
        """K and V of token `positions[i]` of request `reqs[i]` in `layer`:
        two [n][num_kv_heads][head_dim] tensors. The same (layer, request,
        position) always gives the same values, so recomputed K/V after a
        preemption are identical to the originals."""
        per_tok = 2 * self.num_kv_heads * self.head_dim
        r = torch.as_tensor(np.asarray(reqs, dtype=np.int64), device=device)
        p = torch.as_tensor(np.asarray(positions, dtype=np.int64), device=device)
        base = (self._owner(r, p) * TRACE_MAX_POS + p) * per_tok
        c = base[:, None] + torch.arange(per_tok, device=device)[None, :]
        x = values(stream_key(self.seed, TAG_TRACE_KV, layer), c).to(TORCH_DTYPE[self.dtype])
        x = x.reshape(len(r), 2, self.num_kv_heads, self.head_dim)
        return x[:, 0].contiguous(), x[:, 1].contiguous()

    def prompt_q_values(self, layer: int, reqs, positions, device="cpu"):
        """Query of prompt token `positions[i]` of request `reqs[i]` in `layer`
        (the prefill queries): [n][H][D]. The same (layer, request, position)
        always gives the same values."""
        per = self.num_heads * self.head_dim
        r = torch.as_tensor(np.asarray(reqs, dtype=np.int64), device=device)
        p = torch.as_tensor(np.asarray(positions, dtype=np.int64), device=device)
        c = ((r * TRACE_MAX_POS + p) * per)[:, None] + torch.arange(per, device=device)[None, :]
        x = values(stream_key(self.seed, TAG_TRACE_PQ, layer), c).to(TORCH_DTYPE[self.dtype])
        return x.reshape(len(r), self.num_heads, self.head_dim)

    def step_inputs(self, step: int, running, seq_lens, prompt_reqs, prompt_pos, device,
                    chunk_elems: int = 1 << 26, stacked: bool = False, prefill: bool = False):
        """Per-layer inputs of one continuous-batching step: the query and the
        new token's K/V of each running request (position seq_len - 1), and the
        prompt K/V of the (re)admitted requests (with prefill, their prompt
        queries too), generated layer by layer in chunks of at most
        `chunk_elems` values."""
        per_tok = 2 * self.num_kv_heads * self.head_dim
        reqs_p = np.asarray(prompt_reqs, np.int64)
        pos_p = np.asarray(prompt_pos, np.int64)
        dec_pos = np.asarray(seq_lens, np.int64) - 1
        step_chunk = max(1, chunk_elems // per_tok)
        dt = TORCH_DTYPE[self.dtype]
        n = len(running)
        L = self.num_layers
        # decode-token K/V and queries of every layer in one generator call each
        kv_keys = torch.tensor([stream_key(self.seed, TAG_TRACE_KV, l) for l in range(L)],
                               dtype=torch.int64, device=device)[:, None]
        q_keys = torch.tensor([stream_key(self.seed, TAG_TRACE_Q, l) for l in range(L)],
                              dtype=torch.int64, device=device)[:, None]
        r = torch.as_tensor(np.asarray(running, np.int64), device=device)
        p = torch.as_tensor(dec_pos, device=device)
        c = (((self._owner(r, p) * TRACE_MAX_POS + p) * per_tok)[:, None]
             + torch.arange(per_tok, device=device)[None, :]).reshape(1, -1)
        kv_all = values(kv_keys, c).to(dt).reshape(L, n, 2, self.num_kv_heads, self.head_dim)
        per_q = self.num_heads * self.head_dim
        cq = (((step * TRACE_MAX_REQ + r) * per_q)[:, None]
              + torch.arange(per_q, device=device)[None, :]).reshape(1, -1)
        q_all = values(q_keys, cq).to(dt).reshape(L, n, self.num_heads, self.head_dim)
        out = []
        for layer in range(L):
            k_d = kv_all[layer, :, 0].contiguous()
            v_d = kv_all[layer, :, 1].contiguous()
            q = q_all[layer].contiguous()
            if len(reqs_p) <= step_chunk:
                k_p, v_p = self.kv_values(layer, reqs_p, pos_p, device)
            else:
                parts = [self.kv_values(layer, reqs_p[i:i + step_chunk], pos_p[i:i + step_chunk], device)
                         for i in range(0, len(reqs_p), step_chunk)]
                k_p = torch.cat([a for a, _ in parts])
                v_p = torch.cat([b for _, b in parts])
            item = {"q": q, "k_dec": k_d, "v_dec": v_d, "k_prompt": k_p, "v_prompt": v_p}
            if prefill:
                per_q_tok = self.num_heads * self.head_dim
                qchunk = max(1, chunk_elems // per_q_tok)
                item["q_prompt"] = torch.cat(
                    [self.prompt_q_values(layer, reqs_p[i:i + qchunk], pos_p[i:i + qchunk], device)
                     for i in range(0, len(reqs_p), qchunk)]) if len(reqs_p) else \
                    torch.empty(0, self.num_heads, self.head_dim, dtype=dt, device=device)
            out.append(item)
        if stacked:
            return out, (q_all, kv_all[:, :, 0], kv_all[:, :, 1])
        return out

    def q_values(self, layer: int, step: int, reqs, device="cpu"):
        """Query of each request in `reqs` at (layer, step): [n][H][D]."""
        per = self.num_heads * self.head_dim
        r = torch.as_tensor(np.asarray(reqs, dtype=np.int64), device=device)
        c = ((step * TRACE_MAX_REQ + r) * per)[:, None] + torch.arange(per, device=device)[None, :]
        x = values(stream_key(self.seed, TAG_TRACE_Q, layer), c).to(TORCH_DTYPE[self.dtype])
        return x.reshape(len(r), self.num_heads, self.head_dim)


def trace_case(seed: int = 0, n_requests: int = 2000, rate: float = 50.0,
               num_blocks: int = 40000, num_layers: int = 32, output_cap: int = 2048) -> TraceCase:
    rng = np.random.default_rng(seed + 505)
    arrivals = []
    step = 0
    while len(arrivals) < n_requests:
        k = int(rng.poisson(rate))
        arrivals.extend([step] * k)
        step += 1
    arrivals = np.asarray(arrivals[:n_requests], dtype=np.int32)
    prompt = rng.integers(16, 1024, size=n_requests, endpoint=True).astype(np.int32)
    output = np.minimum(rng.geometric(1.0 / 200.0, size=n_requests), output_cap).astype(np.int32)
    return TraceCase(seed=seed, arrival_step=arrivals, prompt_len=prompt, output_len=output,
                     num_blocks=num_blocks, num_layers=num_layers, num_heads=32,
                     num_kv_heads=8, head_dim=128, dtype="bf16", scale=128 ** -0.5,
                     table_width=192)


def prefix_trace_case(seed: int = 0, n_requests: int = 2000, rate: float = 50.0,
                      num_blocks: int = 40000, num_layers: int = 32, n_system: int = 8,
                      vocab: int = 32000) -> TraceCase:
    """The arrival trace with shared prompts: every request's prompt is one of
    `n_system` system prompts (length uniform in [256, 1024]) followed by its
    own user tokens (length uniform in [16, 512]); token ids uniform in
    [0, vocab). Arrivals and output lengths as in trace_case."""
    rng = np.random.default_rng(seed + 606)
    arrivals = []
    step = 0
    while len(arrivals) < n_requests:
        arrivals.extend([step] * int(rng.poisson(rate)))
        step += 1
    arrivals = np.asarray(arrivals[:n_requests], dtype=np.int32)
    systems = [rng.integers(0, vocab, size=int(rng.integers(256, 1024, endpoint=True))).astype(np.int32)
               for _ in range(n_system)]
    sys_id = rng.integers(0, n_system, size=n_requests).astype(np.int32)
    prompts = []
    for i in range(n_requests):
        user = rng.integers(0, vocab, size=int(rng.integers(16, 512, endpoint=True))).astype(np.int32)
        prompts.append(np.concatenate([systems[sys_id[i]], user]))
    prompt_len = np.asarray([len(p) for p in prompts], dtype=np.int32)
    output = np.minimum(rng.geometric(1.0 / 200.0, size=n_requests), 2048).astype(np.int32)
    sys_len = np.asarray([len(systems[s]) for s in sys_id], dtype=np.int32)
    return TraceCase(seed=seed, arrival_step=arrivals, prompt_len=prompt_len, output_len=output,
                     num_blocks=num_blocks, num_layers=num_layers, num_heads=32, num_kv_heads=8,
                     head_dim=128, dtype="bf16", scale=128 ** -0.5, table_width=224,
                     prompt_tokens=prompts, sys_id=sys_id, sys_len=sys_len)
