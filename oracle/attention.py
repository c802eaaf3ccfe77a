"""fp64 oracle for the paged KV cache: cache append, block copy, decode attention.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): used by tests/, smoke() and
bench.py's CPU baseline; never by the product path.

Pool layout read here: kv_pool[num_blocks][2][num_kv_heads][16][head_dim], index
0 of axis 1 = K, 1 = V. A pool may be a float array (fp32/fp64) or the raw
uint16/int16 bits of bf16 values (pass dtype="bf16"); gathered rows are upcast
to fp64 exactly.

Sources:
  "大模型推理性能优化：PagedAttention与Continuous Batching原理与实践" §2.1
      (K/V of every earlier token are kept; per layer [batch, heads, seq, dim]),
      §2.2 (fixed 16-token pages anywhere in a pooled buffer, a logical->physical
      page table, and the gather of the scattered blocks into a logical view at
      attention time; the new token's K/V is scattered into its slot).
  "vLLM 原理：PagedAttention 和 Continuous Batching", "工作原理" (page table per
      request; position p sits in logical page p // 16).
"""
from __future__ import annotations

import numpy as np

BLOCK_SIZE = 16  # tokens per page (both pages: 16 tokens of KV per page)


# --------------------------------------------------------------------------
# element decoding
# --------------------------------------------------------------------------
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 numbers given as their 16-bit patterns.

    A bf16 number is the upper half of an IEEE binary32; widening the pattern
    to 32 bits with 16 zero low bits gives the same value as a float32.
    """
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):  # NaN patterns stay NaN
        return b.view(np.float32).astype(np.float64)


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Upcast an element array of the given storage dtype to fp64 (exact)."""
    if dtype == "bf16":
        return bf16_bits_to_f64(x)
    if dtype in ("f32", "f64"):
        return np.asarray(x, dtype=np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


# --------------------------------------------------------------------------
# gather through the page table
# --------------------------------------------------------------------------
def slot_of(block_table, position: int) -> int:
    """Slot of token position p: table[p // 16] * 16 + p % 16 ("工作原理":
    the page table maps the request's logical pages to physical pages)."""
    return int(block_table[position // BLOCK_SIZE]) * BLOCK_SIZE + position % BLOCK_SIZE


def gather_kv(pool, block_table, seq_len: int, dtype: str):
    """Logical K and V of one sequence, [seq_len][num_kv_heads][head_dim] fp64.

    Follows the page table one token at a time: token t is read from physical
    block table[t // 16], row t % 16 ("PagedAttention与Continuous Batching原理与
    实践" §2.2: the scattered physical blocks are gathered into a logical view).
    """
    n_kv, d = pool.shape[2], pool.shape[4]
    K = np.empty((seq_len, n_kv, d), dtype=np.float64)
    V = np.empty((seq_len, n_kv, d), dtype=np.float64)
    for t in range(seq_len):
        blk = int(block_table[t // BLOCK_SIZE])
        row = t % BLOCK_SIZE
        K[t] = to_f64(pool[blk, 0, :, row, :], dtype)
        V[t] = to_f64(pool[blk, 1, :, row, :], dtype)
    return K, V


# --------------------------------------------------------------------------
# decode attention
# --------------------------------------------------------------------------
def softmax_attention(q_h: np.ndarray, K_g: np.ndarray, V_g: np.ndarray,
                      scale: float) -> np.ndarray:
    """Textbook single-query attention in fp64:
    s_t = scale * <q, K_t>;  p = exp(s - max s) / sum exp(s - max s);  o = sum p_t V_t.
    """
    s = scale * (K_g @ q_h)
    s = s - s.max()
    p = np.exp(s)
    p = p / p.sum()
    return p @ V_g


def paged_decode(q, pool, block_tables, seq_lens, scale: float, dtype: str):
    """out[b][h] = softmax(scale * K_b q_bh) V_b over the sequence's gathered KV.

    q: [B][H][D] in storage dtype `dtype`; query head h reads KV head
    h // (H / num_kv_heads). A sequence of length 0 gives zeros.
    Returns fp64 [B][H][D].
    """
    qf = to_f64(q, dtype)
    B, H, D = qf.shape
    n_kv = pool.shape[2]
    G = H // n_kv
    out = np.zeros((B, H, D), dtype=np.float64)
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        K, V = gather_kv(pool, block_tables[b], L, dtype)
        for h in range(H):
            g = h // G
            out[b, h] = softmax_attention(qf[b, h], K[:, g, :], V[:, g, :], scale)
    return out


# --------------------------------------------------------------------------
# split-KV reading: per-partition online-softmax state and its merge
# --------------------------------------------------------------------------
def partition_state(q_h, K_g, V_g, scale: float, start: int, stop: int):
    """State of one partition [start, stop) of the tokens:
    m = max_t s_t;  l = sum_t exp(s_t - m);  acc = sum_t exp(s_t - m) V_t."""
    s = scale * (K_g[start:stop] @ q_h)
    m = s.max()
    e = np.exp(s - m)
    return m, e.sum(), e @ V_g[start:stop]


def merge_partition_states(states):
    """Log-sum-exp merge of partition states into the attention output:
    M = max m_P;  L = sum l_P exp(m_P - M);  out = sum exp(m_P - M) acc_P / L."""
    M = max(m for m, _, _ in states)
    L = sum(l * np.exp(m - M) for m, l, _ in states)
    acc = sum(np.exp(m - M) * a for m, _, a in states)
    return acc / L


def paged_decode_split(q, pool, block_tables, seq_lens, scale: float, dtype: str,
                       partition_tokens: int):
    """Same result as paged_decode, computed as partitions of
    `partition_tokens` tokens each, merged by merge_partition_states."""
    qf = to_f64(q, dtype)
    B, H, D = qf.shape
    G = H // pool.shape[2]
    out = np.zeros((B, H, D), dtype=np.float64)
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        K, V = gather_kv(pool, block_tables[b], L, dtype)
        for h in range(H):
            g = h // G
            states = [partition_state(qf[b, h], K[:, g, :], V[:, g, :], scale,
                                      p0, min(p0 + partition_tokens, L))
                      for p0 in range(0, L, partition_tokens)]
            out[b, h] = merge_partition_states(states)
    return out


# --------------------------------------------------------------------------
# cache append and block copy (bit copies)
# --------------------------------------------------------------------------
def reshape_and_cache(pool, k, v, slot_mapping):
    """Scatter each token's K/V into its slot, in place, as a bit copy
    ("PagedAttention与Continuous Batching原理与实践" §2.2, scatter):
    pool[s // 16][0][:, s % 16, :] = k[t]; pool[s // 16][1][...] = v[t].
    A negative slot is padding and skipped. A slot past the pool is skipped
    and reported. Returns the list of rejected token indices."""
    n_slots = pool.shape[0] * BLOCK_SIZE
    rejected = []
    for t, s in enumerate(np.asarray(slot_mapping).tolist()):
        if s < 0:
            continue
        if s >= n_slots:
            rejected.append(t)
            continue
        blk, row = divmod(s, BLOCK_SIZE)
        pool[blk, 0, :, row, :] = k[t]
        pool[blk, 1, :, row, :] = v[t]
    return rejected


def copy_blocks(pool, src, dst):
    """pool[dst[i]] = pool[src[i]] for each pair in order (whole block: K and V,
    every head). Out-of-range ids skip the pair and are reported."""
    n = pool.shape[0]
    rejected = []
    for i, (s, d) in enumerate(zip(np.asarray(src).tolist(), np.asarray(dst).tolist())):
        if not (0 <= s < n and 0 <= d < n):
            rejected.append(i)
            continue
        pool[d] = pool[s]
    return rejected


# --------------------------------------------------------------------------
# prefill / chunked prefill: the new tokens of each sequence attend causally
# --------------------------------------------------------------------------
def paged_prefill(q, pool, block_tables, seq_lens, query_lens, scale: float, dtype: str):
    """Causal attention of each sequence's newest query_lens[b] tokens.

    Sequence b holds seq_lens[b] tokens of KV (its new tokens included, as the
    last query_lens[b] positions). Query row i of sequence b (rows of q are the
    sequences' new tokens, concatenated in order) sits at position
    p = seq_lens[b] - query_lens[b] + i and attends to positions 0..p
    ("PagedAttention与Continuous Batching原理与实践" §2: prefill processes the
    whole prompt; each token sees itself and every earlier token).
    q: [sum(query_lens)][H][D] in storage dtype; returns fp64 of that shape."""
    qf = to_f64(q, dtype)
    T, H, D = qf.shape
    G = H // pool.shape[2]
    out = np.zeros((T, H, D), dtype=np.float64)
    row = 0
    for b, (L, n) in enumerate(zip(seq_lens, query_lens)):
        L, n = int(L), int(n)
        if n == 0:
            continue
        K, V = gather_kv(pool, block_tables[b], L, dtype)
        for i in range(n):
            p = L - n + i
            for h in range(H):
                g = h // G
                out[row + i, h] = softmax_attention(qf[row + i, h], K[:p + 1, g, :], V[:p + 1, g, :], scale)
        row += n
    return out
