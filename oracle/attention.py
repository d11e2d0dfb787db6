"""Decode attention through the block table, in float64 (oracle side).

What it computes is the plain definition the method reaches: for sequence
``s`` and query head ``h``, gather the keys and values of tokens
``0..ctx_s-1`` through the block table into contiguous arrays, then take
``softmax(scale * K q) V``. The pages say the kernel follows the block-table
mapping while it computes attention and that the indirection is invisible to
the result, the way an MMU hides physical frames ("vLLM: PagedAttention and
continuous batching", direct answer; "PagedAttention: The vLLM Paper", "The
Core Idea", note under the block-table figure).

Readings where the pages are silent:
  * Query head ``h`` reads KV head ``h // G`` with ``G = Hq / Hkv`` (grouped-query
    attention is only named on the pages, in "Impact and Follow-Ups", item 3).
  * The context length includes the token written in the same decode step, so a
    decode query attends to itself; no mask beyond ``t < ctx``.
  * A sequence with no tokens yields a zero output.

The split-KV partial state and its merge are restated too: a partition of the
context produces ``(m, l, acc)`` = (max logit, sum of exp(logit - m), sum of
exp(logit - m) * v), and partitions merge by rescaling to the common maximum.
This is exact in real arithmetic, which the tests check against the unsplit form.
"""

from __future__ import annotations

import numpy as np

from .fpbits import bits_to_f64


def softmax_attention(q, K, V, scale: float) -> np.ndarray:
    """``softmax(scale * K q) V`` for one query, float64; zeros when K is empty."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(V.shape[1] if V.ndim == 2 else q.shape[0], dtype=np.float64)
    x = scale * (K @ q)
    x = x - x.max()
    p = np.exp(x)
    p = p / p.sum()
    return p @ V


def gather_sequence(cache_bits, table_row, ctx: int, kv_head: int, block_size: int):
    """Bits of one KV head's rows for tokens ``0..ctx-1`` of a sequence, in order.

    Token ``t`` sits at offset ``t % block_size`` of physical block
    ``table_row[t // block_size]``.
    """
    t = np.arange(ctx)
    blocks = np.asarray(table_row, dtype=np.int64)[t // block_size]
    if ctx and (blocks.min() < 0 or blocks.max() >= cache_bits.shape[0]):
        raise IndexError("block table entry outside the pool")
    return cache_bits[blocks, kv_head, t % block_size, :]


def paged_decode(q_bits, k_cache_bits, v_cache_bits, block_tables, context_lens, scale: float,
                 dtype: str, block_size: int = 16, rows=None) -> np.ndarray:
    """Decode attention for every (sequence, query head), or only for ``rows``.

    ``q_bits`` is ``[B, Hq, d]``; caches are ``[NB, Hkv, block_size, d]``; all as
    uint16 bit patterns of ``dtype``. Returns float64 ``[B, Hq, d]`` (entries
    outside ``rows`` are left NaN when ``rows`` is given).
    """
    B, Hq, d = q_bits.shape
    Hkv = k_cache_bits.shape[1]
    if Hq % Hkv:
        raise ValueError("query heads must be a multiple of KV heads")
    G = Hq // Hkv
    out = np.full((B, Hq, d), np.nan if rows is not None else 0.0, dtype=np.float64)
    todo = rows if rows is not None else [(s, h) for s in range(B) for h in range(Hq)]
    cache: dict = {}
    for s, h in todo:
        kvh = h // G
        key = (s, kvh)
        if key not in cache:
            ctx = int(context_lens[s])
            K = bits_to_f64(gather_sequence(k_cache_bits, block_tables[s], ctx, kvh, block_size),
                            dtype)
            V = bits_to_f64(gather_sequence(v_cache_bits, block_tables[s], ctx, kvh, block_size),
                            dtype)
            cache = {key: (K, V)}
        K, V = cache[key]
        out[s, h] = softmax_attention(bits_to_f64(q_bits[s, h], dtype), K, V, scale)
    return out


def partition_state(q, K, V, scale: float):
    """``(m, l, acc)`` of one split-KV partition (float64)."""
    x = scale * (np.asarray(K, np.float64) @ np.asarray(q, np.float64))
    m = x.max()
    p = np.exp(x - m)
    return m, p.sum(), p @ np.asarray(V, np.float64)


def merge_states(states) -> np.ndarray:
    """Combine partition states into the normalised attention output."""
    ms = np.array([s[0] for s in states], dtype=np.float64)
    M = ms.max()
    w = np.exp(ms - M)
    L = sum(wi * s[1] for wi, s in zip(w, states))
    acc = sum(wi * s[2] for wi, s in zip(w, states))
    return acc / L


def split_kv_attention(q, K, V, scale: float, partition_tokens: int) -> np.ndarray:
    """Attention computed as independent partitions of ``partition_tokens`` tokens, merged."""
    n = K.shape[0]
    if n == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    states = [partition_state(q, K[b:b + partition_tokens], V[b:b + partition_tokens], scale)
              for b in range(0, n, partition_tokens)]
    return merge_states(states)
