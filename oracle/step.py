"""One decode step of a workload, end to end, on the oracle side.

The order of operations is the method's: the block manager hands out slots
as tokens arrive ("Pages, from operating systems"), each token's keys and
values are written into their slot, shared blocks are copied before a
sequence writes into them (copy-on-write), and attention then reads the cache
through the block tables.

Decode workloads (independent sequences): sequence ``s`` first holds its
``ctx_s - 1`` earlier tokens; the step appends one token per sequence, writes
it, and decodes over all ``ctx_s`` tokens.

Shared-prefix workloads: each prompt is registered and written, forked into
its samples, every sample appends its own tokens in index order (collecting
slots and copy pairs), the copy pairs are applied, all appended tokens are
written in one pass, and every sample is decoded.

``full_pool`` steps build the whole pool and are meant for sizes the oracle
finishes in seconds. ``sampled_outputs`` computes chosen outputs of any size
straight from each sequence's logical keys and values (the definition of the
result, independent of where blocks sit).
"""

from __future__ import annotations

import numpy as np

from workloads import gen

from .attention import paged_decode, softmax_attention
from .block_manager import BlockManager
from .cache_ops import copy_blocks, reshape_and_cache
from .fpbits import bits_to_f64


class OracleStep:
    """Everything the oracle produced for one step (host arrays)."""

    def __init__(self):
        self.prefill_slots = None     # int64 [T_prefill]
        self.step_slots = None        # int64 [T_step]
        self.cow_pairs = None         # int64 [n, 2]
        self.block_tables = None      # int32 [B, max_blocks]
        self.k_cache = None           # uint16 [NB, Hkv, bs, d]
        self.v_cache = None
        self.q = None                 # uint16 [B, Hq, d]
        self.out = None               # float64 [B, Hq, d]
        self.bm = None


def _empty_pool(wl):
    shape = (wl.num_blocks, wl.num_kv_heads, wl.block_size, wl.head_dim)
    return np.zeros(shape, np.uint16), np.zeros(shape, np.uint16)


def decode_step(wl, compute_out: bool = True) -> OracleStep:
    """Full-pool oracle step for an independent-sequence decode workload."""
    res = OracleStep()
    bm = BlockManager(wl.num_blocks, wl.block_size, wl.free_order)
    kc, vc = _empty_pool(wl)
    ctx = wl.context_lens.astype(np.int64)
    kv = gen.many_seq_kv_bits(wl.seed, range(wl.num_seqs), ctx, wl.num_kv_heads, wl.head_dim,
                              wl.dtype)
    prefill_slots = []
    for s in range(wl.num_seqs):
        n = int(ctx[s]) - 1
        slots = bm.add_seq(s, n)
        reshape_and_cache(kc, vc, kv[s][0][:n], kv[s][1][:n], slots, wl.block_size)
        prefill_slots += slots
    step_slots = []
    for s in range(wl.num_seqs):
        slots, pairs = bm.append_slots(s, 1)
        assert not pairs
        step_slots += slots
    new_k = np.stack([kv[s][0][int(ctx[s]) - 1] for s in range(wl.num_seqs)])
    new_v = np.stack([kv[s][1][int(ctx[s]) - 1] for s in range(wl.num_seqs)])
    reshape_and_cache(kc, vc, new_k, new_v, step_slots, wl.block_size)
    res.prefill_slots = np.asarray(prefill_slots, np.int64)
    res.step_slots = np.asarray(step_slots, np.int64)
    res.cow_pairs = np.zeros((0, 2), np.int64)
    res.block_tables = bm.block_tables(range(wl.num_seqs), wl.max_blocks_per_seq)
    res.k_cache, res.v_cache = kc, vc
    res.q = gen.query_bits(wl.seed, wl.num_seqs, wl.num_q_heads, wl.head_dim, wl.dtype)
    res.bm = bm
    if compute_out:
        res.out = paged_decode(res.q, kc, vc, res.block_tables, wl.context_lens, wl.scale,
                               wl.dtype, wl.block_size)
    return res


def shared_prefix_step(wl, duplicate: bool = False, compute_out: bool = True) -> OracleStep:
    """Full-pool oracle step for a prompt-forking workload.

    With ``duplicate`` every sample gets private copies of the prompt's blocks
    instead of sharing them (the same logical sequences, no copy-on-write).
    """
    res = OracleStep()
    bm = BlockManager(wl.num_blocks, wl.block_size, wl.free_order)
    kc, vc = _empty_pool(wl)
    S, P, L = wl.samples, wl.num_prompts, wl.prompt_len
    prompts = gen.many_seq_kv_bits(wl.seed, range(P), [L] * P, wl.num_kv_heads, wl.head_dim,
                                   wl.dtype)
    prefill_slots = []
    for p in range(P):
        owners = [p * S + i for i in range(S)] if duplicate else [p * S]
        for seq in owners:
            slots = bm.add_seq(seq, L)
            reshape_and_cache(kc, vc, prompts[p][0], prompts[p][1], slots, wl.block_size)
            prefill_slots += slots
        if not duplicate:
            for i in range(1, S):
                bm.fork(p * S, p * S + i)
    step_slots, pairs, ks, vs = [], [], [], []
    for seq in range(P * S):
        n = int(wl.own_lens[seq])
        if n == 0:
            continue
        slots, cow = bm.append_slots(seq, n)
        k, v = gen.own_token_kv_bits(wl.seed, seq, n, wl.num_kv_heads, wl.head_dim, wl.dtype)
        step_slots += slots
        pairs += cow
        ks.append(k)
        vs.append(v)
    pairs = np.asarray(pairs, np.int64).reshape(-1, 2)
    copy_blocks(kc, vc, pairs)
    if ks:
        reshape_and_cache(kc, vc, np.concatenate(ks), np.concatenate(vs), step_slots,
                          wl.block_size)
    res.prefill_slots = np.asarray(prefill_slots, np.int64)
    res.step_slots = np.asarray(step_slots, np.int64)
    res.cow_pairs = pairs
    res.block_tables = bm.block_tables(range(P * S), wl.max_blocks_per_seq)
    res.k_cache, res.v_cache = kc, vc
    res.q = gen.query_bits(wl.seed, wl.num_seqs, wl.num_q_heads, wl.head_dim, wl.dtype)
    res.bm = bm
    if compute_out:
        res.out = paged_decode(res.q, kc, vc, res.block_tables, wl.context_lens, wl.scale,
                               wl.dtype, wl.block_size)
    return res


def oracle_step(wl, **kw) -> OracleStep:
    if wl.kind == "shared_prefix":
        return shared_prefix_step(wl, **kw)
    return decode_step(wl, **kw)


def logical_kv_bits(wl, seq: int):
    """The keys and values sequence ``seq`` holds at decode time, in token order."""
    if wl.kind == "shared_prefix":
        p = seq // wl.samples
        pk, pv = gen.seq_kv_bits(wl.seed, p, wl.prompt_len, wl.num_kv_heads, wl.head_dim,
                                 wl.dtype)
        n = int(wl.own_lens[seq])
        ok, ov = gen.own_token_kv_bits(wl.seed, seq, n, wl.num_kv_heads, wl.head_dim, wl.dtype)
        return np.concatenate([pk, ok]), np.concatenate([pv, ov])
    ctx = int(wl.context_lens[seq])
    return gen.seq_kv_bits(wl.seed, seq, ctx, wl.num_kv_heads, wl.head_dim, wl.dtype)


def sampled_outputs(wl, rows, q_bits=None) -> np.ndarray:
    """Float64 outputs for the chosen ``(seq, q_head)`` rows, from logical K/V."""
    if q_bits is None:
        q_bits = gen.query_bits(wl.seed, wl.num_seqs, wl.num_q_heads, wl.head_dim, wl.dtype)
    G = wl.num_q_heads // wl.num_kv_heads
    out = np.zeros((len(rows), wl.head_dim), np.float64)
    by_seq: dict = {}
    for i, (s, h) in enumerate(rows):
        by_seq.setdefault(s, []).append((i, h))
    for s, items in by_seq.items():
        kb, vb = logical_kv_bits(wl, s)
        for i, h in items:
            kvh = h // G
            K = bits_to_f64(kb[:, kvh, :], wl.dtype)
            V = bits_to_f64(vb[:, kvh, :], wl.dtype)
            out[i] = softmax_attention(bits_to_f64(q_bits[s, h], wl.dtype), K, V, wl.scale)
    return out
