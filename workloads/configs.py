"""The decode workloads: shapes, context-length mixes and seeded block placement.

Five workloads are described here, each named by what it is:

* ``tiny_mha_d64``       4 sequences with contexts {1, 16, 17, 70}, 4 heads, head_dim 64,
                         fp16, a 32-block pool.
* ``mha_7b_fp16``        64 sequences, 32 query = 32 KV heads, head_dim 128, fp16, contexts
                         uniform in [128, 2048], a 16384-block pool; one new token per sequence
                         is written to the cache in the same step.
* ``gqa_32_8_bf16``      256 sequences, 32 query / 8 KV heads, head_dim 128, bf16, contexts
                         lognormal(6.5, 0.8) rounded and clipped to [16, 4096], 65536 blocks.
* ``prefix_share_cow``   16 prompts of 1000 tokens, each forked into 8 samples that share the
                         prompt's blocks and append U[0, 200] tokens of their own; 32 heads,
                         head_dim 128, fp16.
* ``long_ctx_split_kv``  8 sequences with contexts uniform in [32768, 131072], 64 query / 8 KV
                         heads, head_dim 128, bf16, a pool sized to fit, 512-token split-KV
                         partitions.

Physical placement is a seeded permutation of the pool that the block manager
hands out in order, so logically consecutive blocks land far apart in memory.
Context lengths count the token written during the decode step itself.
"""

from __future__ import annotations

import math

import numpy as np

from .gen import STREAM_META, bits_dtype_name

BLOCK_SIZE = 16


class DecodeWorkload:
    """A batch of independent sequences decoded in one step."""

    kind = "decode"

    def __init__(self, name, seed, num_seqs, num_q_heads, num_kv_heads, head_dim, dtype,
                 context_lens, num_blocks, free_order, partition_tokens=0,
                 block_size=BLOCK_SIZE):
        self.name = name
        self.seed = int(seed)
        self.num_seqs = int(num_seqs)
        self.num_q_heads = int(num_q_heads)
        self.num_kv_heads = int(num_kv_heads)
        self.head_dim = int(head_dim)
        self.dtype = bits_dtype_name(dtype)
        self.block_size = int(block_size)
        self.context_lens = np.asarray(context_lens, dtype=np.int32)
        self.num_blocks = int(num_blocks)
        self.free_order = np.asarray(free_order, dtype=np.int32)
        self.partition_tokens = int(partition_tokens)
        self.scale = 1.0 / math.sqrt(self.head_dim)
        assert self.context_lens.shape == (self.num_seqs,)
        assert self.free_order.shape == (self.num_blocks,)

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def max_blocks_per_seq(self) -> int:
        return max(1, -(-self.max_context_len // self.block_size))

    @property
    def elem_bytes(self) -> int:
        return 2

    def kv_token_bytes(self) -> int:
        """Bytes of K plus V for one token across all KV heads."""
        return 2 * self.num_kv_heads * self.head_dim * self.elem_bytes

    def describe(self) -> dict:
        return {
            "workload": self.name,
            "num_seqs": self.num_seqs,
            "num_q_heads": self.num_q_heads,
            "num_kv_heads": self.num_kv_heads,
            "head_dim": self.head_dim,
            "dtype": self.dtype,
            "block_size": self.block_size,
            "num_blocks": self.num_blocks,
            "sum_context": int(self.context_lens.astype(np.int64).sum()),
            "max_context": self.max_context_len,
            "partition_tokens": self.partition_tokens,
            "seed": self.seed,
        }


class SharedPrefixWorkload(DecodeWorkload):
    """Prompts forked into parallel samples that share the prompt's blocks.

    Sequence ``p * samples + i`` is sample ``i`` of prompt ``p``; sample 0 is the
    prompt's own sequence and samples 1.. are forks of it. After forking, the
    samples append their own tokens one sample at a time, in index order.
    """

    kind = "shared_prefix"

    def __init__(self, name, seed, num_prompts, samples, prompt_len, own_lens, num_q_heads,
                 num_kv_heads, head_dim, dtype, num_blocks, free_order, partition_tokens=0):
        self.num_prompts = int(num_prompts)
        self.samples = int(samples)
        self.prompt_len = int(prompt_len)
        self.own_lens = np.asarray(own_lens, dtype=np.int32)
        assert self.own_lens.shape == (self.num_prompts * self.samples,)
        ctx = self.prompt_len + self.own_lens
        super().__init__(name, seed, self.num_prompts * self.samples, num_q_heads, num_kv_heads,
                         head_dim, dtype, ctx, num_blocks, free_order, partition_tokens)

    def describe(self) -> dict:
        d = super().describe()
        d.update(num_prompts=self.num_prompts, samples=self.samples, prompt_len=self.prompt_len,
                 sum_own=int(self.own_lens.sum()))
        return d


def _meta_rng(seed):
    return np.random.default_rng([seed, STREAM_META])


def tiny_mha_d64(seed=3521):
    rng = _meta_rng(seed)
    nb = 32
    return DecodeWorkload("tiny_mha_d64", seed, 4, 4, 4, 64, "f16", [1, 16, 17, 70], nb,
                          rng.permutation(nb))


def mha_7b_fp16(seed=3522, num_seqs=64, ctx_lo=128, ctx_hi=2048, num_blocks=16384,
                partition_tokens=0, name="mha_7b_fp16"):
    rng = _meta_rng(seed)
    ctx = rng.integers(ctx_lo, ctx_hi + 1, size=num_seqs)
    return DecodeWorkload(name, seed, num_seqs, 32, 32, 128, "f16", ctx, num_blocks,
                          rng.permutation(num_blocks), partition_tokens)


def gqa_32_8_bf16(seed=3523, num_seqs=256, num_blocks=65536, mu=6.5, sigma=0.8, lo=16,
                  hi=4096, partition_tokens=0, name="gqa_32_8_bf16"):
    rng = _meta_rng(seed)
    ctx = np.clip(np.rint(np.exp(rng.normal(mu, sigma, size=num_seqs))), lo, hi).astype(np.int32)
    return DecodeWorkload(name, seed, num_seqs, 32, 8, 128, "bf16", ctx, num_blocks,
                          rng.permutation(num_blocks), partition_tokens)


def prefix_share_cow(seed=3524, num_prompts=16, samples=8, prompt_len=1000, own_hi=200,
                     num_blocks=4096, partition_tokens=0, name="prefix_share_cow"):
    rng = _meta_rng(seed)
    own = rng.integers(0, own_hi + 1, size=num_prompts * samples)
    return SharedPrefixWorkload(name, seed, num_prompts, samples, prompt_len, own, 32, 32, 128,
                                "f16", num_blocks, rng.permutation(num_blocks), partition_tokens)


def long_ctx_split_kv(seed=3525, num_seqs=8, ctx_lo=32768, ctx_hi=131072, partition_tokens=512,
                      num_q_heads=64, num_kv_heads=8, name="long_ctx_split_kv"):
    rng = _meta_rng(seed)
    ctx = rng.integers(ctx_lo, ctx_hi + 1, size=num_seqs)
    nb = int(sum(-(-int(c) // BLOCK_SIZE) for c in ctx))
    return DecodeWorkload(name, seed, num_seqs, num_q_heads, num_kv_heads, 128, "bf16", ctx, nb,
                          rng.permutation(nb), partition_tokens)


# Full-size workloads, in the order they are usually listed.
WORKLOADS = {
    "tiny_mha_d64": tiny_mha_d64,
    "mha_7b_fp16": mha_7b_fp16,
    "gqa_32_8_bf16": gqa_32_8_bf16,
    "prefix_share_cow": prefix_share_cow,
    "long_ctx_split_kv": long_ctx_split_kv,
}

# Reduced versions with the same head layout, dtype and context mix shape, small
# enough for the oracle to check every output in seconds while still spanning
# several blocks, several split-KV partitions and ragged last blocks.
SMALL_WORKLOADS = {
    "tiny_mha_d64": tiny_mha_d64,
    "mha_7b_fp16": lambda: mha_7b_fp16(num_seqs=6, num_blocks=1024, name="mha_7b_fp16_small"),
    "gqa_32_8_bf16": lambda: gqa_32_8_bf16(num_seqs=12, num_blocks=2048,
                                           name="gqa_32_8_bf16_small"),
    "prefix_share_cow": lambda: prefix_share_cow(num_prompts=2, samples=8, prompt_len=200,
                                                 own_hi=40, num_blocks=256,
                                                 name="prefix_share_cow_small"),
    "long_ctx_split_kv": lambda: long_ctx_split_kv(num_seqs=2, ctx_lo=1500, ctx_hi=5000,
                                                   name="long_ctx_split_kv_small"),
}


def truncated(wl, num_seqs: int, num_blocks: int):
    """The first ``num_seqs`` sequences of an independent-sequence workload in a pool
    of ``num_blocks`` blocks (a smaller case with the same per-sequence shapes)."""
    if wl.kind != "decode":
        raise ValueError("only independent-sequence workloads can be truncated")
    ctx = wl.context_lens[:num_seqs]
    need = int(sum(-(-int(c) // wl.block_size) for c in ctx))
    if num_blocks < need:
        raise ValueError(f"{num_blocks} blocks cannot hold {need}")
    order = _meta_rng(wl.seed).permutation(num_blocks)
    return DecodeWorkload(f"{wl.name}[:{num_seqs}]/{num_blocks}blk", wl.seed, num_seqs,
                          wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.dtype, ctx,
                          num_blocks, order, wl.partition_tokens, wl.block_size)


def workload(name: str, small: bool = False):
    table = SMALL_WORKLOADS if small else WORKLOADS
    if name not in table:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(table)}")
    return table[name]()
