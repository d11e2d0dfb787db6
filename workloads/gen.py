"""Seeded random draws, stored as raw 16-bit patterns.

Every tensor is drawn as float32 N(0,1) with NumPy's PCG64 generator and then
rounded to the cache's storage type (IEEE half or bfloat16, round to nearest
even). Values are returned as ``uint16`` bit patterns so that both sides of a
comparison start from the same bits and decode them independently.

Each sequence has its own sub-stream keyed by ``[seed, stream, index]``; a
test can therefore regenerate exactly the keys and values of one sequence
without drawing the whole batch, which is how full-size workloads are checked
on sampled outputs.
"""

from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
import hashlib
import os

import numpy as np

# Sub-stream identifiers inside one workload seed.
STREAM_SEQ_KV = 1      # per-sequence key/value rows (prompt + generated tokens)
STREAM_QUERY = 2       # the decode step's queries
STREAM_OWN_KV = 3      # per-sample tokens appended after a fork (shared-prefix workload)
STREAM_META = 4        # context lengths and block placement
STREAM_REQUEST_KV = 5  # request traces: one key/value row per (request, branch, position)
STREAM_STEP_QUERY = 6  # request traces: one query per (request, sample, step)
STREAM_PREFIX_KV = 7   # request traces with token ids: one key/value row per prompt prefix

_DTYPES = ("f16", "bf16")


def bits_dtype_name(dtype: str) -> str:
    if dtype not in _DTYPES:
        raise ValueError(f"unsupported storage type {dtype!r}; expected one of {_DTYPES}")
    return dtype


def f32_to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to half or bfloat16 (nearest even) and return the bits."""
    bits_dtype_name(dtype)
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    u = x.view(np.uint32)
    # bfloat16 keeps the top 16 bits; add half an ulp plus the tie-break bit.
    # Inputs here are finite normals, so no NaN/overflow special-casing is needed.
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def normal_bits(key, shape, dtype: str, scale: float = 1.0) -> np.ndarray:
    rng = np.random.default_rng(key)
    x = rng.standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return f32_to_bits(x, dtype)


def _threads() -> int:
    try:
        return max(1, min(16, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover - non-Linux
        return max(1, min(16, os.cpu_count() or 1))


def seq_kv_bits(seed: int, seq: int, ntok: int, num_kv_heads: int, head_dim: int, dtype: str):
    """Keys and values of sequence ``seq`` for token positions ``0..ntok-1``.

    Returns two uint16 arrays of shape ``[ntok, num_kv_heads, head_dim]``. The
    key and value rows of one sequence come from one sub-stream (keys first).
    """
    rng = np.random.default_rng([seed, STREAM_SEQ_KV, seq])
    shape = (ntok, num_kv_heads, head_dim)
    k = f32_to_bits(rng.standard_normal(shape, dtype=np.float32), dtype)
    v = f32_to_bits(rng.standard_normal(shape, dtype=np.float32), dtype)
    return k, v


def many_seq_kv_bits(seed: int, seqs, ntoks, num_kv_heads: int, head_dim: int, dtype: str):
    """``seq_kv_bits`` for several sequences, drawn on a thread pool (order kept)."""
    seqs = list(seqs)
    ntoks = list(ntoks)
    with ThreadPoolExecutor(_threads()) as ex:
        return list(ex.map(lambda a: seq_kv_bits(seed, a[0], a[1], num_kv_heads, head_dim, dtype),
                           zip(seqs, ntoks)))


def query_bits(seed: int, num_seqs: int, num_q_heads: int, head_dim: int, dtype: str,
               scale: float = 1.0) -> np.ndarray:
    """Decode-step queries ``[num_seqs, num_q_heads, head_dim]`` as bits."""
    return normal_bits([seed, STREAM_QUERY], (num_seqs, num_q_heads, head_dim), dtype, scale)


def own_token_kv_bits(seed: int, sample: int, ntok: int, num_kv_heads: int, head_dim: int,
                      dtype: str):
    """Keys and values of the tokens a forked sample appends after the shared prompt."""
    rng = np.random.default_rng([seed, STREAM_OWN_KV, sample])
    shape = (ntok, num_kv_heads, head_dim)
    k = f32_to_bits(rng.standard_normal(shape, dtype=np.float32), dtype)
    v = f32_to_bits(rng.standard_normal(shape, dtype=np.float32), dtype)
    return k, v


def request_token_kv_bits(seed: int, request: int, branch: int, position: int,
                          num_kv_heads: int, head_dim: int, dtype: str):
    """Key and value rows ``[num_kv_heads, head_dim]`` of one token of a request
    trace. ``branch`` 0 holds the prompt (shared by every sample); branch
    ``1 + s`` holds the tokens sample ``s`` generates."""
    b = normal_bits([seed, STREAM_REQUEST_KV, request, branch, position],
                    (2, num_kv_heads, head_dim), dtype)
    return b[0], b[1]


def step_query_bits(seed: int, request: int, sample: int, step: int, num_q_heads: int,
                    head_dim: int, dtype: str) -> np.ndarray:
    """The query ``[num_q_heads, head_dim]`` of one sample at one step of a trace."""
    return normal_bits([seed, STREAM_STEP_QUERY, request, sample, step],
                       (num_q_heads, head_dim), dtype)


def prefix_keys(tokens) -> list:
    """A 64-bit key per prompt position identifying the whole prefix up to it (a
    chained BLAKE2b): two prompts share a position's key exactly when they share
    every token up to it, as a model's keys and values would."""
    keys, h = [], b""
    for t in tokens:
        h = hashlib.blake2b(h + int(t).to_bytes(4, "little", signed=True), digest_size=8).digest()
        keys.append(int.from_bytes(h, "little"))
    return keys


class RequestTokens:
    """Memoised token rows of a request trace: position ``p`` of sample ``s`` of
    request ``r`` is a prompt row when ``p < prompt_len[r]``, else sample ``s``'s own.
    A request given its prompt token ids (``prompt_tokens[r]``) draws its prompt
    rows by prefix key, so requests sharing a prompt prefix share those rows."""

    def __init__(self, seed: int, prompt_len: dict, num_kv_heads: int, head_dim: int,
                 dtype: str, prompt_tokens: dict = None):
        self.seed, self.prompt_len = seed, prompt_len
        self.hkv, self.d, self.dtype = num_kv_heads, head_dim, dtype
        self._rows = {}
        self._keys = {r: prefix_keys(t) for r, t in (prompt_tokens or {}).items()
                      if t is not None}

    def row(self, request: int, sample: int, position: int):
        if position < self.prompt_len[request] and request in self._keys:
            k = self._keys[request][position]
            key = ("prefix", k)
            if key not in self._rows:
                b = normal_bits([self.seed, STREAM_PREFIX_KV, k >> 32, k & 0xffffffff, position],
                                (2, self.hkv, self.d), self.dtype)
                self._rows[key] = (b[0], b[1])
            return self._rows[key]
        branch = 0 if position < self.prompt_len[request] else 1 + sample
        key = (request, branch, position)
        if key not in self._rows:
            self._rows[key] = request_token_kv_bits(self.seed, request, branch, position,
                                                    self.hkv, self.d, self.dtype)
        return self._rows[key]

    def rows(self, request: int, sample: int, positions):
        ks, vs = zip(*(self.row(request, sample, p) for p in positions)) if len(positions) else ((), ())
        shape = (0, self.hkv, self.d)
        return (np.stack(ks) if ks else np.zeros(shape, np.uint16),
                np.stack(vs) if vs else np.zeros(shape, np.uint16))
