"""Pins the oracle to things other than itself (CPU only).

Each ``pin_*`` function checks the oracle against something the pages or the
mathematics fix: the 70-token worked example and the block-table figure
(golden fixtures), closed forms worked by hand, brute force on tiny inputs, a
library attention routine (PyTorch's scaled_dot_product_attention in float64
on the CPU), and invariants the pages state (waste below one block, no
external fragmentation, sharing invisible to the result). ``test_planted_*``
then plants plausible mistakes in the oracle and checks that some pin fails.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import block_manager as BMmod
from oracle import cache_ops as C
from oracle import step as S
from oracle.fpbits import bits_to_f64
import workloads
from workloads import gen

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _golden(name):
    import json
    import os
    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", name)
    with open(here) as f:
        return json.load(f)


def _bf(x):
    """Round float64 test values to half bits (exact for the small values used)."""
    return np.asarray(x, np.float64).astype(np.float16).view(np.uint16)


# --------------------------------------------------------------------------
# block manager
# --------------------------------------------------------------------------

def pin_seventy_tokens():
    g = _golden("seventy_tokens.json")
    bm = BMmod.BlockManager(64, g["block_size"])
    slots = bm.add_seq(7, g["tokens"])
    table = bm.table(7)
    assert len(table) == g["blocks"]
    bs = g["block_size"]
    per_block = [sum(1 for s in slots if s // bs == b) for b in table]
    assert per_block[:-1] == [bs] * g["full_blocks"]
    assert per_block[-1] == g["last_block_used"]
    assert len(table) * bs - g["tokens"] <= g["max_waste_per_request"]
    assert bm.num_free() == 64 - g["blocks"]


def pin_block_table_figure():
    """Rebuild the figure's pool with ordinary operations: A and B grow block by
    block, interleaved with two short requests that finish and hand their blocks
    back, which leaves B3 and B5 empty."""
    g = _golden("block_table_figure.json")
    bs = g["block_size"]
    bm = BMmod.BlockManager(g["pool_blocks"], bs)
    A_, B_, C_, D_ = 10, 11, 12, 13
    bm.add_seq(A_, bs)            # A-1
    bm.add_seq(B_, bs)            # B-1
    bm.append_slots(A_, bs)       # A-2
    bm.add_seq(C_, bs)            # short request
    bm.append_slots(B_, bs)       # B-2
    bm.add_seq(D_, bs)            # short request
    bm.append_slots(A_, bs)       # A-3
    bm.append_slots(B_, bs)       # B-3
    bm.free_seq(C_)
    bm.free_seq(D_)
    assert bm.table(A_) == g["tables"]["A"]
    assert bm.table(B_) == g["tables"]["B"]
    assert sorted(bm.free_list()) == g["free"]
    occ = [None] * g["pool_blocks"]
    for name, sid in (("A", A_), ("B", B_)):
        for i, b in enumerate(bm.table(sid)):
            occ[b] = f"{name}-{i + 1}"
    assert occ == g["occupancy"]


def pin_slot_numbering():
    """Slot of position p = table[p // 16] * 16 + p % 16, checked on literals."""
    bm = BMmod.BlockManager(8, 16, [5, 2, 7, 0, 1, 3, 4, 6])
    slots = bm.add_seq(1, 18)
    assert bm.table(1) == [5, 2]
    assert slots[0] == 80 and slots[15] == 95 and slots[16] == 32 and slots[17] == 33
    s, pairs = bm.append_slots(1, 15)
    assert pairs == [] and s[0] == 2 * 16 + 2      # position 18: offset 2 of block 2
    assert bm.table(1) == [5, 2, 7]
    assert s[-1] == 7 * 16 + 0  # position 32 is offset 0 of the third block


def pin_lifo_reuse_and_release_order():
    bm = BMmod.BlockManager(6, 16, [3, 1, 4, 0, 5, 2])
    bm.add_seq(1, 40)   # takes 3, 1, 4
    assert bm.table(1) == [3, 1, 4]
    bm.free_seq(1)      # releases 4, 1, 3 (last logical block first) -> 3 on top
    assert bm.free_list() == [3, 1, 4, 0, 5, 2]
    bm.add_seq(2, 17)
    assert bm.table(2) == [3, 1]


def pin_copy_on_write():
    bm = BMmod.BlockManager(16, 16)
    bm.add_seq(0, 20)                    # blocks 0, 1; block 1 holds 4 tokens
    bm.fork(0, 1)
    bm.fork(0, 2)
    assert [bm.refcount(b) for b in (0, 1)] == [3, 3]
    s, pairs = bm.append_slots(1, 1)     # writes into shared partial block -> copy
    assert pairs == [(1, 2)] and bm.table(1) == [0, 2] and s == [2 * 16 + 4]
    assert bm.refcount(1) == 2 and bm.refcount(2) == 1
    s, pairs = bm.append_slots(2, 1)
    assert pairs == [(1, 3)] and bm.table(2) == [0, 3]
    s, pairs = bm.append_slots(0, 1)     # last holder writes in place
    assert pairs == [] and s == [1 * 16 + 4] and bm.refcount(1) == 1
    # A shared block that is full is never copied: the next token opens a new block.
    bm.add_seq(5, 32)
    bm.fork(5, 6)
    s, pairs = bm.append_slots(6, 1)
    assert pairs == [] and len(bm.table(6)) == 3 and bm.table(6)[:2] == bm.table(5)
    # Freeing the fork drops refcounts back without freeing shared blocks.
    bm.free_seq(6)
    assert all(bm.refcount(b) == 1 for b in bm.table(5))


def pin_all_or_nothing():
    bm = BMmod.BlockManager(4, 16)
    bm.add_seq(0, 40)
    snap = (bm.free_list(), bm.table(0), bm.seq_len(0), [bm.refcount(b) for b in range(4)])
    with pytest.raises(BMmod.BlockManagerError) as e:
        bm.append_slots(0, 30)            # needs 2 more blocks, 1 free
    assert e.value.code == BMmod.ERR_NO_FREE_BLOCKS
    with pytest.raises(BMmod.BlockManagerError):
        bm.add_seq(1, 17)
    assert snap == (bm.free_list(), bm.table(0), bm.seq_len(0),
                    [bm.refcount(b) for b in range(4)])
    bm.fork(0, 1)                         # last block shared, partly filled
    with pytest.raises(BMmod.BlockManagerError):
        bm.append_slots(1, 9)             # copy (1) + new block (1) > 1 free
    assert bm.table(1) == bm.table(0)


def _check_invariants(bm, nb, bs):
    used = {}
    for sid in bm.seq_ids():
        t = bm.table(sid)
        n = bm.seq_len(sid)
        assert len(t) == -(-n // bs)
        assert len(t) * bs - n <= bs - 1        # waste within one block
        for b in t:
            used[b] = used.get(b, 0) + 1
    for b in range(nb):
        assert bm.refcount(b) == used.get(b, 0)  # refcounts = number of tables holding it
    assert bm.num_free() + len(used) == nb        # every block is free or in use
    assert sorted(set(bm.free_list())) == sorted(bm.free_list())
    assert not set(bm.free_list()) & set(used)


def pin_invariants_random_ops():
    rng = np.random.default_rng(11)
    nb, bs = 96, 16
    bm = BMmod.BlockManager(nb, bs, rng.permutation(nb))
    live, next_id = [], 0
    for _ in range(600):
        op = rng.integers(0, 4)
        try:
            if op == 0 or not live:
                bm.add_seq(next_id, int(rng.integers(0, 60)))
                live.append(next_id)
                next_id += 1
            elif op == 1:
                parent = live[rng.integers(len(live))]
                bm.fork(parent, next_id)
                live.append(next_id)
                next_id += 1
            elif op == 2:
                sid = live[rng.integers(len(live))]
                before = bm.table(sid)
                slots, pairs = bm.append_slots(sid, int(rng.integers(1, 20)))
                assert len(pairs) <= 1
                if pairs:
                    assert pairs[0][0] == before[-1]
            else:
                sid = live.pop(rng.integers(len(live)))
                bm.free_seq(sid)
        except BMmod.BlockManagerError as e:
            assert e.code == BMmod.ERR_NO_FREE_BLOCKS
            if op in (0, 1):
                pass
        _check_invariants(bm, nb, bs)


def pin_no_two_writers_share_a_slot():
    """After copy-on-write, slots handed out in one round never collide."""
    rng = np.random.default_rng(5)
    bm = BMmod.BlockManager(256, 16, rng.permutation(256))
    bm.add_seq(0, 37)
    for c in range(1, 8):
        bm.fork(0, c)
    seen = set()
    for c in range(8):
        slots, _ = bm.append_slots(c, int(rng.integers(1, 30)))
        assert not seen & set(slots)
        seen |= set(slots)


def pin_swap_bookkeeping():
    bm = BMmod.BlockManager(8, 16, [3, 1, 4, 0, 5, 2, 7, 6])
    bm.set_host_pool(5)
    bm.add_seq(1, 40)                     # blocks 3, 1, 4
    bm.fork(1, 2)                         # shared
    pairs = bm.swap_out(1)
    assert pairs == [(3, 0), (1, 1), (4, 2)] and bm.is_swapped(1)
    assert bm.table(2) == [3, 1, 4] and all(bm.refcount(b) == 1 for b in (3, 1, 4))
    assert bm.num_free() == 5 and bm.num_free_host() == 2 and bm.seq_len(1) == 40
    for op in (lambda: bm.append_slots(1, 1), lambda: bm.fork(1, 9), lambda: bm.swap_out(1),
               lambda: bm.block_tables([1], 4)):
        with pytest.raises(BMmod.BlockManagerError) as e:
            op()
        assert e.value.code == BMmod.ERR_SEQ_SWAPPED
    with pytest.raises(BMmod.BlockManagerError) as e:
        bm.swap_in(2)                     # resident
    assert e.value.code == BMmod.ERR_SEQ_SWAPPED
    bm.free_seq(2)                        # releases 4, 1, 3 (last first) -> 3 on top
    pairs = bm.swap_in(1)
    assert pairs == [(0, 3), (1, 1), (2, 4)] and not bm.is_swapped(1)
    assert bm.num_free_host() == 5 and bm.host_free_list() == [0, 1, 2, 3, 4]
    # host pool exhaustion leaves everything unchanged
    bm.add_seq(5, 80)                     # 5 blocks -> 0 device blocks left
    with pytest.raises(BMmod.BlockManagerError) as e:
        bm.swap_out(5) if bm.num_free_host() < 5 else (bm.set_host_pool(0), bm.swap_out(5))
    assert e.value.code in (BMmod.ERR_NO_FREE_BLOCKS, BMmod.ERR_INVALID_ARG)
    assert not bm.is_swapped(5) and len(bm.table(5)) == 5


def pin_swap_round_trip():
    """Swap out, let another sequence overwrite the freed blocks, swap in: the
    sequence's logical keys/values and its decode output are unchanged."""
    rng = np.random.default_rng(17)
    nb, hkv, d = 12, 2, 8
    kc = gen.f32_to_bits(rng.standard_normal((nb, hkv, 16, d)).astype(np.float32), "f16")
    vc = gen.f32_to_bits(rng.standard_normal((nb, hkv, 16, d)).astype(np.float32), "f16")
    hk = np.zeros((6, hkv, 16, d), np.uint16)
    hv = np.zeros_like(hk)
    q = gen.f32_to_bits(rng.standard_normal((1, hkv, d)).astype(np.float32), "f16")
    bm = BMmod.BlockManager(nb, 16, rng.permutation(nb))
    bm.set_host_pool(6)
    bm.add_seq(0, 37)
    before_k = A.gather_sequence(kc, bm.table(0), 37, 1, 16).copy()
    before = A.paged_decode(q, kc, vc, bm.block_tables([0], 3), [37], 0.3, "f16")
    C.swap_blocks(kc, vc, hk, hv, bm.swap_out(0))
    bm.add_seq(1, 16 * nb)                 # takes every device block, including the freed ones
    noise = gen.f32_to_bits(rng.standard_normal((16 * nb, hkv, d)).astype(np.float32), "f16")
    C.reshape_and_cache(kc, vc, noise, noise, list(range(16 * nb)), 16)
    bm.free_seq(1)
    C.swap_blocks(hk, hv, kc, vc, bm.swap_in(0))
    assert np.array_equal(A.gather_sequence(kc, bm.table(0), 37, 1, 16), before_k)
    after = A.paged_decode(q, kc, vc, bm.block_tables([0], 3), [37], 0.3, "f16")
    assert np.array_equal(before, after)


def pin_prefix_cache_hits():
    bm = BMmod.BlockManager(32, 16)
    P = list(range(100, 140))                       # 40 tokens: 2 full blocks + 8
    s1, c1 = bm.add_seq_cached(1, P)
    assert c1 == 0 and bm.num_cached() == 2
    s2, c2 = bm.add_seq_cached(2, P)
    assert c2 == 32 and bm.table(2)[:2] == bm.table(1)[:2] and bm.table(2)[2] != bm.table(1)[2]
    assert s2[:32] == s1[:32] and s2[32:] != s1[32:]
    assert [bm.refcount(b) for b in bm.table(1)[:2]] == [2, 2]
    _, c3 = bm.add_seq_cached(3, P[:16] + list(range(7, 30)))
    assert c3 == 16 and bm.table(3)[0] == bm.table(1)[0] and bm.table(3)[1] != bm.table(1)[1]
    _, c4 = bm.add_seq_cached(4, [5] + P[1:])        # first block differs: no hit at all
    assert c4 == 0
    _, c5 = bm.add_seq_cached(5, P[:15])             # no full block
    assert c5 == 0 and bm.num_cached() == 2 + 1 + 2


def pin_prefix_cache_eviction_is_exact():
    """Freed cached blocks stay reusable; when evicted (oldest first) their cached
    descendants go too, so a reused block id never matches a stale key."""
    bm = BMmod.BlockManager(6, 16)
    A = list(range(32))                              # 2 full blocks
    bm.add_seq_cached(1, A)
    a0, a1 = bm.table(1)
    bm.free_seq(1)
    assert bm.num_free() == 6 and bm.evictable_list() == [a1, a0]
    _, c = bm.add_seq_cached(2, A)                   # revived from the evictable list
    assert c == 32 and bm.table(2) == [a0, a1]
    bm.free_seq(2)
    bm.add_seq(3, 16 * 4)                            # takes the 4 free blocks
    bm.add_seq(4, 16)                                # evicts the oldest released: a1
    assert bm.table(4) == [a1] and bm.num_cached() == 1
    bm.free_seq(3)
    bm.free_seq(4)
    # a0 is evicted next and then reused for different tokens B; the old child key
    # (a0, A[16:]) must not match B followed by A[16:]
    bm.add_seq(5, 16 * 5)                            # every free block: evicts a0 last
    bm.free_seq(5)
    B = list(range(500, 516)) + A[16:]
    _, c = bm.add_seq_cached(6, B)
    assert c == 0
    bm2 = BMmod.BlockManager(3, 16)
    bm2.add_seq_cached(1, A)                         # a0 -> a1 cached
    p0, p1 = bm2.table(1)
    bm2.free_seq(1)                                  # evictable: [p1, p0]
    bm2.add_seq(2, 16)                               # free block
    bm2.add_seq(3, 16)                               # evicts p1 (a leaf)
    bm2.free_seq(2)
    bm2.free_seq(3)
    bm2.add_seq(4, 48)                               # needs p0 too: evicted with descendants
    bm2.free_seq(4)
    _, c = bm2.add_seq_cached(5, list(range(900, 916)) + A[16:])
    assert c == 0 and bm2.num_cached() == 2          # only the new request's own blocks


def pin_prefix_cache_decode():
    """A request reading a cached prefix equals attention over its own tokens."""
    rng = np.random.default_rng(8)
    nb, hkv, d = 16, 2, 8
    kc = np.zeros((nb, hkv, 16, d), np.uint16)
    vc = np.zeros_like(kc)
    bm = BMmod.BlockManager(nb, 16, rng.permutation(nb))
    prompt = list(range(40))
    kv = gen.f32_to_bits(rng.standard_normal((2, 60, hkv, d)).astype(np.float32), "f16")
    slots, c = bm.add_seq_cached(1, prompt)
    C.reshape_and_cache(kc, vc, kv[0, :40], kv[1, :40], slots, 16)
    tail = list(range(40)) + [77] * 12                 # same 40 tokens, then 12 of its own
    slots2, c2 = bm.add_seq_cached(2, tail)
    assert c2 == 32
    own_k = np.concatenate([kv[0, :32], kv[0, 40:60]])   # token 32.. are the request's own
    own_v = np.concatenate([kv[1, :32], kv[1, 40:60]])
    C.reshape_and_cache(kc, vc, own_k[32:], own_v[32:], slots2[32:], 16)
    q = gen.f32_to_bits(rng.standard_normal((1, hkv, d)).astype(np.float32), "f16")
    out = A.paged_decode(q, kc, vc, bm.block_tables([2], 4), [52], 0.4, "f16")
    for h in range(hkv):
        ref = A.softmax_attention(bits_to_f64(q[0, h], "f16"), bits_to_f64(own_k[:, h], "f16"),
                                  bits_to_f64(own_v[:, h], "f16"), 0.4)
        np.testing.assert_allclose(out[0, h], ref, rtol=1e-14, atol=0)


# --------------------------------------------------------------------------
# cache writes and block copies
# --------------------------------------------------------------------------

def pin_reshape_and_cache_layout():
    nb, hkv, bs, d = 3, 2, 16, 4
    kc = np.zeros((nb, hkv, bs, d), np.uint16)
    vc = np.zeros_like(kc)
    key = np.arange(1, 1 + 3 * hkv * d, dtype=np.uint16).reshape(3, hkv, d)
    val = key + np.uint16(1000)
    C.reshape_and_cache(kc, vc, key, val, [37, -1, 0], bs)
    flat_k, flat_v = kc.reshape(-1), vc.reshape(-1)
    # slot 37 = block 2, offset 5; head 1 starts at ((2*2+1)*16+5)*4 = 340
    assert list(flat_k[340:344]) == list(key[0, 1])
    assert list(flat_k[((2 * 2 + 0) * 16 + 5) * 4:][:4]) == list(key[0, 0])
    assert list(flat_v[340:344]) == list(val[0, 1])
    # slot 0 = block 0, offset 0: heads at flat 0 and 16*4
    assert list(flat_k[0:4]) == list(key[2, 0]) and list(flat_k[64:68]) == list(key[2, 1])
    written = {*range(340, 344), *range(276, 280), *range(0, 4), *range(64, 68)}
    others = [i for i in range(flat_k.size) if i not in written]
    assert not flat_k[others].any() and not flat_v[others].any()   # token 1 (slot -1) skipped


def pin_copy_blocks():
    rng = np.random.default_rng(3)
    kc = rng.integers(0, 65535, (5, 2, 16, 8), dtype=np.uint16)
    vc = rng.integers(0, 65535, (5, 2, 16, 8), dtype=np.uint16)
    k0, v0 = kc.copy(), vc.copy()
    C.copy_blocks(kc, vc, [(0, 3), (4, 1)])
    assert (kc[3] == k0[0]).all() and (kc[1] == k0[4]).all()
    assert (vc[3] == v0[0]).all() and (vc[1] == v0[4]).all()
    for b in (0, 2, 4):
        assert (kc[b] == k0[b]).all() and (vc[b] == v0[b]).all()


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def pin_bits_decode():
    # half: 1.0 = 0x3C00, -2.0 = 0xC000, smallest subnormal = 2**-24
    assert list(bits_to_f64(np.array([0x3C00, 0xC000, 0x0001], np.uint16), "f16")) == \
        [1.0, -2.0, 2.0 ** -24]
    # bfloat16: 1.0 = 0x3F80, -0.5 = 0xBF00, 3.0 = 0x4040, 2**-133 = 0x0001 (subnormal)
    assert list(bits_to_f64(np.array([0x3F80, 0xBF00, 0x4040, 0x0001], np.uint16), "bf16")) == \
        [1.0, -0.5, 3.0, 2.0 ** -133]


def pin_closed_forms():
    for case in _golden("closed_form_decode.json")["cases"]:
        out = A.softmax_attention(case["q"], np.array(case["K"]), np.array(case["V"]),
                                  case["scale"])
        np.testing.assert_allclose(out, case["out"], rtol=1e-14, atol=1e-14)


def pin_special_cases():
    rng = np.random.default_rng(0)
    d = 8
    q, k, v = rng.standard_normal(d), rng.standard_normal((1, d)), rng.standard_normal((1, d))
    assert (A.softmax_attention(q, k, v, 0.3) == v[0]).all()          # one token: out = v
    K = np.stack([k[0], k[0]])
    V = rng.standard_normal((2, d))
    np.testing.assert_allclose(A.softmax_attention(q, K, V, 0.3), V.mean(0), rtol=1e-14)
    K = rng.standard_normal((9, d))
    V = rng.standard_normal((9, d))
    np.testing.assert_allclose(A.softmax_attention(np.zeros(d), K, V, 0.3), V.mean(0),
                               rtol=1e-13, atol=1e-15)
    assert (A.softmax_attention(q, np.zeros((0, d)), np.zeros((0, d)), 0.3) == 0).all()
    # A dominant key picks its value row.
    K[4] = 40 * q
    np.testing.assert_allclose(A.softmax_attention(q, K, V, 1.0), V[4], rtol=1e-12, atol=1e-12)


def pin_brute_force_tiny():
    rng = np.random.default_rng(1)
    for n in (1, 2, 3, 5):
        d = 3
        q = rng.standard_normal(d)
        K = rng.standard_normal((n, d))
        V = rng.standard_normal((n, d))
        scale = 0.7
        w = [math.exp(scale * sum(q[i] * K[t][i] for i in range(d))) for t in range(n)]
        z = sum(w)
        ref = [sum(w[t] * V[t][i] for t in range(n)) / z for i in range(d)]
        np.testing.assert_allclose(A.softmax_attention(q, K, V, scale), ref, rtol=1e-13)


def _contiguous_case(B, Hq, Hkv, d, ctx, seed, dtype="f16"):
    """Caches where sequence s owns consecutive blocks in order (identity mapping)."""
    bs = 16
    nblk = [-(-c // bs) for c in ctx]
    nb = sum(nblk)
    kc = np.zeros((nb, Hkv, bs, d), np.uint16)
    vc = np.zeros_like(kc)
    tables = np.full((B, max(nblk)), -1, np.int32)
    logical = []
    base = 0
    for s in range(B):
        kb = gen.normal_bits([seed, s, 0], (ctx[s], Hkv, d), dtype)
        vb = gen.normal_bits([seed, s, 1], (ctx[s], Hkv, d), dtype)
        for t in range(ctx[s]):
            kc[base + t // bs, :, t % bs] = kb[t]
            vc[base + t // bs, :, t % bs] = vb[t]
        tables[s, :nblk[s]] = np.arange(base, base + nblk[s])
        base += nblk[s]
        logical.append((kb, vb))
    q = gen.normal_bits([seed, 99], (B, Hq, d), dtype)
    return q, kc, vc, tables, logical


def pin_library_attention():
    """Identity mapping + contiguous blocks reduce to ordinary attention; compare with
    PyTorch's scaled_dot_product_attention (float64, CPU, grouped-query heads)."""
    B, Hq, Hkv, d = 3, 8, 2, 16
    ctx = [1, 33, 70]
    for dtype in ("f16", "bf16"):
        q, kc, vc, tables, logical = _contiguous_case(B, Hq, Hkv, d, ctx, 7, dtype)
        scale = 1 / math.sqrt(d)
        out = A.paged_decode(q, kc, vc, tables, np.array(ctx), scale, dtype)
        for s in range(B):
            qt = torch.from_numpy(bits_to_f64(q[s], dtype))[None, :, None, :]      # [1,Hq,1,d]
            kt = torch.from_numpy(bits_to_f64(logical[s][0], dtype)).permute(1, 0, 2)[None]
            vt = torch.from_numpy(bits_to_f64(logical[s][1], dtype)).permute(1, 0, 2)[None]
            ref = torch.nn.functional.scaled_dot_product_attention(
                qt, kt, vt, scale=scale, enable_gqa=True)[0, :, 0, :].numpy()
            np.testing.assert_allclose(out[s], ref, rtol=1e-12, atol=1e-12)


def pin_figure_decode():
    """Decoding through the figure's table [0, 2, 6] equals attention over request A's
    contiguous keys and values, whatever sits in the other blocks."""
    g = _golden("block_table_figure.json")
    rng = np.random.default_rng(21)
    bs, d, hkv = g["block_size"], 8, 1
    kc = gen.f32_to_bits(rng.standard_normal((g["pool_blocks"], hkv, bs, d)).astype(np.float32),
                         "f16")
    vc = gen.f32_to_bits(rng.standard_normal((g["pool_blocks"], hkv, bs, d)).astype(np.float32),
                         "f16")
    q = gen.f32_to_bits(rng.standard_normal((1, 1, d)).astype(np.float32), "f16")
    for ctx in (1, 16, 17, 40, 48):
        table = np.array([g["tables"]["A"]], np.int32)
        out = A.paged_decode(q, kc, vc, table, np.array([ctx]), 0.35, "f16")
        Kc = np.concatenate([kc[b, 0] for b in g["tables"]["A"]])[:ctx]
        Vc = np.concatenate([vc[b, 0] for b in g["tables"]["A"]])[:ctx]
        ref = A.softmax_attention(bits_to_f64(q[0, 0], "f16"), bits_to_f64(Kc, "f16"),
                                  bits_to_f64(Vc, "f16"), 0.35)
        np.testing.assert_allclose(out[0, 0], ref, rtol=1e-15, atol=0)


def pin_split_merge():
    rng = np.random.default_rng(4)
    d = 16
    for n in (1, 15, 16, 17, 100, 513):
        q, K, V = rng.standard_normal(d), rng.standard_normal((n, d)), rng.standard_normal((n, d))
        ref = A.softmax_attention(q, K, V, 0.25)
        for p in (16, 32, 64, 512, 1024):
            np.testing.assert_allclose(A.split_kv_attention(q, K, V, 0.25, p), ref,
                                       rtol=1e-12, atol=1e-14)


def pin_placement_invariance():
    """Any permutation of physical placement gives the identical result."""
    wl = workloads.workload("tiny_mha_d64")
    ref = S.decode_step(wl).out
    for seed in (1, 2):
        wl2 = workloads.workload("tiny_mha_d64")
        wl2.free_order = np.random.default_rng(seed).permutation(wl2.num_blocks).astype(np.int32)
        st = S.decode_step(wl2)
        assert not np.array_equal(st.block_tables, S.decode_step(wl).block_tables)
        assert np.array_equal(st.out, ref)


def pin_shared_equals_duplicated():
    wl = workloads.workload("prefix_share_cow", small=True)
    shared = S.shared_prefix_step(wl)
    dup = S.shared_prefix_step(wl, duplicate=True)
    assert len(shared.cow_pairs) > 0 and len(dup.cow_pairs) == 0
    assert shared.bm.num_free() > dup.bm.num_free()          # sharing saves blocks
    assert np.array_equal(shared.out, dup.out)
    # and both equal attention over each sample's logical keys/values
    rows = [(s, h) for s in range(wl.num_seqs) for h in (0, wl.num_q_heads - 1)]
    ref = S.sampled_outputs(wl, rows)
    got = np.stack([shared.out[s, h] for s, h in rows])
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def pin_step_matches_logical():
    """The full-pool step equals attention over each sequence's logical keys/values."""
    for name in ("tiny_mha_d64", "gqa_32_8_bf16"):
        wl = workloads.workload(name, small=True)
        st = S.decode_step(wl)
        rows = [(s, h) for s in range(wl.num_seqs) for h in range(0, wl.num_q_heads, 5)]
        ref = S.sampled_outputs(wl, rows)
        got = np.stack([st.out[s, h] for s, h in rows])
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


# --------------------------------------------------------------------------
# planted mistakes: each must make at least one pin fail
# --------------------------------------------------------------------------

def _fails_some_pin():
    for pin in PINS:
        try:
            pin()
        except (Exception, pytest.fail.Exception):
            return True
    return False


def _softmax_no_scale(q, K, V, scale):
    return _ORIG["softmax_attention"](q, K, V, 1.0)


def _softmax_kv_swapped(q, K, V, scale):
    return _ORIG["softmax_attention"](q, V, K, scale) if np.shape(K) == np.shape(V) else \
        _ORIG["softmax_attention"](q, K, V, scale)


def _gather_transposed(cache_bits, table_row, ctx, kv_head, block_size):
    t = np.arange(ctx)
    blocks = np.asarray(table_row, dtype=np.int64)[np.minimum(t % block_size, len(table_row) - 1)]
    blocks = np.where(blocks < 0, 0, blocks)
    return cache_bits[blocks, kv_head, (t // block_size) % block_size, :]


def _merge_no_rescale(states):
    L = sum(s[1] for s in states)
    return sum(s[2] for s in states) / L


def _paged_decode_gqa_mod(q_bits, k_cache_bits, v_cache_bits, block_tables, context_lens, scale,
                          dtype, block_size=16, rows=None):
    B, Hq, d = q_bits.shape
    Hkv = k_cache_bits.shape[1]
    out = np.zeros((B, Hq, d))
    for s in range(B):
        for h in range(Hq):
            kvh = h % Hkv
            K = bits_to_f64(A.gather_sequence(k_cache_bits, block_tables[s], int(context_lens[s]),
                                              kvh, block_size), dtype)
            V = bits_to_f64(A.gather_sequence(v_cache_bits, block_tables[s], int(context_lens[s]),
                                              kvh, block_size), dtype)
            out[s, h] = A.softmax_attention(bits_to_f64(q_bits[s, h], dtype), K, V, scale)
    return out


_ORIG = {"softmax_attention": A.softmax_attention}


def _fifo_init(self, num_blocks, block_size, initial_free_order=None):
    _ORIG_BM_INIT(self, num_blocks, block_size, initial_free_order)
    self._free = list(reversed(self._free))


def _append_no_cow(self, seq_id, n):
    """append_slots that writes into shared blocks in place (never copies)."""
    self._need(seq_id)
    table = self._tables[seq_id]
    length = self._lens[seq_id]
    bs = self.block_size
    if -(-(length + n) // bs) - len(table) > len(self._free):
        raise BMmod.BlockManagerError(BMmod.ERR_NO_FREE_BLOCKS, "pool exhausted")
    slots = []
    for p in range(length, length + n):
        if p % bs == 0:
            b = self._free.pop()
            self._ref[b] = 1
            table.append(b)
        slots.append(self._slot(table, p))
    self._lens[seq_id] = length + n
    return slots, []


_ORIG_BM_INIT = BMmod.BlockManager.__init__
_ORIG_APPEND = BMmod.BlockManager.append_slots


def _reshape_offset_off_by_one(k_cache, v_cache, key, value, slot_mapping, block_size):
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64).tolist()):
        if slot < 0:
            continue
        block, offset = divmod(slot + 1, block_size)
        if block >= k_cache.shape[0]:
            continue
        k_cache[block, :, offset, :] = key[t]
        v_cache[block, :, offset, :] = value[t]


def _free_first_to_last(self, seq_id):
    self._need(seq_id)
    for b in self._tables[seq_id]:
        self._ref[b] -= 1
        if self._ref[b] == 0:
            self._free.append(b)
    del self._tables[seq_id]
    del self._lens[seq_id]


def _swap_in_reversed(self, seq_id):
    pairs = _ORIG_SWAP_IN(self, seq_id)
    table = self._tables[seq_id]
    table.reverse()
    return [(h, b) for (h, _), b in zip(pairs, table)]


_ORIG_SWAP_IN = BMmod.BlockManager.swap_in


def _no_cache_hits(self, seq_id, token_ids):
    slots = self.add_seq(seq_id, len(list(token_ids)))
    return slots, 0


MISTAKES = {
    "prefix_cache_never_hits": (BMmod.BlockManager, "add_seq_cached", _no_cache_hits),
    "swap_in_reversed": (BMmod.BlockManager, "swap_in", _swap_in_reversed),
    "dropped_scale": (A, "softmax_attention", _softmax_no_scale),
    "k_v_swapped": (A, "softmax_attention", _softmax_kv_swapped),
    "gather_block_offset_transposed": (A, "gather_sequence", _gather_transposed),
    "merge_without_rescale": (A, "merge_states", _merge_no_rescale),
    "gqa_head_modulo": (A, "paged_decode", _paged_decode_gqa_mod),
    "free_list_fifo": (BMmod.BlockManager, "__init__", _fifo_init),
    "no_copy_on_write": (BMmod.BlockManager, "append_slots", _append_no_cow),
    "release_first_to_last": (BMmod.BlockManager, "free_seq", _free_first_to_last),
    "slot_offset_off_by_one": (C, "reshape_and_cache", _reshape_offset_off_by_one),
}


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_planted_mistake_is_caught(name, monkeypatch):
    owner, attr, bad = MISTAKES[name]
    monkeypatch.setattr(owner, attr, bad)
    if owner is A and attr in ("softmax_attention",):
        # step.py imported the name directly; patch it there too
        monkeypatch.setattr(S, attr, bad)
    if owner is A and attr == "paged_decode":
        monkeypatch.setattr(S, attr, bad)
    if owner is C:
        monkeypatch.setattr(S, attr, bad)
    assert _fails_some_pin(), f"planted mistake {name!r} passed every pin"
