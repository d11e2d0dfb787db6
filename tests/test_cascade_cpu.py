"""Cascade decode without a GPU: the C++ grouping of a batch into sequences that
share leading blocks (pa_bm_prefix_groups) against the oracle's restatement of
the rule over random fork trees, the invariants every group must satisfy, and
the host-side argument checks of pa_paged_decode_cascade."""

import ctypes

import numpy as np
import pytest

from oracle import block_manager as OBM
import paged_kv_cache_352_b200 as pa
from paged_kv_cache_352_b200 import _lib as L

FAKE = ctypes.c_void_p(4096)  # never dereferenced: every call below fails validation first


def _fork_forest(seed, nb=3000):
    """Random prompts forked into samples that append their own tokens, driven
    through both block managers with one free order. Returns the two managers
    and the batch order (a shuffle of every live sequence)."""
    rng = np.random.default_rng(seed)
    order = rng.permutation(nb).astype(np.int32)
    cbm = pa.BlockManager(nb, 16, order)
    obm = OBM.BlockManager(nb, 16, order.tolist())
    sid = 0
    live = []
    for _ in range(int(rng.integers(2, 9))):
        plen = int(rng.integers(1, 400))
        root = sid
        sid += 1
        for bm in (cbm, obm):
            bm.add_seq(root, plen)
        fam = [root]
        for _ in range(int(rng.integers(0, 12))):
            parent = int(rng.choice(fam))
            child = sid
            sid += 1
            for bm in (cbm, obm):
                bm.fork(parent, child)
            fam.append(child)
        for s in fam:
            n = int(rng.integers(0, 60))
            if n:
                cbm.append_slots(s, n)
                obm.append_slots(s, n)
        live += fam
    batch = [live[i] for i in rng.permutation(len(live))]
    return cbm, obm, batch


@pytest.mark.parametrize("seed", range(12))
@pytest.mark.parametrize("group_size", [2, 3, 4, 5, 8])
def test_prefix_groups_match_oracle(seed, group_size):
    cbm, obm, batch = _fork_forest(seed)
    g = cbm.prefix_groups(batch, group_size)
    members, prefix, sgroup, smember = obm.prefix_groups(batch, group_size)
    assert g.num_groups == len(members)
    for k, run in enumerate(members):
        row = g.members[k].tolist()
        assert row[:len(run)] == run and all(x == -1 for x in row[len(run):])
    assert g.prefix_blocks.tolist() == prefix
    assert g.seq_group.tolist() == sgroup and g.seq_member.tolist() == smember
    assert g.max_prefix_blocks == (max(prefix) if prefix else 0)


@pytest.mark.parametrize("seed", range(12))
def test_prefix_groups_invariants(seed):
    """Every group: 2..group_size members, each named back by seq_group/seq_member,
    all holding the leader's first P blocks as full blocks; no sequence twice."""
    cbm, _, batch = _fork_forest(seed)
    gs = 8
    g = cbm.prefix_groups(batch, gs)
    tables = cbm.block_tables(batch, 64)
    seen = set()
    for k in range(g.num_groups):
        mem = [m for m in g.members[k].tolist() if m >= 0]
        P = int(g.prefix_blocks[k])
        assert 2 <= len(mem) <= gs and P >= 1
        for slot, i in enumerate(mem):
            assert i not in seen
            seen.add(i)
            assert g.seq_group[i] == k and g.seq_member[i] == slot
            assert cbm.seq_len(batch[i]) // 16 >= P
            assert tables[i, :P].tolist() == tables[mem[0], :P].tolist()
    for i in range(len(batch)):
        if i not in seen:
            assert g.seq_group[i] == -1 and g.seq_member[i] == -1


def test_prefix_groups_of_forked_prompt():
    """A 1000-token prompt forked 8 ways, each sample appending: one group over
    the prompt's 62 full blocks (the partly filled 63rd is copied on write)."""
    bm = pa.BlockManager(1024)
    bm.add_seq(0, 1000)
    for c in range(1, 8):
        bm.fork(0, c)
    for c in range(8):
        bm.append_slots(c, 1 + 3 * c)
    g = bm.prefix_groups(range(8), 8)
    assert g.num_groups == 1 and g.prefix_blocks.tolist() == [62]
    assert g.members.tolist() == [list(range(8))]
    h = bm.prefix_groups(range(8), 4)          # runs of 4
    assert h.num_groups == 2 and h.members.tolist() == [[0, 1, 2, 3], [4, 5, 6, 7]]
    solo = bm.prefix_groups([3], 8)            # a lone sequence forms no group
    assert solo.num_groups == 0 and solo.seq_group.tolist() == [-1]


def test_prefix_groups_errors():
    bm = pa.BlockManager(64)
    bm.add_seq(1, 40)
    with pytest.raises(L.PAError):
        bm.prefix_groups([1, 2], 4)            # unknown sequence
    with pytest.raises(L.PAError):
        bm.prefix_groups([1], 0)               # bad group size


def test_cascade_argument_checks():
    lib = L.lib()
    dummy = np.zeros(16, np.int32)

    def call(**kw):
        a = dict(hq=32, hkv=32, d=128, bs=16, B=8, maxctx=1200, mb=76, nb=4096, ng=1, gs=8,
                 mp=62, ws=None, wsb=0, dt=L.PA_F16)
        a.update(kw)
        p = dummy.ctypes.data
        return lib.pa_paged_decode_cascade(
            FAKE, FAKE, FAKE, FAKE, FAKE, a["mb"], FAKE, None, a["B"], a["maxctx"], a["hq"],
            a["hkv"], a["d"], a["bs"], a["nb"], 0.1, p, p, p, p, a["ng"], a["gs"], a["mp"], a["ws"],
            a["wsb"], None, a["dt"], None)

    assert call(gs=3) == L.PA_ERR_UNSUPPORTED            # 3 stacked heads per KV head
    assert call(hq=64, hkv=8, gs=2) == L.PA_ERR_UNSUPPORTED  # 8 x 2 = 16 heads
    assert call(mp=0) == L.PA_ERR_INVALID_ARG            # groups need a prefix bound
    assert call(mp=77) == L.PA_ERR_INVALID_ARG           # bound above the table width
    assert call(d=96) == L.PA_ERR_UNSUPPORTED
    assert call(bs=8) == L.PA_ERR_UNSUPPORTED
    assert call() == L.PA_ERR_INVALID_ARG                # no workspace
    assert "workspace" in L.last_error()
    assert call(B=0) == L.PA_OK                          # nothing to do
    ws = ctypes.c_void_p(256 * 4096)                     # aligned, never dereferenced
    big = 1 << 40
    assert call(ws=ws, wsb=big, hq=32, hkv=16) == L.PA_ERR_UNSUPPORTED  # 8 x 2 stacked heads
    assert call(ws=ctypes.c_void_p(256 * 4096 + 16), wsb=big) == L.PA_ERR_INVALID_ARG
    assert "256-byte" in L.last_error()
    assert call(ws=ws, wsb=1) == L.PA_ERR_INVALID_ARG    # workspace too small
    assert call(ws=ws, wsb=big, dt=7) == L.PA_ERR_UNSUPPORTED
    assert call(ws=ws, wsb=big, ng=-1) == L.PA_ERR_INVALID_ARG
    n = pa.pa_paged_decode_cascade_workspace_size(8, 32, 32, 128, 1200, 76, 1, 8, 62)
    assert n > 0
    assert pa.pa_paged_decode_cascade_workspace_size(8, 32, 32, 128, 1200, 76, 0, 1, 0) < n


def test_cascade_workspace_covers_both_decodes():
    """The workspace holds the stacked queries, both table sets and the partition
    states of both decodes: at least their element counts."""
    B, hq, hkv, d, maxctx, mb, ng, gs, mp = 128, 32, 32, 128, 1208, 76, 16, 8, 62
    n = pa.pa_paged_decode_cascade_workspace_size(B, hq, hkv, d, maxctx, mb, ng, gs, mp)
    gq = ng * hkv * gs * d * 2
    states_g = ng * hkv * gs * (d + 2) * 4             # at least one partition per group
    states_s = B * hkv * 1 * (d + 2) * 4
    tables = (ng + B) * mb * 4
    assert n >= gq + states_g + states_s + tables


def test_prefix_groups_of_empty_and_unshared_batches():
    bm = pa.BlockManager(256)
    g = bm.prefix_groups([], 8)
    assert g.num_groups == 0 and g.max_prefix_blocks == 0 and len(g.seq_group) == 0
    for s, n in ((0, 40), (1, 16), (2, 0), (3, 300)):
        bm.add_seq(s, n)
    g = bm.prefix_groups([3, 0, 2, 1], 8)     # no two sequences share a block
    assert g.num_groups == 0 and g.seq_group.tolist() == [-1] * 4
    assert g.seq_member.tolist() == [-1] * 4
    ws = pa.pa_paged_decode_cascade_workspace_size(4, 8, 8, 64, 300, 19, g.num_groups, 1,
                                                   g.max_prefix_blocks)
    assert ws > 0


def _own_tokens_order(ctx, seq_group, prefix_blocks):
    """The order pa_cascade_order promises, by the rule stated plainly: tokens
    after the group's prefix (whole context outside a group), longest first,
    ties by batch index."""
    own = []
    for i, c in enumerate(ctx):
        g = int(seq_group[i])
        pre = 16 * int(prefix_blocks[g]) if 0 <= g < len(prefix_blocks) else 0
        own.append(max(0, int(c) - pre))
    return sorted(range(len(ctx)), key=lambda i: (-own[i], i))


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_cascade_order_lists_own_blocks_longest_first(seed):
    bm, _, batch = _fork_forest(seed)
    g = bm.prefix_groups(batch, 4)
    ctx = np.array([bm.seq_len(s) for s in batch], np.int32)
    got = pa.pa_cascade_order(ctx, g).tolist()
    assert got == _own_tokens_order(ctx, g.seq_group, g.prefix_blocks)
    assert sorted(got) == list(range(len(batch)))


def test_cascade_order_edge_cases():
    lib = L.lib()
    ctx = np.array([30, 50, 50, 7, 0], np.int32)
    # no groups: plain longest first, ties by index
    g0 = L.PrefixGroups(np.zeros((0, 2), np.int32), np.zeros(0, np.int32),
                        np.full(5, -1, np.int32), np.full(5, -1, np.int32), 2, 0)
    assert pa.pa_cascade_order(ctx, g0).tolist() == [1, 2, 0, 3, 4]
    # a group of sequences 1 and 2 with 3 shared blocks (48 tokens): 2 and 2 own
    # tokens; a group index past num_groups counts as no group; a prefix longer
    # than the context counts as 0 own tokens
    sg = np.array([1, 0, 0, 7, 1], np.int32)
    pb = np.array([3, 4], np.int32)
    g = L.PrefixGroups(np.array([[1, 2], [0, 4]], np.int32), pb, sg,
                       np.array([0, 0, 1, -1, 1], np.int32), 2, 4)
    assert pa.pa_cascade_order(ctx, g).tolist() == _own_tokens_order(ctx, sg, pb)
    assert pa.pa_cascade_order(ctx, g).tolist() == [3, 1, 2, 0, 4]
    out = np.empty(5, np.int32)
    assert lib.pa_cascade_order(ctx.ctypes.data, None, None, 1, 5,
                                out.ctypes.data) == L.PA_ERR_INVALID_ARG
    assert lib.pa_cascade_order(None, None, None, 0, 0, None) == L.PA_OK
    assert lib.pa_cascade_order(ctx.ctypes.data, None, None, 0, -1,
                                out.ctypes.data) == L.PA_ERR_INVALID_ARG


def test_cascade_plan():
    """pa_paged_decode_cascade_plan: a group prefix stays one partition (up to the
    decode's 128-block cap) when groups and sequences together give the GPU
    enough (group or sequence, KV head) pairs, and is split into partitions of
    at least 32 blocks when they do not; launches are 3 for the single-launch
    shapes (8 stacked query heads) and for batches without groups, 4 when the
    two decodes run on two streams, 0 for an empty batch."""
    # 16 prompts forked 8 ways, 62-block prefixes, 32 KV heads: 4608 pairs
    p = L.pa_paged_decode_cascade_plan(128, 32, 32, 128, 1200, 76, 16, 8, 62)
    assert p == {"prefix_part_blocks": 62, "prefix_parts": 1, "own_part_blocks": 75,
                 "own_parts": 1, "launches": 3}
    assert L.pa_paged_decode_cascade_plan(128, 32, 32, 128, 1200, 76, 16, 8, 62, dtype="bf16",
                                          fp8_cache=True)["launches"] == 3
    # a prefix longer than the cap is split at the cap
    p = L.pa_paged_decode_cascade_plan(128, 32, 32, 128, 6000, 376, 16, 8, 300)
    assert (p["prefix_part_blocks"], p["prefix_parts"]) == (128, 3)
    # 1 group of 2 and 2 KV heads: 6 pairs, so 1024 / 6 -> 171 parts wanted, floored at 32 blocks
    p = L.pa_paged_decode_cascade_plan(2, 2, 2, 64, 4000, 250, 1, 2, 200)
    assert (p["prefix_part_blocks"], p["prefix_parts"]) == (32, 7)
    assert p["launches"] == 4          # 2 stacked heads: the two decodes on two streams
    p = L.pa_paged_decode_cascade_plan(40, 16, 4, 128, 900, 60, 0, 2, 1)
    assert (p["prefix_part_blocks"], p["prefix_parts"], p["launches"]) == (0, 0, 3)
    assert L.pa_paged_decode_cascade_plan(0, 16, 4, 128, 0, 1, 0, 2, 1)["launches"] == 0
    with pytest.raises(pa.PAError):    # 3 x 4 stacked heads per KV head
        L.pa_paged_decode_cascade_plan(8, 16, 4, 128, 900, 60, 2, 3, 10)
    with pytest.raises(pa.PAError):
        L.pa_paged_decode_cascade_plan(8, 16, 4, 96, 900, 60, 2, 2, 10)
