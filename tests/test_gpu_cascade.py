"""pa_paged_decode_cascade on a B200 against the oracle: batches of forked
sequences (groups sharing leading blocks, sequences in no group, empty contexts,
members whose whole context is the shared prefix), both arithmetic paths of the
decode over the shared blocks (stacked heads on CUDA cores and on tensor cores),
16- and 8-bit caches, the shared-prefix workload through the runner, and
descriptors that lie (a member without the prefix blocks, a slot that does not
name its sequence back): flagged with PA_DEVERR_GROUP and still correct."""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_352_b200 as pa
from oracle import fp8 as F
from oracle.attention import paged_decode
from paged_kv_cache_352_b200.runner import DecodeRunner
from tests.parity import assert_close, out_to_f64, tensor_bits
import workloads
from workloads import gen

pytestmark = pytest.mark.gpu

TDT = {"f16": torch.float16, "bf16": torch.bfloat16}


def _dev(bits, dt):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(TDT[dt]).cuda()


def _forest(seed, nb, exact=False):
    """Prompts forked into samples that append their own tokens (none, and prompts
    of whole blocks, when ``exact``), plus one empty sequence. Returns the block
    manager, the batch (shuffled sequence ids) and its context lengths."""
    rng = np.random.default_rng(seed)
    bm = pa.BlockManager(nb, 16, rng.permutation(nb).astype(np.int32))
    sid, live = 0, []
    for _ in range(int(rng.integers(3, 7))):
        plen = 16 * int(rng.integers(1, 20)) if exact else int(rng.integers(1, 350))
        root = sid
        sid += 1
        bm.add_seq(root, plen)
        fam = [root]
        for _ in range(int(rng.integers(0, 10))):
            child = sid
            sid += 1
            bm.fork(int(rng.choice(fam)), child)
            fam.append(child)
        if not exact:
            for s in fam:
                n = int(rng.integers(0, 50))
                if n:
                    bm.append_slots(s, n)
        live += fam
    bm.add_seq(sid, 0)
    live.append(sid)
    batch = [live[i] for i in rng.permutation(len(live))]
    ctx = np.array([bm.seq_len(s) for s in batch], np.int32)
    return bm, batch, ctx


def _run(bm, batch, ctx, hq, hkv, d, dt, nb, seed, group_size, corrupt=None, fp8=None,
         order=None, keep=None):
    """order: None, "cascade" (pa_cascade_order) or "random" (a seeded
    permutation) as the call's seq_order; keep: a dict that receives the raw
    output bits under "out"."""
    mb = int(max(1, max(-(-int(c) // 16) for c in ctx)))
    tables = bm.block_tables(batch, mb)
    groups = bm.prefix_groups(batch, group_size)
    if corrupt is not None:
        tables, groups = corrupt(tables, groups)
    B = len(batch)
    q = gen.normal_bits([seed, 3], (B, hq, d), dt)
    scale = 1 / math.sqrt(d)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(B, hq, d, dtype=TDT[dt], device="cuda")
    maxctx = int(ctx.max())
    g = groups.to("cuda")
    ws = pa.cascade_workspace(B, hq, hkv, d, maxctx, mb, g)
    td, cd = torch.from_numpy(tables).cuda(), torch.from_numpy(ctx).cuda()
    so = None
    if order == "cascade":
        so = torch.from_numpy(pa.pa_cascade_order(ctx, groups)).cuda()
    elif order == "random":
        so = torch.from_numpy(np.random.default_rng([seed, 7]).permutation(B).astype(np.int32)).cuda()
    if fp8 is None:
        kb = gen.normal_bits([seed, 1], (nb, hkv, 16, d), dt)
        vb = gen.normal_bits([seed, 2], (nb, hkv, 16, d), dt)
        pa.pa_paged_decode_cascade(out, _dev(q, dt), _dev(kb, dt), _dev(vb, dt), td, cd, maxctx,
                                   scale, g, ws, dev_error=err, seq_order=so)
        want = paged_decode(q, kb, vb, tables, ctx, scale, dt)
    else:
        ks, vs = fp8
        rng = np.random.default_rng([seed, 9])
        codes = [(rng.integers(0, 0x7E, (nb, hkv, 16, d)) |
                  (rng.integers(0, 2, (nb, hkv, 16, d)) << 7)).astype(np.uint8) for _ in range(2)]
        pa.pa_paged_decode_cascade(out, _dev(q, dt), torch.from_numpy(codes[0]).cuda(),
                                   torch.from_numpy(codes[1]).cuda(), td, cd, maxctx, scale, g,
                                   ws, dev_error=err, k_scale=ks, v_scale=vs, seq_order=so)
        want = F.paged_decode_fp8(q, codes[0], codes[1], tables, ctx, scale, ks, vs, dt)
    torch.cuda.synchronize()
    if keep is not None:
        keep["out"] = tensor_bits(out)
    got = out_to_f64(out, dt)
    for s in range(B):
        assert_close(got[s], want[s], f"seq {s} ctx {ctx[s]}")
    return int(err.item()), groups


# (hq, hkv, d, dtype, group_size): group_size x G stacked heads per KV head = 8
# (tensor cores), 4 (tensor cores) or 2 (CUDA cores)
SHAPES = [(4, 4, 128, "f16", 8), (8, 4, 64, "bf16", 4), (16, 4, 128, "bf16", 2),
          (8, 8, 128, "f16", 4), (4, 4, 64, "f16", 2)]


@pytest.mark.parametrize("hq,hkv,d,dt,gs", SHAPES)
@pytest.mark.parametrize("seed", [1, 2])
def test_cascade_matches_oracle(hq, hkv, d, dt, gs, seed):
    nb = 1200
    bm, batch, ctx = _forest(seed * 31 + hq, nb)
    err, groups = _run(bm, batch, ctx, hq, hkv, d, dt, nb, seed, gs)
    assert err == 0
    assert groups.num_groups >= 1


# one launch (8 stacked heads) and two (2 stacked heads)
@pytest.mark.parametrize("hq,hkv,d,dt,gs", [SHAPES[0], SHAPES[1], SHAPES[4]])
def test_cascade_results_do_not_depend_on_the_order(hq, hkv, d, dt, gs):
    """The own-block decode scheduled in pa_cascade_order's order and in a random
    permutation: outputs bit-identical to the call without an order, and within
    tolerance of the oracle."""
    nb = 1200
    runs = {}
    for order in (None, "cascade", "random"):
        bm, batch, ctx = _forest(41 + hq, nb)
        keep = {}
        err, groups = _run(bm, batch, ctx, hq, hkv, d, dt, nb, 3, gs, order=order, keep=keep)
        assert err == 0 and groups.num_groups >= 1
        runs[order] = keep["out"]
    assert np.array_equal(runs[None], runs["cascade"])
    assert np.array_equal(runs[None], runs["random"])


def test_cascade_fp8_results_do_not_depend_on_the_order():
    nb = 900
    runs = {}
    for order in (None, "cascade"):
        bm, batch, ctx = _forest(19, nb)
        keep = {}
        err, _ = _run(bm, batch, ctx, 8, 4, 128, "bf16", nb, 12, 4, fp8=(0.05, 0.02),
                      order=order, keep=keep)
        assert err == 0
        runs[order] = keep["out"]
    assert np.array_equal(runs[None], runs["cascade"])


@pytest.mark.parametrize("hq,hkv,d,dt,gs", SHAPES[:2])
def test_cascade_prefix_is_the_whole_context(hq, hkv, d, dt, gs):
    """Prompts of whole blocks forked without appends: every member's context is
    the shared prefix and its own-block decode is empty."""
    nb = 800
    bm, batch, ctx = _forest(77, nb, exact=True)
    err, groups = _run(bm, batch, ctx, hq, hkv, d, dt, nb, 5, gs)
    assert err == 0 and groups.num_groups >= 1
    grouped = groups.seq_group >= 0
    assert all(int(ctx[i]) == 16 * int(groups.prefix_blocks[groups.seq_group[i]])
               for i in np.nonzero(grouped)[0])


@pytest.mark.parametrize("hq,hkv,d,dt,gs", [(4, 4, 128, "f16", 8), (8, 4, 128, "bf16", 4)])
def test_cascade_fp8_prefix_is_the_whole_context(hq, hkv, d, dt, gs):
    """Over 8-bit caches: forked whole-block prompts without appends, so every
    member's own-block decode is empty and its output is the prefix alone."""
    nb = 800
    bm, batch, ctx = _forest(78, nb, exact=True)
    err, groups = _run(bm, batch, ctx, hq, hkv, d, dt, nb, 6, gs, fp8=(0.05, 0.02))
    assert err == 0 and groups.num_groups >= 1


def test_cascade_rejects_a_member_without_the_prefix():
    """One member's first prefix block is pointed elsewhere: the group is decoded
    without its prefix (flagged), and every output still matches the oracle over
    the tables as given."""
    nb = 1200
    bm, batch, ctx = _forest(3, nb)

    def corrupt(tables, groups):
        k = int(np.argmax(groups.prefix_blocks))
        member = int(groups.members[k][1])
        tables = tables.copy()
        used = set(tables[tables >= 0].tolist())
        tables[member, 0] = next(b for b in range(nb) if b not in used)
        return tables, groups

    err, _ = _run(bm, batch, ctx, 4, 4, 128, "f16", nb, 4, 8, corrupt=corrupt)
    assert err & pa.PA_DEVERR_GROUP


def test_cascade_rejects_a_prefix_past_the_members_contexts():
    """A group claims one more shared block than its leader holds (still within
    the batch's longest context): the prefix decode reads past the leader's
    blocks, the group is rejected and flagged, and every output still matches
    the oracle."""
    nb = 1200
    bm, batch, ctx = _forest(5, nb)
    cap = int(ctx.max()) // 16

    def corrupt(tables, groups):
        for k in range(groups.num_groups):
            leader = int(groups.members[k][0])
            held = int((tables[leader] >= 0).sum())
            if held + 1 <= cap:
                groups.prefix_blocks[k] = held + 1
                groups.max_prefix_blocks = max(groups.max_prefix_blocks, held + 1)
                return tables, groups
        raise AssertionError("no group with room for a longer prefix")

    err, _ = _run(bm, batch, ctx, 4, 4, 128, "f16", nb, 6, 8, corrupt=corrupt)
    assert err & pa.PA_DEVERR_GROUP


@pytest.mark.parametrize("lie", ["empty_leader_slot", "prefix_over_the_bound"])
def test_cascade_rejects_an_inconsistent_group(lie):
    """A group whose leader slot is empty, or whose prefix count exceeds the
    caller's max_prefix_blocks: the prefix CTAs read nothing for it (they check
    the leader and the count themselves), prepare rejects it, and its members
    are decoded over their whole contexts, flagged and correct."""
    nb = 1200
    bm, batch, ctx = _forest(9, nb)

    def corrupt(tables, groups):
        k = int(np.argmax(groups.prefix_blocks))
        if lie == "empty_leader_slot":
            groups.members[k][0] = -1
        else:
            groups.prefix_blocks[k] = groups.max_prefix_blocks + 1
        return tables, groups

    err, _ = _run(bm, batch, ctx, 4, 4, 128, "f16", nb, 10, 8, corrupt=corrupt)
    assert err & pa.PA_DEVERR_GROUP


def test_cascade_rejects_a_slot_that_does_not_name_back():
    """Two members' slots swapped in seq_member: neither is owned by the group;
    both are decoded over their whole contexts, flagged, and correct."""
    nb = 1200
    bm, batch, ctx = _forest(6, nb)

    def corrupt(tables, groups):
        k = 0
        a, b = int(groups.members[k][0]), int(groups.members[k][1])
        groups.seq_member[a], groups.seq_member[b] = groups.seq_member[b], groups.seq_member[a]
        return tables, groups

    err, _ = _run(bm, batch, ctx, 8, 4, 64, "bf16", nb, 8, 4, corrupt=corrupt)
    assert err & pa.PA_DEVERR_GROUP


# 8 stacked heads (one launch) at 1, 2 and 4 query heads per KV head, and 2 (two launches)
@pytest.mark.parametrize("hq,hkv,d,dt,gs", [(4, 4, 128, "f16", 8), (8, 4, 128, "bf16", 4),
                                            (16, 4, 128, "bf16", 2), (4, 4, 64, "f16", 2),
                                            (8, 4, 64, "f16", 4)])
def test_cascade_fp8_matches_oracle(hq, hkv, d, dt, gs):
    nb = 900
    bm, batch, ctx = _forest(11 + hq, nb)
    err, groups = _run(bm, batch, ctx, hq, hkv, d, dt, nb, 12, gs, fp8=(0.05, 0.02))
    assert err == 0 and groups.num_groups >= 1


def test_shared_prefix_workload_through_the_runner():
    """The shared-prefix workload (reduced): the step's decode goes through the
    cascade, matches the oracle and the plain decode of the same batch."""
    wl = workloads.workload("prefix_share_cow", small=True)
    r = DecodeRunner(wl)
    assert r.groups is not None and r.groups.num_groups == wl.num_prompts
    out = r.step().clone()
    plain = torch.empty_like(out)
    r.decode(plain)
    torch.cuda.synchronize()
    assert r.error_bits() == 0
    ref = paged_decode(tensor_bits(r.q), tensor_bits(r.k_cache), tensor_bits(r.v_cache),
                       r.block_tables_host, r.context_lens_host, wl.scale, wl.dtype)
    got = out_to_f64(out, wl.dtype)
    for s in range(wl.num_seqs):
        assert_close(got[s], ref[s], f"seq {s}")
    assert_close(out_to_f64(plain, wl.dtype), got, "cascade vs plain decode")
