"""Pins of the oracle's grouping rule for decoding shared blocks once
(``oracle.block_manager.BlockManager.prefix_groups``), on the oracle alone.

The pages share a prompt's blocks among the samples forked from it and copy a
block only when one of them writes into it ("PagedAttention: The vLLM Paper",
"Implementation Essentials", prefix sharing; "PagedAttention and Continuous
Batching", "Pages, from operating systems"). They name no rule for grouping
the sharers at decode time; the oracle's rule is this build's reading:
sequences with a full block are bucketed by their first block id (buckets in
order of first appearance, members in batch order), buckets are cut into runs
of ``group_size``, and a run of two or more is a group whose prefix is the
longest run of leading block ids that every member holds as full blocks.

The pins here do not call the CUDA-side library: a hand-worked batch whose
groups were derived on paper from the rule, the pages' forked-prompt case, and
invariants over random fork trees (every group's prefix is shared, full and
maximal; runs respect bucket order and the size cap). ``test_planted_*``
plants plausible mistakes in the oracle's rule and checks that a pin fails.
"""

import numpy as np
import pytest

from oracle import block_manager as OBM


# --------------------------------------------------------------------------
# the batches
# --------------------------------------------------------------------------

def _hand_batch():
    """A batch built step by step with the identity free order (block 0 is
    handed out first). The tables, worked by hand from the stack free list and
    the copy-on-write rule:

      seq 10: 40 tokens            -> [0, 1, 2]        (2 full blocks; 8 tokens in 2)
      fork 10 -> 11, 10 -> 12      -> both [0, 1, 2]   (block 2 refcount 3)
      seq 20: 70 tokens            -> [3, 4, 5, 6, 7]  (4 full; 6 tokens in 7)
      fork 20 -> 21
      seq 40: 20 tokens            -> [8, 9]           (1 full; 4 tokens in 9)
      fork 40 -> 41                -> [8, 9]           (block 9 shared, partly filled)
      seq 50: 32 tokens            -> [10, 11]         (exactly 2 full blocks)
      fork 50 -> 51
      seq 30: 15 tokens            -> [12]             (no full block)
      seq 31: 33 tokens            -> [13, 14, 15]     (2 full; alone in its bucket)
      11 appends 10 tokens: block 2 is shared and partly filled -> copy to 16;
                            50 tokens -> [0, 1, 16, 17]   (3 full)
      21 appends 26 tokens: block 7 shared, partly filled -> copy to 18;
                            96 tokens -> [3, 4, 5, 6, 18, 19]   (6 full)
      51 appends 16 tokens: block 11 is full, so a fresh block 20 and no copy;
                            48 tokens -> [10, 11, 20]   (3 full)
    """
    bm = OBM.BlockManager(64, 16, list(range(64)))
    bm.add_seq(10, 40)
    bm.fork(10, 11)
    bm.fork(10, 12)
    bm.add_seq(20, 70)
    bm.fork(20, 21)
    bm.add_seq(40, 20)
    bm.fork(40, 41)
    bm.add_seq(50, 32)
    bm.fork(50, 51)
    bm.add_seq(30, 15)
    bm.add_seq(31, 33)
    assert bm.append_slots(11, 10)[1] == [(2, 16)]
    assert bm.append_slots(21, 26)[1] == [(7, 18)]
    assert bm.append_slots(51, 16)[1] == []
    return bm


# batch order: index 0..10
HAND_BATCH = [21, 10, 30, 12, 41, 51, 20, 11, 31, 40, 50]

# Worked by hand. Buckets by first block, in order of first appearance:
#   first block 3:  21 (i0), 20 (i6)
#   first block 0:  10 (i1), 12 (i3), 11 (i7)
#   (30 has no full block: no bucket)
#   first block 8:  41 (i4), 40 (i9)
#   first block 10: 51 (i5), 50 (i10)
#   first block 13: 31 (i8) alone
# group_size 8:
#   [0, 6]:    tables [3,4,5,6,18,19] / [3,4,5,6,7]; full 6 / 4 -> prefix 4
#   [1, 3, 7]: [0,1,2] / [0,1,2] / [0,1,16,17]; full 2 / 2 / 3 -> prefix 2
#   [4, 9]:    [8,9] / [8,9]; full 1 / 1 -> prefix 1 (block 9 is shared but partly filled)
#   [5, 10]:   [10,11,20] / [10,11]; full 3 / 2 -> prefix 2
# group_size 2: bucket 0 is cut into [1, 3] and [7]; the lone [7] is no group.
HAND_GROUPS = {
    8: ([[0, 6], [1, 3, 7], [4, 9], [5, 10]], [4, 2, 1, 2]),
    2: ([[0, 6], [1, 3], [4, 9], [5, 10]], [4, 2, 1, 2]),
    3: ([[0, 6], [1, 3, 7], [4, 9], [5, 10]], [4, 2, 1, 2]),
}


def _fork_forest(seed, nb=3000):
    """Random prompts forked into samples (forks of forks too) that append their
    own tokens, on the oracle manager; returns it and a shuffled batch."""
    rng = np.random.default_rng(seed)
    bm = OBM.BlockManager(nb, 16, rng.permutation(nb).tolist())
    sid, live = 0, []
    for _ in range(int(rng.integers(2, 9))):
        root = sid
        sid += 1
        bm.add_seq(root, int(rng.integers(1, 400)))
        fam = [root]
        for _ in range(int(rng.integers(0, 12))):
            child = sid
            sid += 1
            bm.fork(int(rng.choice(fam)), child)
            fam.append(child)
        for s in fam:
            n = int(rng.integers(0, 60))
            if n:
                bm.append_slots(s, n)
        live += fam
    return bm, [live[i] for i in rng.permutation(len(live))]


def _check_invariants(bm, batch, group_size):
    members, prefix, sgroup, smember = bm.prefix_groups(batch, group_size)
    tables = [bm.table(s) for s in batch]
    full = [bm.seq_len(s) // 16 for s in batch]
    seen = set()
    for k, (run, P) in enumerate(zip(members, prefix)):
        assert 2 <= len(run) <= group_size
        assert run == sorted(run)                                  # batch order
        assert len({tables[i][0] for i in run}) == 1               # one bucket
        assert P >= 1
        for slot, i in enumerate(run):
            assert i not in seen
            seen.add(i)
            assert sgroup[i] == k and smember[i] == slot
            assert full[i] >= P                                     # the prefix is full
            assert tables[i][:P] == tables[run[0]][:P]              # and shared
        # maximal: one block more is partly filled somewhere or not shared by all
        if P < min(full[i] for i in run):
            assert len({tables[i][P] for i in run}) > 1
    for i in range(len(batch)):
        if i not in seen:
            assert sgroup[i] == -1 and smember[i] == -1
    # runs: each bucket (first block id; buckets in order of their first member,
    # members in batch order) is cut into consecutive runs of group_size; the
    # groups are some of these runs, listed in this order
    buckets = {}
    for i in range(len(batch)):
        if full[i] >= 1:
            buckets.setdefault(tables[i][0], []).append(i)
    runs = [b[c:c + group_size] for b in buckets.values() for c in range(0, len(b), group_size)]
    assert all(run in runs for run in members)
    idx = [runs.index(run) for run in members]
    assert idx == sorted(idx)
    return members, prefix


# --------------------------------------------------------------------------
# pins
# --------------------------------------------------------------------------

def pin_hand_worked_batch():
    bm = _hand_batch()
    assert [bm.table(s) for s in (10, 11, 12)] == [[0, 1, 2], [0, 1, 16, 17], [0, 1, 2]]
    assert [bm.table(s) for s in (20, 21)] == [[3, 4, 5, 6, 7], [3, 4, 5, 6, 18, 19]]
    assert [bm.table(s) for s in (40, 41, 50, 51)] == [[8, 9], [8, 9], [10, 11], [10, 11, 20]]
    for gs, (want_members, want_prefix) in HAND_GROUPS.items():
        members, prefix, sgroup, smember = bm.prefix_groups(HAND_BATCH, gs)
        assert members == want_members, (gs, members)
        assert prefix == want_prefix, (gs, prefix)
        for k, run in enumerate(want_members):
            for slot, i in enumerate(run):
                assert (sgroup[i], smember[i]) == (k, slot)
        grouped = {i for run in want_members for i in run}
        assert all(sgroup[i] == -1 for i in range(len(HAND_BATCH)) if i not in grouped)


def pin_forked_prompt_of_62_blocks():
    """The shared-prefix workload's shape: a 1000-token prompt (62 full blocks and
    8 tokens in a 63rd) forked 8 ways; every sample appends, so the 63rd block is
    copied on write by all but the last writer, and the group's prefix is the 62
    full blocks."""
    bm = OBM.BlockManager(1024, 16)
    bm.add_seq(0, 1000)
    for c in range(1, 8):
        bm.fork(0, c)
    for c in range(8):
        bm.append_slots(c, 1 + 3 * c)
    members, prefix, _, _ = bm.prefix_groups(range(8), 8)
    assert members == [list(range(8))] and prefix == [62]
    members, prefix, _, _ = bm.prefix_groups(range(8), 4)
    assert members == [[0, 1, 2, 3], [4, 5, 6, 7]] and prefix == [62, 62]
    members, prefix, sgroup, smember = bm.prefix_groups([3], 8)
    assert members == [] and prefix == [] and sgroup == [-1] and smember == [-1]


def pin_unshared_and_empty_batches():
    bm = OBM.BlockManager(256, 16)
    assert bm.prefix_groups([], 8) == ([], [], [], [])
    for s, n in ((0, 40), (1, 16), (2, 0), (3, 300)):
        bm.add_seq(s, n)
    assert bm.prefix_groups([3, 0, 2, 1], 8) == ([], [], [-1] * 4, [-1] * 4)


def pin_invariants_over_random_fork_trees():
    grouped = 0
    for seed in range(10):
        bm, batch = _fork_forest(seed)
        for gs in (2, 3, 5, 8):
            members, _ = _check_invariants(bm, batch, gs)
            grouped += len(members)
    assert grouped > 50        # the forests do form groups


def pin_prefix_is_longest_full_shared_run():
    """Maximality against a brute-force search over every candidate length: the
    prefix is the largest P such that every member holds blocks 0..P-1 as full
    blocks and all members' first P ids agree."""
    for seed in range(6):
        bm, batch = _fork_forest(100 + seed)
        members, prefix, _, _ = bm.prefix_groups(batch, 8)
        for run, P in zip(members, prefix):
            tabs = [bm.table(batch[i]) for i in run]
            full = [bm.seq_len(batch[i]) // 16 for i in run]
            best = 0
            for cand in range(1, max(len(t) for t in tabs) + 1):
                if all(f >= cand for f in full) and all(t[:cand] == tabs[0][:cand] for t in tabs):
                    best = cand
            assert P == best


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


# --------------------------------------------------------------------------
# planted mistakes: each must make at least one pin fail
# --------------------------------------------------------------------------

def _rule(self, seq_ids, group_size, key=lambda t: t[0], cap_full=True, cut=True,
          bucket_order="appearance", min_run=2, member_order="batch"):
    """The oracle's rule with knobs that each switch one step to a plausible
    mistake (test code only)."""
    seq_ids = list(seq_ids)
    full = [self._lens[s] // self.block_size for s in seq_ids]
    buckets = {}
    for i, s in enumerate(seq_ids):
        if full[i] >= 1:
            buckets.setdefault(key(self._tables[s]), []).append(i)
    if member_order == "seq_id":
        buckets = {k: sorted(v, key=lambda i: seq_ids[i]) for k, v in buckets.items()}
    sources = list(buckets.values())
    if bucket_order == "block_id":
        sources = [buckets[k] for k in sorted(buckets)]
    members, prefix = [], []
    sgroup = [-1] * len(seq_ids)
    smember = [-1] * len(seq_ids)
    for src in sources:
        step = group_size if cut else len(src)
        for c in range(0, len(src), step):
            run = src[c:c + step]
            if len(run) < min_run:
                continue
            tables = [self._tables[seq_ids[i]] for i in run]
            p = min(full[i] for i in run) if cap_full else min(len(t) for t in tables)
            shared = 0
            while shared < p and all(shared < len(t) and t[shared] == tables[0][shared]
                                     for t in tables):
                shared += 1
            if shared == 0:
                continue
            for slot, i in enumerate(run):
                sgroup[i] = len(members)
                smember[i] = slot
            members.append(run)
            prefix.append(shared)
    return members, prefix, sgroup, smember


MISTAKES = {
    # the prefix runs into a shared but partly filled block
    "prefix_not_capped_at_full_blocks": dict(cap_full=False),
    # sequences bucketed by their last block instead of their first
    "bucketed_by_last_block": dict(key=lambda t: t[-1]),
    # a bucket larger than group_size stays one group
    "runs_not_cut_at_group_size": dict(cut=False),
    # buckets taken in order of block id instead of first appearance
    "buckets_in_block_id_order": dict(bucket_order="block_id"),
    # a lone sequence forms a group of one
    "lone_run_is_a_group": dict(min_run=1),
    # members taken in sequence-id order instead of batch order
    "members_in_seq_id_order": dict(member_order="seq_id"),
}


def _fails_some_pin():
    for pin in PINS:
        try:
            pin()
        except Exception:
            return True
    return False


def test_rule_with_no_knob_is_the_oracle():
    """The knob-free restatement above agrees with the oracle, so each planted
    mistake differs from the oracle in exactly its one step."""
    for seed in range(6):
        bm, batch = _fork_forest(200 + seed)
        for gs in (2, 4, 8):
            assert _rule(bm, batch, gs) == bm.prefix_groups(batch, gs)


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_planted_mistake_is_caught(name, monkeypatch):
    knobs = MISTAKES[name]
    monkeypatch.setattr(OBM.BlockManager, "prefix_groups",
                        lambda self, seq_ids, group_size: _rule(self, seq_ids, group_size,
                                                                **knobs))
    assert _fails_some_pin(), f"planted mistake {name!r} passed every pin"
