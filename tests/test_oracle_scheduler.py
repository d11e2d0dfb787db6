"""Pins of the oracle's continuous-batching scheduler against what the pages and
plain counting fix: the pages' A/B/C/D example, closed forms without memory
pressure, and a brute-force replay of every plan on token tags (every position
of every decoded context must hold exactly that token after the step's copies
and writes run in device order). Planted mistakes show each pin has teeth."""

import inspect
import json
import os
import textwrap

import numpy as np
import pytest

from oracle import scheduler as SCH
from oracle.block_manager import BlockManagerError

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden(name):
    with open(os.path.join(HERE, "golden", name)) as f:
        return json.load(f)


def _run(sched, max_steps=100000):
    plans = []
    while not sched.idle():
        plans.append(sched.step())
        assert len(plans) < max_steps, "scheduler does not finish"
    return plans


# -- pins -------------------------------------------------------------------
def pin_pages_example():
    g = _golden("iteration_level_example.json")
    names = [r["name"] for r in g["requests"]]
    s = SCH.Scheduler(64, 16, max_num_seqs=g["max_num_seqs"])
    for i, r in enumerate(g["requests"]):
        s.submit(i, 5, r["output_len"], 1, r["arrival"])
    plans = _run(s)
    got = [[names[r] for r, _, _ in p.batch] for p in plans]
    want = g["iteration_level_batches"]
    # after the last batch, one more step only frees the finished requests
    assert got[:len(want)] == want and not any(got[len(want):]), got
    # D is admitted at the first step after A finishes, long before the
    # request-level schedule would start it
    first_d = next(p.step for p in plans if 3 in p.admitted)
    assert first_d < g["request_level_first_step_of_D"]


def pin_unconstrained_closed_form():
    """Pool and batch never short: request i runs exactly at steps
    arrival .. arrival + O - 1 with context P + k + 1 at its k-th step, and is
    freed at step arrival + O."""
    rng = np.random.default_rng(5)
    s = SCH.Scheduler(4096, 16, max_num_seqs=1000)
    reqs = []
    for i in range(40):
        p, o, a = int(rng.integers(1, 70)), int(rng.integers(1, 30)), int(rng.integers(0, 25))
        s.submit(i, p, o, 1, a)
        reqs.append((p, o, a))
    plans = _run(s)
    for i, (p, o, a) in enumerate(reqs):
        seen = [(pl.step, c) for pl in plans for r, _, c in pl.batch if r == i]
        assert seen == [(a + k, p + k + 1) for k in range(o)], (i, seen[:3])
        assert any(i in pl.finished and pl.step == a + o for pl in plans)
        assert not any(r == i for pl in plans for r, _ in pl.preempted)


def pin_batch_cap_waves():
    """Everything arrives at once with equal lengths and a cap of C requests:
    request i starts at step (i // C) * O (first come, first served)."""
    C, O = 4, 7
    s = SCH.Scheduler(4096, 16, max_num_seqs=C)
    for i in range(13):
        s.submit(i, 20, O, 1, 0)
    plans = _run(s)
    for i in range(13):
        start = min(pl.step for pl in plans for r, _, _ in pl.batch if r == i)
        assert start == (i // C) * O, (i, start)
    assert all(len(pl.batch) <= C for pl in plans)


def _replay(sched_factory, trace, check_fcfs=True):
    """Replay every plan on tags: a device and a host pool whose slots hold
    (request, branch, position) tags, branch -1 for prompt positions. Copies run
    in device order (swap-out, swap-in, prefill, copy-on-write, new tokens); then every
    decoded context is gathered through its block table and must read back its
    own tokens. Also checks counts, the batch cap, first-come-first-served
    admission, newest-first preemption and internal fragmentation."""
    s = sched_factory()
    bs = s.block_size
    prompts = {}
    for entry in trace:
        rid, p, o, n, a = entry[:5]
        toks = entry[5] if len(entry) > 5 else None
        s.submit(rid, p, o, n, a, tokens=toks)
        prompts[rid] = toks

    def tag(r, smp, pos):
        # a prompt token's keys/values depend on its whole prefix: requests that
        # share a prompt prefix share these tags; everything else is per request
        if pos < info[r][0] and prompts[r] is not None:
            return ("prefix", hash(tuple(prompts[r][:pos + 1])))
        return (r, -1 if pos < info[r][0] else smp, pos)
    dev = {}
    host = {}
    produced = {e[0]: 0 for e in trace}
    info = {e[0]: tuple(e[1:5]) for e in trace}
    order = {e[0]: k for k, e in enumerate(trace)}
    steps = 0
    while not s.idle():
        running_before = [r.rid for r in s.running]
        waiting_before = sorted([r.rid for r in s.waiting + s.pending if r.arrival <= s.step_index],
                                key=lambda r: (info[r][3], order[r]))
        pl = s.step()
        steps += 1
        assert steps < 20000
        # newest-first preemption: victims are a suffix of the running list
        victims = [r for r, _ in pl.preempted]
        if victims:
            tail = [r for r in running_before if r not in pl.finished][-len(victims):]
            assert tail == victims[::-1], (tail, victims)
            assert not pl.admitted and not pl.resumed
        # first come, first served among requests admitted for the first time
        if check_fcfs:
            fresh = [r for r in pl.admitted if produced[r] == 0]
            for r in fresh:
                earlier = [w for w in waiting_before
                           if (info[w][3], order[w]) < (info[r][3], order[r])]
                assert all(w in pl.admitted for w in earlier), (r, earlier)
        # device order of the copies
        for d, h in pl.swap_out:
            for o_ in range(bs):
                host[h * bs + o_] = dev.get(d * bs + o_)
        for h, d in pl.swap_in:
            for o_ in range(bs):
                dev[d * bs + o_] = host.get(h * bs + o_)
        for r, smp, pos, slot in pl.prefill:
            dev[slot] = tag(r, smp, pos)
        for src, dst in pl.copies:
            for o_ in range(bs):
                dev[dst * bs + o_] = dev.get(src * bs + o_)
        for r, smp, pos, slot in pl.writes:
            dev[slot] = tag(r, smp, pos)
        assert sum(1 for _ in pl.batch) <= s.max_num_seqs
        ids = [SCH.seq_id(r, smp) for r, smp, _ in pl.batch]
        maxb = max([-(-c // bs) for _, _, c in pl.batch], default=1)
        tables = s.bm.block_tables(ids, maxb) if ids else np.zeros((0, 1), np.int32)
        for (r, smp, ctx), row in zip(pl.batch, tables):
            for pos in range(ctx):
                want = tag(r, smp, pos)
                got = dev.get(int(row[pos // bs]) * bs + pos % bs)
                assert got == want, (pl.step, r, smp, pos, got, want)
        for r, smp, ctx in pl.batch:
            # the k-th decode of a sample sees its prompt and k tokens
            assert ctx == info[r][0] + produced[r] + 1, (pl.step, r, smp, ctx)
        for r in {r for r, _, _ in pl.batch}:
            produced[r] += 1
        # admission only while nothing is swapped out
        assert not (pl.admitted and s.swapped), (pl.step, pl.admitted)
        filled, alloc = s.kv_usage()
        nseq = sum(rq.num_samples for rq in s.running + s.finishing)
        assert 0 <= alloc - filled < bs * max(nseq, 1)
    for rid, (p, o, n, a) in info.items():
        assert produced[rid] == o, (rid, produced[rid], o)
    assert s.bm.num_free() == s.bm.num_blocks   # cached blocks left behind count as free
    return steps


def _trace(seed, n_req, max_samples, prompt=(1, 60), out=(1, 40), arrive=30):
    rng = np.random.default_rng(seed)
    return [(i, int(rng.integers(*prompt)), int(rng.integers(*out)),
             int(rng.integers(1, max_samples + 1)), int(rng.integers(0, arrive)))
            for i in range(n_req)]


def pin_replay_swap_mode():
    tr = _trace(7, 30, 3)
    _replay(lambda: SCH.Scheduler(22, 16, np.random.default_rng(1).permutation(22),
                                  max_num_seqs=12, num_host_blocks=400), tr)


def pin_replay_recompute_mode():
    tr = _trace(8, 30, 1)
    _replay(lambda: SCH.Scheduler(24, 16, np.random.default_rng(2).permutation(24),
                                  max_num_seqs=10, preempt_mode=SCH.PREEMPT_RECOMPUTE), tr)


def pin_replay_swap_falls_back_to_recompute():
    tr = _trace(9, 25, 1)
    _replay(lambda: SCH.Scheduler(20, 16, None, max_num_seqs=8, num_host_blocks=6), tr)


def _prompt_trace(seed, n_req, max_samples, systems=3, sys_len=(20, 70), own=(0, 30),
                  out=(1, 30), arrive=40):
    """Requests whose prompts are one of a few shared system prompts plus tokens of
    their own, with their token ids."""
    rng = np.random.default_rng(seed)
    sys_prompts = [rng.integers(0, 1000, int(rng.integers(*sys_len))).tolist()
                   for _ in range(systems)]
    trace = []
    for i in range(n_req):
        toks = sys_prompts[int(rng.integers(systems))] + \
            rng.integers(1000, 2000, int(rng.integers(*own))).tolist()
        trace.append((i, len(toks), int(rng.integers(*out)), int(rng.integers(1, max_samples + 1)),
                      int(rng.integers(0, arrive)), toks))
    return trace


def pin_prefix_cache_closed_form():
    """A second request with the same 100-token prompt shares its 6 full blocks:
    96 tokens found cached, 4 written; a third with a different third block
    shares only the first 2 blocks."""
    prompt = list(range(500, 600))
    other = prompt[:32] + [7] * 16 + prompt[48:]
    s = SCH.Scheduler(64, 16, max_num_seqs=8)
    s.submit(0, 100, 5, 1, 0, tokens=prompt)
    s.submit(1, 100, 5, 1, 2, tokens=prompt)
    s.submit(2, 100, 5, 1, 3, tokens=other)
    plans = _run(s)
    adm = {r: pl for pl in plans for r in pl.admitted}
    assert adm[0].cached == 0 and len(adm[0].prefill) == 100
    assert adm[1].cached == 96 and [p for _, _, p, _ in adm[1].prefill] == [96, 97, 98, 99]
    assert adm[2].cached == 32 and len(adm[2].prefill) == 68
    t0 = SCH.seq_id(0, 0)
    assert t0 not in s.bm._tables          # finished and freed, blocks left cached
    assert s.bm.num_cached() > 0 and s.bm.num_free() == 64


def pin_prefix_cache_recompute_hits_own_blocks():
    """A request dropped for recomputation finds its own prompt blocks still cached
    when it is admitted again: only the partial block and its generated tokens
    are written again."""
    prompt = list(range(40))                       # 2 full blocks + 8 tokens
    s = SCH.Scheduler(6, 16, max_num_seqs=4, preempt_mode=SCH.PREEMPT_RECOMPUTE)
    s.submit(0, 40, 40, 1, 0, tokens=prompt)       # grows to 80 tokens: 5 blocks
    s.submit(1, 30, 30, 1, 0)                      # uncached; preempted when short
    plans = _run(s)
    rec = [(pl.step, r) for pl in plans for r, m in pl.preempted if m == SCH.PREEMPT_RECOMPUTE]
    assert rec, "the trace must preempt"
    readmits = [pl for pl in plans for r in pl.admitted if r == 0 and pl.step > 0]
    for pl in readmits:
        assert pl.cached == 32 and min(p for r, _, p, _ in pl.prefill if r == 0) == 32


def pin_replay_prefix_cache_swap_mode():
    _replay(lambda: SCH.Scheduler(30, 16, np.random.default_rng(3).permutation(30),
                                  max_num_seqs=12, num_host_blocks=400),
            _prompt_trace(21, 30, 3), check_fcfs=True)


def pin_replay_prefix_cache_recompute_mode():
    _replay(lambda: SCH.Scheduler(18, 16, np.random.default_rng(4).permutation(18),
                                  max_num_seqs=10, preempt_mode=SCH.PREEMPT_RECOMPUTE),
            _prompt_trace(22, 30, 1), check_fcfs=True)


PINS = [pin_pages_example, pin_unconstrained_closed_form, pin_batch_cap_waves,
        pin_replay_swap_mode, pin_replay_recompute_mode, pin_replay_swap_falls_back_to_recompute,
        pin_prefix_cache_closed_form, pin_prefix_cache_recompute_hits_own_blocks,
        pin_replay_prefix_cache_swap_mode, pin_replay_prefix_cache_recompute_mode]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_scheduler_pin(pin):
    pin()


def test_replays_exercise_preemption_and_sharing():
    """The replay pins only mean something if the traces really preempt, swap,
    recompute and copy on write."""
    counts = {}
    for name, mk, tr in [
        ("swap", lambda: SCH.Scheduler(22, 16, None, max_num_seqs=12, num_host_blocks=400),
         _trace(7, 30, 3)),
        ("recompute", lambda: SCH.Scheduler(24, 16, None, max_num_seqs=10,
                                            preempt_mode=SCH.PREEMPT_RECOMPUTE), _trace(8, 30, 1)),
        ("fallback", lambda: SCH.Scheduler(20, 16, None, max_num_seqs=8, num_host_blocks=6),
         _trace(9, 25, 1)),
    ]:
        s = mk()
        for t in tr:
            s.submit(*t)
        plans = _run(s)
        counts[name] = {
            "swap": sum(1 for p in plans for _, m in p.preempted if m == SCH.PREEMPT_SWAP),
            "recompute": sum(1 for p in plans for _, m in p.preempted
                             if m == SCH.PREEMPT_RECOMPUTE),
            "cow": sum(len(p.copies) for p in plans),
            "swap_in": sum(len(p.swap_in) for p in plans),
        }
    assert counts["swap"]["swap"] > 0 and counts["swap"]["swap_in"] > 0
    assert counts["swap"]["cow"] > 0
    assert counts["recompute"]["recompute"] > 0
    assert counts["fallback"]["swap"] > 0 and counts["fallback"]["recompute"] > 0


def test_submit_validation():
    s = SCH.Scheduler(8, 16, max_num_seqs=4)
    with pytest.raises(BlockManagerError):
        s.submit(0, 0, 5)
    with pytest.raises(BlockManagerError):
        s.submit(0, 100, 100)          # 13 blocks > 8: can never fit
    with pytest.raises(BlockManagerError):
        s.submit(0, 5, 5, num_samples=5)
    s.submit(0, 5, 5)
    with pytest.raises(BlockManagerError):
        s.submit(0, 5, 5)
    r = SCH.Scheduler(8, 16, preempt_mode=SCH.PREEMPT_RECOMPUTE)
    with pytest.raises(BlockManagerError):
        r.submit(1, 5, 5, num_samples=2)


# -- planted mistakes -------------------------------------------------------
def _mutant(method: str, old: str, new: str):
    """The scheduler method ``method`` with one source fragment replaced."""
    src = textwrap.dedent(inspect.getsource(getattr(SCH.Scheduler, method)))
    assert old in src, (method, old)
    ns = {}
    exec(compile(src.replace(old, new, 1), f"<mutant {method}>", "exec"), vars(SCH), ns)
    return ns[method]


# Two checks of the scheduler cannot change its behaviour under its own rules,
# so mutants of them would be equivalent and are not planted: the copy-on-write
# count in ``_append_need`` (samples share a partly filled block only right after
# the fork at admission, whose first append admission itself accounts for) and
# the batch cap on resume (nothing is admitted while a request is swapped out,
# so resumed requests fit the cap they fitted before).
MISTAKES = {
    "prefix_cache_ignored": (
        "step", "if r.tokens is None:\n                slots = self.bm.add_seq",
        "if True:\n                slots = self.bm.add_seq", False),
    "admit_need_ignores_revived": (
        "_admit_need", "- hits + revived + extra", "- hits + extra", False),
    "recompute_rewrites_whole_prompt": (
        "step", "for p in range(cached, r.prompt_len))",
        "for p in range(0, r.prompt_len))", False),
    "admission_newest_first": (
        "_insert_by_arrival", "queue.insert(i, r)", "queue.insert(0, r)", True),
    "admit_need_ignores_samples": (
        "_admit_need", "extra = r.num_samples if", "extra = 0 if", False),
    "finished_never_freed": (
        "step", "for r in self.finishing:", "for r in []:", False),
    "copy_on_write_pairs_dropped": (
        "_append", "plan.copies.extend(pairs)", "pass", False),
    "swap_out_drops_a_block": (
        "_preempt", "plan.swap_out.extend(self.bm.swap_out(seq_id(r.rid, s)))",
        "plan.swap_out.extend(self.bm.swap_out(seq_id(r.rid, s))[:-1])", False),
    "preempt_oldest": (
        "step", "self._preempt(self.running.pop(), plan)",
        "self._preempt(self.running.pop(0 if self.running[0] is not r else -1), plan)", False),
    "recompute_forgets_generated": (
        "step", "length = r.prompt_len + r.generated", "length = r.prompt_len", False),
    "admit_while_swapped": (
        "step", "while not self.swapped and self.waiting:", "while self.waiting:", False),
    "admit_ignores_batch_cap": (
        "step", "if self._running_seqs() + r.num_samples > self.max_num_seqs:\n"
                "                break\n            if self._admit_need",
        "if False:\n                break\n            if self._admit_need", False),
}


def _fails_some_pin():
    for pin in PINS:
        try:
            pin()
        except (Exception, pytest.fail.Exception):
            return True
    return False


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_planted_mistake_is_caught(name, monkeypatch):
    method, old, new, static = MISTAKES[name]
    bad = _mutant(method, old, new)
    monkeypatch.setattr(SCH.Scheduler, method, staticmethod(bad) if static else bad)
    assert _fails_some_pin(), f"planted mistake {name!r} passed every pin"
