"""The library's continuous-batching scheduler (pa_sched_*) against the oracle
scheduler, on the CPU: every step's plan (freed, preempted, resumed and admitted
requests, swap and copy-on-write pairs, prefill and new-token writes, the decode
batch and its block tables) must match bit for bit, over traces that preempt by
swap and by recompute and share prompts between samples."""

import numpy as np
import pytest

import paged_kv_cache_352_b200 as pa
from oracle import scheduler as SCH
from oracle.block_manager import BlockManagerError


def _pair(nb, order, cap, host, mode):
    c = pa.Scheduler(nb, 16, order, max_num_seqs=cap, num_host_blocks=host, preempt_mode=mode)
    o = SCH.Scheduler(nb, 16, order, max_num_seqs=cap, num_host_blocks=host, preempt_mode=mode)
    return c, o


def _compare_run(c, o, trace):
    for t in trace:
        toks = t[5] if len(t) > 5 else None
        c.submit(*t[:5], tokens=toks)
        o.submit(*t[:5], tokens=toks)
    steps = 0
    stats = {"preempt": 0, "swap_in": 0, "cow": 0, "prefill": 0}
    while not o.idle():
        assert not c.idle()
        c.step()
        op = o.step()
        cp = c.plan()
        assert cp["step"] == op.step
        assert cp["cached"] == op.cached
        for f in ("finished", "preempted", "resumed", "admitted", "swap_out", "swap_in",
                  "copies", "prefill", "writes", "batch"):
            got = [tuple(x) if isinstance(x, (tuple, list)) else x for x in cp[f]]
            want = [tuple(x) if isinstance(x, (tuple, list)) else x for x in getattr(op, f)]
            assert got == want, (op.step, f, got[:6], want[:6])
        if op.batch:
            ids = o.batch_seq_ids(op)
            want_t = o.bm.block_tables(ids, cp["tables"].shape[1])
            assert np.array_equal(cp["tables"], want_t), op.step
        assert c.counts.total_context == sum(ctx for _, _, ctx in op.batch)
        assert c.kv_usage() == o.kv_usage()
        assert c.bm.free_list() == o.bm.free_list()
        stats["preempt"] += len(op.preempted)
        stats["swap_in"] += len(op.swap_in)
        stats["cow"] += len(op.copies)
        stats["prefill"] += len(op.prefill)
        steps += 1
    assert c.idle()
    return stats


def _trace(seed, n_req, max_samples, prompt=(1, 60), out=(1, 40), arrive=30):
    rng = np.random.default_rng(seed)
    return [(i, int(rng.integers(*prompt)), int(rng.integers(*out)),
             int(rng.integers(1, max_samples + 1)), int(rng.integers(0, arrive)))
            for i in range(n_req)]


@pytest.mark.parametrize("seed", range(6))
def test_swap_mode_matches_oracle(seed):
    nb = 22 + 6 * seed
    order = np.random.default_rng(seed).permutation(nb)
    c, o = _pair(nb, order, 12, 400, pa.PA_PREEMPT_SWAP)
    st = _compare_run(c, o, _trace(100 + seed, 30, 3))
    assert st["cow"] > 0


@pytest.mark.parametrize("seed", range(6))
def test_recompute_mode_matches_oracle(seed):
    nb = 24 + 4 * seed
    order = np.random.default_rng(50 + seed).permutation(nb)
    c, o = _pair(nb, order, 10, 0, pa.PA_PREEMPT_RECOMPUTE)
    _compare_run(c, o, _trace(200 + seed, 30, 1))


@pytest.mark.parametrize("seed", range(4))
def test_small_host_pool_falls_back_to_recompute(seed):
    c, o = _pair(20, None, 8, 6, pa.PA_PREEMPT_SWAP)
    _compare_run(c, o, _trace(300 + seed, 25, 1))


def test_traces_exercise_every_branch():
    totals = {"preempt": 0, "swap_in": 0, "cow": 0, "prefill": 0}
    for seed in range(3):
        c, o = _pair(22, None, 12, 400, pa.PA_PREEMPT_SWAP)
        st = _compare_run(c, o, _trace(100 + seed, 30, 3))
        for k in totals:
            totals[k] += st[k]
    assert all(v > 0 for v in totals.values()), totals


def test_large_trace_matches_oracle():
    rng = np.random.default_rng(9)
    trace = [(i, int(rng.integers(16, 400)), int(rng.integers(1, 120)),
              int(rng.choice([1, 1, 1, 2, 4])), int(rng.integers(0, 200))) for i in range(150)]
    c, o = _pair(600, rng.permutation(600), 64, 5000, pa.PA_PREEMPT_SWAP)
    st = _compare_run(c, o, trace)
    assert st["preempt"] > 0 and st["cow"] > 0


def test_submit_validation_matches_oracle():
    cases = [(0, 0, 5, 1, 0), (0, 100, 100, 1, 0), (0, 5, 5, 5, 0), (-1, 5, 5, 1, 0),
             (0, 5, 5, 65, 0)]
    for case in cases:
        c = pa.Scheduler(8, 16, max_num_seqs=4)
        o = SCH.Scheduler(8, 16, max_num_seqs=4)
        with pytest.raises(pa.PAError) as ce:
            c.submit(*case)
        with pytest.raises(BlockManagerError) as oe:
            o.submit(*case)
        assert ce.value.code == oe.value.code, case
    c = pa.Scheduler(8, 16, preempt_mode=pa.PA_PREEMPT_RECOMPUTE)
    with pytest.raises(pa.PAError):
        c.submit(1, 5, 5, 2)
    with pytest.raises(pa.PAError):
        pa.Scheduler(8, 16, num_host_blocks=4, preempt_mode=pa.PA_PREEMPT_RECOMPUTE)


def test_many_sample_request_that_cannot_swap_fails_the_scheduler():
    # two 3-sample requests; no host pool, so the newer one cannot be preempted
    c, o = _pair(16, None, 8, 0, pa.PA_PREEMPT_SWAP)
    for t in [(0, 40, 30, 3, 0), (1, 40, 30, 3, 0)]:
        c.submit(*t)
        o.submit(*t)
    err_c = err_o = None
    for _ in range(100):
        try:
            o.step()
        except BlockManagerError as e:
            err_o = e
        try:
            c.step()
        except pa.PAError as e:
            err_c = e
        if err_c or err_o:
            break
    assert err_c is not None and err_o is not None
    assert err_c.code == err_o.code == pa._lib.PA_ERR_NO_FREE_BLOCKS
    with pytest.raises(pa.PAError):
        c.step()


def test_execute_requires_attach_and_a_plan():
    c = pa.Scheduler(8, 16)
    st = c._lib.pa_sched_execute(c._h, None, None, None, None, None, None, None, None, None,
                                 None, 1.0, None, None)
    assert st == pa._lib.PA_ERR_INVALID_ARG and "no executor attached" in pa.last_error()


@pytest.mark.parametrize("seed", range(4))
def test_prefix_cached_requests_match_oracle(seed):
    from tests.test_oracle_scheduler import _prompt_trace
    mode = pa.PA_PREEMPT_SWAP if seed % 2 == 0 else pa.PA_PREEMPT_RECOMPUTE
    host = 400 if mode == pa.PA_PREEMPT_SWAP else 0
    samples = 3 if mode == pa.PA_PREEMPT_SWAP else 1
    nb = 26 + 4 * seed
    c, o = _pair(nb, np.random.default_rng(seed).permutation(nb), 10, host, mode)
    trace = _prompt_trace(400 + seed, 30, samples)
    _compare_run(c, o, trace)
    assert c.bm.num_cached() == o.bm.num_cached() > 0


def test_submit_tokens_checks_length():
    c = pa.Scheduler(8, 16)
    with pytest.raises(pa.PAError):
        c.submit(0, 5, 3, tokens=[1, 2, 3])


def test_host_planning_measurement_runs_the_whole_trace():
    """The bench's host-planning figure plans a whole trace: every request's
    prompt and output tokens get slots."""
    import bench
    trace = bench.continuous_batching_trace(60)
    r = bench.measure_host_planning(num_requests=60)
    want = sum(t[2] * t[3] for t in trace)   # generated tokens: output length x samples
    assert r["steps"] > 0 and r["slots"] >= want and r["us_per_step"] > 0
