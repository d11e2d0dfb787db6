"""Continuous batching on a B200: the library's scheduler plans every step, the
executor runs it through the swap, cache-write, copy-on-write and decode
kernels, and each step's outputs are compared with the oracle's attention over
every decoded sample's logical keys and values (prompt + its own tokens), with
the plans checked bit for bit against the oracle scheduler."""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_352_b200 as pa
from oracle import fp8 as F
from oracle import scheduler as SCH
from oracle.attention import softmax_attention
from oracle.fpbits import bits_to_f64
from tests.parity import assert_close, out_to_f64
from workloads import gen

pytestmark = pytest.mark.gpu


def _run_trace(trace, nb, cap, host, mode, hq, hkv, d, dt, seed, fp8=None, cascade=None):
    """fp8 = (k_scale, v_scale) runs the loop over E4M3 caches; the oracle then
    attends to the quantized-then-dequantized rows. cascade sets the executor's
    cascade mode (PA_SCHED_CASCADE_*; the library's default otherwise)."""
    tdt = torch.float16 if dt == "f16" else torch.bfloat16
    cdt = torch.uint8 if fp8 else tdt
    order = np.random.default_rng(seed).permutation(nb)
    c = pa.Scheduler(nb, 16, order, max_num_seqs=cap, num_host_blocks=host, preempt_mode=mode)
    o = SCH.Scheduler(nb, 16, order, max_num_seqs=cap, num_host_blocks=host, preempt_mode=mode)
    for t in trace:
        toks = t[5] if len(t) > 5 else None
        c.submit(*t[:5], tokens=toks)
        o.submit(*t[:5], tokens=toks)
    max_ctx = max(t[1] + t[2] for t in trace)
    c.attach(hq, hkv, d, tdt, max_ctx, fp8_scales=fp8)
    if cascade is not None:
        c.set_cascade(cascade)
    kc = torch.zeros(nb, hkv, 16, d, dtype=cdt, device="cuda")
    vc = torch.zeros_like(kc)
    hk = torch.zeros(max(host, 1), hkv, 16, d, dtype=cdt).pin_memory() if host else None
    hv = torch.zeros_like(hk).pin_memory() if host else None
    toks = gen.RequestTokens(seed, {t[0]: t[1] for t in trace}, hkv, d, dt,
                             prompt_tokens={t[0]: (t[5] if len(t) > 5 else None) for t in trace})
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    scale = 1 / math.sqrt(d)
    G = hq // hkv
    stats = {"steps": 0, "preempt": 0, "swap": 0, "cow": 0, "seqs": 0, "cached": 0,
             "cascade_steps": 0, "cascade_groups": 0}
    while not o.idle():
        c.step()
        op = o.step()
        cp = c.plan()
        for f in ("preempted", "swap_out", "swap_in", "copies", "prefill", "writes", "batch"):
            assert [tuple(x) for x in cp[f]] == [tuple(x) for x in getattr(op, f)], (op.step, f)

        def rows(ws):
            k = np.zeros((len(ws), hkv, d), np.uint16)
            v = np.zeros_like(k)
            for i, (r, s, p, _) in enumerate(ws):
                k[i], v[i] = toks.row(r, s, p)
            return (torch.from_numpy(k.view(np.int16)).view(tdt).cuda(),
                    torch.from_numpy(v.view(np.int16)).view(tdt).cuda())

        pk, pv = rows(op.prefill)
        wk, wv = rows(op.writes)
        q_bits = np.stack([gen.step_query_bits(seed, r, s, op.step, hq, d, dt)
                           for r, s, _ in op.batch]) if op.batch else np.zeros((0, hq, d), np.uint16)
        q = torch.from_numpy(q_bits.view(np.int16)).view(tdt).cuda()
        out = torch.empty(len(op.batch), hq, d, dtype=tdt, device="cuda")
        c.execute(kc, vc, hk, hv, pk, pv, wk, wv, q, out, scale, dev_error=err)
        torch.cuda.synchronize()
        ng, _ = c.last_cascade()
        stats["cascade_steps"] += ng > 0
        stats["cascade_groups"] += ng
        got = out_to_f64(out, dt)
        for i, (r, s, ctx) in enumerate(op.batch):
            K, V = toks.rows(r, s, range(ctx))
            if fp8:
                Kf = F.dequantize(F.quantize(K, dt, fp8[0]), fp8[0])
                Vf = F.dequantize(F.quantize(V, dt, fp8[1]), fp8[1])
            else:
                Kf, Vf = bits_to_f64(K, dt), bits_to_f64(V, dt)
            ref = np.stack([softmax_attention(bits_to_f64(q_bits[i, h], dt), Kf[:, h // G],
                                              Vf[:, h // G], scale)
                            for h in range(hq)])
            assert_close(got[i], ref, f"step {op.step} request {r} sample {s}")
        stats["steps"] += 1
        stats["preempt"] += len(op.preempted)
        stats["swap"] += len(op.swap_out) + len(op.swap_in)
        stats["cow"] += len(op.copies)
        stats["seqs"] += len(op.batch)
        stats["cached"] += op.cached
    assert int(err.item()) == 0
    return stats


def _trace(seed, n, max_samples, prompt=(1, 70), out=(1, 40), arrive=25):
    rng = np.random.default_rng(seed)
    return [(i, int(rng.integers(*prompt)), int(rng.integers(*out)),
             int(rng.integers(1, max_samples + 1)), int(rng.integers(0, arrive)))
            for i in range(n)]


def test_swap_mode_trace_gqa_bf16():
    st = _run_trace(_trace(11, 24, 3), nb=26, cap=12, host=400, mode=pa.PA_PREEMPT_SWAP,
                    hq=8, hkv=2, d=128, dt="bf16", seed=41)
    assert st["preempt"] > 0 and st["swap"] > 0 and st["cow"] > 0, st


def test_recompute_mode_trace_mha_f16():
    st = _run_trace(_trace(12, 24, 1), nb=24, cap=10, host=0, mode=pa.PA_PREEMPT_RECOMPUTE,
                    hq=4, hkv=4, d=64, dt="f16", seed=42)
    assert st["preempt"] > 0, st


def test_long_prompts_split_kv():
    """Contexts of 600 to 2500 tokens, long enough for the decode's default split
    into partitions, through the loop."""
    rng = np.random.default_rng(13)
    trace = [(i, int(rng.integers(600, 2500)), int(rng.integers(1, 30)), 1,
              int(rng.integers(0, 6))) for i in range(8)]
    st = _run_trace(trace, nb=600, cap=8, host=0, mode=pa.PA_PREEMPT_SWAP,
                    hq=16, hkv=2, d=128, dt="bf16", seed=43)
    assert st["steps"] > 0


def test_swap_mode_trace_over_fp8_cache():
    """The loop over E4M3 caches: quantizing writes, copy-on-write and swaps of
    one-byte blocks, decode over the codes (tensor-core path, G = 4)."""
    st = _run_trace(_trace(11, 24, 3), nb=26, cap=12, host=400, mode=pa.PA_PREEMPT_SWAP,
                    hq=8, hkv=2, d=128, dt="bf16", seed=41, fp8=(0.02, 0.015))
    assert st["preempt"] > 0 and st["swap"] > 0 and st["cow"] > 0, st


def test_recompute_mode_trace_over_fp8_cache_mha():
    st = _run_trace(_trace(12, 24, 1), nb=24, cap=10, host=0, mode=pa.PA_PREEMPT_RECOMPUTE,
                    hq=4, hkv=4, d=64, dt="f16", seed=42, fp8=(0.01, 0.01))
    assert st["preempt"] > 0, st


def test_prefix_cached_requests_share_prompt_blocks():
    """Requests submitted with token ids and sharing system prompts: cached prompt
    blocks are read, never rewritten, and every step decodes to the oracle's
    attention over each request's prompt-determined keys and values."""
    from tests.test_oracle_scheduler import _prompt_trace
    st = _run_trace(_prompt_trace(23, 24, 3), nb=30, cap=12, host=400, mode=pa.PA_PREEMPT_SWAP,
                    hq=8, hkv=2, d=128, dt="bf16", seed=44)
    assert st["cached"] > 0 and st["cow"] > 0, st


def test_prefix_cached_recompute_over_fp8_cache():
    from tests.test_oracle_scheduler import _prompt_trace
    st = _run_trace(_prompt_trace(24, 24, 1), nb=18, cap=10, host=0,
                    mode=pa.PA_PREEMPT_RECOMPUTE, hq=4, hkv=4, d=64, dt="f16", seed=45,
                    fp8=(0.02, 0.02))
    assert st["cached"] > 0 and st["preempt"] > 0, st


def test_parallel_samples_decoded_through_the_cascade():
    """Samples forked from one prompt share its full blocks; with the cascade on,
    every step that has such a group reads them once per group, and every output
    still matches the oracle (8 / G = 2 samples per group at G = 4)."""
    st = _run_trace(_trace(31, 24, 4, prompt=(40, 200)), nb=120, cap=12, host=400,
                    mode=pa.PA_PREEMPT_SWAP, hq=8, hkv=2, d=128, dt="bf16", seed=51,
                    cascade=pa.PA_SCHED_CASCADE_ON)
    assert st["cascade_steps"] > 0 and st["cow"] > 0, st


def test_parallel_samples_through_the_cascade_mha_f16():
    """One query head per KV head: groups of up to 8 samples stack 8 heads."""
    st = _run_trace(_trace(32, 16, 6, prompt=(30, 300), arrive=8), nb=400, cap=16, host=400,
                    mode=pa.PA_PREEMPT_SWAP, hq=4, hkv=4, d=64, dt="f16", seed=52,
                    cascade=pa.PA_SCHED_CASCADE_ON)
    assert st["cascade_steps"] > 0, st


def test_prefix_cached_requests_through_the_cascade():
    """Requests sharing system prompts hold the same cached blocks: they are
    grouped across requests and decoded through the cascade."""
    from tests.test_oracle_scheduler import _prompt_trace
    st = _run_trace(_prompt_trace(23, 24, 3), nb=30, cap=12, host=400, mode=pa.PA_PREEMPT_SWAP,
                    hq=8, hkv=2, d=128, dt="bf16", seed=44, cascade=pa.PA_SCHED_CASCADE_ON)
    assert st["cached"] > 0 and st["cascade_steps"] > 0, st


def test_cascade_in_the_loop_over_fp8_cache():
    st = _run_trace(_trace(31, 24, 4, prompt=(40, 200)), nb=120, cap=12, host=400,
                    mode=pa.PA_PREEMPT_SWAP, hq=8, hkv=2, d=128, dt="bf16", seed=51,
                    fp8=(0.02, 0.015), cascade=pa.PA_SCHED_CASCADE_ON)
    assert st["cascade_steps"] > 0, st


def test_cascade_off_decodes_plainly():
    st = _run_trace(_trace(31, 12, 4, prompt=(40, 200)), nb=120, cap=12, host=400,
                    mode=pa.PA_PREEMPT_SWAP, hq=8, hkv=2, d=128, dt="bf16", seed=51,
                    cascade=pa.PA_SCHED_CASCADE_OFF)
    assert st["cascade_steps"] == 0, st
