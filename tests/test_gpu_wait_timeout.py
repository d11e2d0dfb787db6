"""The device side of failure detection: a bounded on-chip wait that runs out.

Every wait of the decode kernels on a stage barrier gives up after a time limit,
reports PA_DEVERR_WAIT_TIMEOUT in the device error word, still waits for the
copies the warp did issue, and returns, so the context stays usable. Here the
library's test hook (pa_test_stall_next_decode) makes the next decode launch
arm each warp's first stage without issuing its copy and lowers the wait limit
to a few milliseconds, so that wait runs out with nothing left in flight. No
GPU fault, trap or unbounded wait is involved: the stalled barrier simply never
completes and the wait gives up.

Each case checks that the call returned, that the error bit is set, that the
hook applied to one launch only, and that the next decode on the same inputs
(workspace zeroed again) matches the float64 oracle. The cases cover both split
modes (one CTA per partition with the last-CTA merge; one warp per partition
plus the merge kernel) and both arithmetic paths (CUDA cores, tensor cores).
"""

import time

import numpy as np
import pytest
import torch

import paged_kv_cache_352_b200 as pa
from oracle.attention import paged_decode as oracle_decode
from paged_kv_cache_352_b200 import _lib as L
from tests.parity import assert_close, out_to_f64
from workloads import gen

pytestmark = pytest.mark.gpu

_TORCH = {"f16": torch.float16, "bf16": torch.bfloat16}
LIMIT_NS = 2_000_000   # 2 ms


def _batch(ctx, hq, hkv, dtype, seed, d=128):
    ctx = np.asarray(ctx, np.int32)
    nblk = [-(-int(c) // 16) for c in ctx]
    nb = sum(nblk) + 4
    kb = gen.normal_bits([seed, 1], (nb, hkv, 16, d), dtype)
    vb = gen.normal_bits([seed, 2], (nb, hkv, 16, d), dtype)
    qb = gen.normal_bits([seed, 3], (len(ctx), hq, d), dtype)
    perm = np.random.default_rng([seed, 4]).permutation(nb).astype(np.int32)
    tables = np.full((len(ctx), max(nblk)), -1, np.int32)
    used = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = perm[used:used + n]
        used += n
    return ctx, kb, vb, qb, tables


@pytest.mark.parametrize("name,ctx,hq,hkv,dtype,pt,launches", [
    # one CTA per partition, CUDA-core path (1 query head per KV head)
    ("cta_split_cuda_cores", [700, 1500, 33, 1], 4, 4, "f16", 256, 1),
    # one CTA per partition, tensor-core path (8 query heads per KV head)
    ("cta_split_tensor_cores", [900, 2100, 64], 16, 2, "bf16", 512, 1),
    # one warp per partition plus the merge kernel, tensor-core path
    ("warp_split_tensor_cores", np.random.default_rng(9).integers(3841, 4097, 64).tolist(),
     16, 4, "bf16", 256, 2),
    # a sequence that is not split at all writes its output directly
    ("unsplit", [300, 200], 8, 8, "f16", 0, 1),
])
def test_wait_runs_out_and_reports(name, ctx, hq, hkv, dtype, pt, launches):
    ctx, kb, vb, qb, tables = _batch(ctx, hq, hkv, dtype, seed=len(name))
    B, d = len(ctx), 128
    _, _, nl = pa.pa_paged_decode_plan(B, hq, hkv, d, int(ctx.max()), pt)
    assert nl == launches
    dev = lambda b: torch.from_numpy(b.view(np.int16)).view(_TORCH[dtype]).cuda()
    q, kc, vc = dev(qb), dev(kb), dev(vb)
    t, cl = torch.from_numpy(tables).cuda(), torch.from_numpy(ctx).cuda()
    scale = 1 / np.sqrt(d)
    ws = pa.decode_workspace(B, hq, hkv, d, int(ctx.max()), pt)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)

    assert L.lib().pa_test_stall_next_decode(LIMIT_NS) == L.PA_OK
    t0 = time.perf_counter()
    pa.pa_paged_decode(out, q, kc, vc, t, cl, int(ctx.max()), scale, pt, ws, err)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 10.0
    assert int(err.item()) & pa.PA_DEVERR_WAIT_TIMEOUT, "the stalled wait was not reported"

    # the request applied to that launch only; the next decode is clean and right
    err.zero_()
    if ws is not None:
        ws.zero_()
    pa.pa_paged_decode(out, q, kc, vc, t, cl, int(ctx.max()), scale, pt, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = oracle_decode(qb, kb, vb, tables, ctx, scale, dtype)
    assert_close(out_to_f64(out, dtype), want, f"{name}: decode after a timed-out launch")


def test_wait_runs_out_in_the_cascade():
    """The cascade's single decode launch: CTAs over the groups' shared prefixes
    (tensor cores) and warps over each sample's own blocks, one per KV head."""
    from tests.test_gpu_cascade import _forest
    nb, hq, hkv, d = 1200, 4, 4, 128
    bm, batch, ctx = _forest(21, nb)
    tables = bm.block_tables(batch, max(1, max(-(-int(c) // 16) for c in ctx)))
    groups = bm.prefix_groups(batch, 8)
    assert groups.num_groups >= 1
    kb = gen.normal_bits([61, 1], (nb, hkv, 16, d), "f16")
    vb = gen.normal_bits([61, 2], (nb, hkv, 16, d), "f16")
    qb = gen.normal_bits([61, 3], (len(batch), hq, d), "f16")
    dev = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.float16).cuda()
    q, kc, vc = dev(qb), dev(kb), dev(vb)
    t, cl = torch.from_numpy(tables).cuda(), torch.from_numpy(ctx).cuda()
    g = groups.to("cuda")
    ws = pa.cascade_workspace(len(batch), hq, hkv, d, int(ctx.max()), tables.shape[1], g)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    scale = 1 / np.sqrt(d)
    assert L.lib().pa_test_stall_next_decode(LIMIT_NS) == L.PA_OK
    pa.pa_paged_decode_cascade(out, q, kc, vc, t, cl, int(ctx.max()), scale, g, ws, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_WAIT_TIMEOUT, "the stalled wait was not reported"
    err.zero_()
    pa.pa_paged_decode_cascade(out, q, kc, vc, t, cl, int(ctx.max()), scale, g, ws, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = oracle_decode(qb, kb, vb, tables, ctx, scale, "f16")
    assert_close(out_to_f64(out, "f16"), want, "cascade after a timed-out launch")

