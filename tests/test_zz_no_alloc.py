"""pa_paged_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers may not allocate device memory: a plugin whose host runtime owns
every allocation, or a latency-critical loop that must never reach cudaMalloc.
For them, pa_paged_decode_noalloc takes its split-KV scratch from an array
built into the library, so the caller passes only inputs and outputs.

This file is named so that pytest collects it last. The checks, through the C
interface on a GPU:
  * on two calls in a row, the output matches the float64 oracle within the
    parity tolerance used everywhere else, and matches pa_paged_decode with a
    caller-owned workspace;
  * a batch that takes the warp-per-partition split (streaming kernel plus the
    separate merge kernel, which reads the scratch in its own layout) matches too;
  * a small batch and then a much larger one: the second call's merge counters
    cover scratch bytes where the first call left partition results, so the
    call's own clearing of the counters is what keeps it right;
  * a scheduling order, and a batch short enough to need no scratch at all;
  * a batch too large for the built-in array, and a buffer that is not device
    memory, are refused with a clear error before anything is launched.
"""

import ctypes

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


class _Case:
    """A seeded batch: random K/V pools, queries and block tables over a shuffled
    pool, as 16-bit patterns (for the oracle) and as device tensors."""

    def __init__(self, ctx, hq, hkv, d=128, dtype="f16", seed=3):
        self.ctx = np.asarray(ctx, np.int32)
        self.hq, self.hkv, self.d, self.dtype = hq, hkv, d, dtype
        nblk = [-(-int(c) // 16) for c in self.ctx]
        nb = sum(nblk) + 8
        self.kb = gen.normal_bits([seed, 1], (nb, hkv, 16, d), dtype)
        self.vb = gen.normal_bits([seed, 2], (nb, hkv, 16, d), dtype)
        self.qb = gen.normal_bits([seed, 3], (len(ctx), hq, d), dtype)
        perm = np.random.default_rng([seed, 4]).permutation(nb).astype(np.int32)
        self.tables = np.full((len(ctx), max(nblk)), -1, np.int32)
        used = 0
        for s, n in enumerate(nblk):
            self.tables[s, :n] = perm[used:used + n]
            used += n
        dev = lambda b: torch.from_numpy(b.view(np.int16)).view(_TORCH[dtype]).cuda()
        self.q, self.kc, self.vc = dev(self.qb), dev(self.kb), dev(self.vb)
        self.t = torch.from_numpy(self.tables).cuda()
        self.cl = torch.from_numpy(self.ctx).cuda()
        self.scale = 1.0 / np.sqrt(d)

    @property
    def max_ctx(self):
        return int(self.ctx.max())

    def oracle(self):
        return oracle_decode(self.qb, self.kb, self.vb, self.tables, self.ctx, self.scale,
                             self.dtype)

    def noalloc(self, pt, err, seq_order=None):
        out = torch.full_like(self.q, float("nan"))
        L.pa_paged_decode_noalloc(out, self.q, self.kc, self.vc, self.t, self.cl, self.max_ctx,
                                  self.scale, pt, err, seq_order=seq_order)
        torch.cuda.synchronize()
        return out

    def with_workspace(self, pt):
        out = torch.empty_like(self.q)
        ws = pa.decode_workspace(len(self.ctx), self.hq, self.hkv, self.d, self.max_ctx, pt)
        pa.pa_paged_decode(out, self.q, self.kc, self.vc, self.t, self.cl, self.max_ctx,
                           self.scale, pt, ws)
        torch.cuda.synchronize()
        return out


def _check(case, out, what):
    assert_close(out_to_f64(out, case.dtype), case.oracle(), what)


def test_noalloc_matches_oracle_and_workspace_decode_twice_in_a_row():
    case = _Case([3000, 17, 1200, 700, 2049, 1], hq=8, hkv=2)   # several split sequences
    pt = 256
    need = pa.pa_paged_decode_workspace_size(6, 8, 2, 128, case.max_ctx, 16, pt)
    assert 0 < need <= L.NOALLOC_WORKSPACE_BYTES
    ref = case.with_workspace(pt)
    want = case.oracle()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out = case.noalloc(pt, err)
        assert err.item() == 0
        assert_close(out_to_f64(out, "f16"), want, "noalloc vs oracle")
        assert_close(out_to_f64(out, "f16"), out_to_f64(ref, "f16"), "noalloc vs workspace")


def test_noalloc_warp_per_partition_split():
    """64 sequences x 4 KV heads with 16 partitions of 256 tokens: the split that
    streams one partition per warp and merges in a second kernel."""
    ctx = np.random.default_rng(5).integers(3841, 4097, 64)
    case = _Case(ctx, hq=8, hkv=4, dtype="bf16", seed=7)
    pt = 256
    _, parts, launches = pa.pa_paged_decode_plan(64, 8, 4, 128, case.max_ctx, pt)
    assert parts == 16 and launches == 2, "this batch should take the warp-per-partition split"
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out = case.noalloc(pt, err)
        assert err.item() == 0
        _check(case, out, "noalloc, warp-per-partition split")


def test_noalloc_small_then_large_batch_clears_stale_counters():
    """The first call leaves partition maxima and sums in the scratch right after
    its 8 counters; the second call's 192 counters cover those bytes. Both calls
    merge in the last CTA of each (sequence, KV head), which trusts the counters."""
    pt = 256
    small = _Case([600, 1000, 800, 999], hq=8, hkv=2, seed=11)
    large = _Case(np.random.default_rng(12).integers(520, 1001, 96), hq=8, hkv=2, seed=13)
    for c in (small, large):
        _, parts, launches = pa.pa_paged_decode_plan(len(c.ctx), 8, 2, 128, c.max_ctx, pt)
        assert parts >= 3 and launches == 1         # the last-CTA merge
    # scratch layout: [units] int counters, then (256-aligned) the partition maxima
    units_small, units_large = 4 * 2, 96 * 2
    ml_off_small = -(-units_small * 4 // 256) * 256
    assert units_large * 4 > ml_off_small + 64      # the counters reach the stale floats
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(small, small.noalloc(pt, err), "noalloc, small batch")
    _check(large, large.noalloc(pt, err), "noalloc, larger batch after a smaller one")
    _check(small, small.noalloc(pt, err), "noalloc, small batch again")
    assert err.item() == 0


def test_noalloc_with_a_scheduling_order():
    case = _Case([90, 2500, 16, 1333, 4000, 640, 1], hq=16, hkv=2, dtype="bf16", seed=17)
    order = torch.from_numpy(pa.pa_longest_first_order(case.ctx)).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out = case.noalloc(512, err, seq_order=order)
        assert err.item() == 0
        _check(case, out, "noalloc with seq_order")


def test_noalloc_batch_that_needs_no_scratch():
    case = _Case([300, 17, 512, 1], hq=4, hkv=4, seed=19)
    assert pa.pa_paged_decode_workspace_size(4, 4, 4, 128, case.max_ctx, 16, 0) == 0
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(case, case.noalloc(0, err), "noalloc without scratch")
    assert err.item() == 0


def test_noalloc_refuses_batches_beyond_the_builtin_scratch():
    # 64 sequences x 8 KV heads x 64 partitions x 8 query heads x 130 floats > 16 MiB
    B, hq, hkv, d = 64, 64, 8, 128
    need = pa.pa_paged_decode_workspace_size(B, hq, hkv, d, 64 * 512, 16, 512)
    assert need > L.NOALLOC_WORKSPACE_BYTES
    q = torch.zeros(B, hq, d, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(4, hkv, 16, d, dtype=torch.bfloat16, device="cuda")
    tables = torch.zeros(B, 1, dtype=torch.int32, device="cuda")
    cl = torch.ones(B, dtype=torch.int32, device="cuda")
    with pytest.raises(pa.PAError) as e:
        L.pa_paged_decode_noalloc(torch.empty_like(q), q, kc, kc, tables, cl, 64 * 512, 0.1, 512)
    assert e.value.code == L.PA_ERR_UNSUPPORTED
    assert "scratch" in str(e.value)


def test_noalloc_refuses_memory_that_is_not_on_the_device():
    """A host buffer passed as the output (through the C interface directly) is
    refused before any launch: the library checks every buffer's device."""
    case = _Case([100, 40], hq=4, hkv=2, seed=23)
    host_out = np.zeros(case.q.numel() * 2, np.uint8)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = L.lib().pa_paged_decode_noalloc(
        ctypes.c_void_p(host_out.ctypes.data), p(case.q), p(case.kc), p(case.vc), p(case.t),
        case.tables.shape[1], p(case.cl), None, 2, case.max_ctx, 4, 2, 128, 16,
        case.kb.shape[0], float(case.scale), 0, None, L.PA_F16,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == L.PA_ERR_INVALID_ARG
    assert "out is not device memory" in L.last_error()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(case, case.noalloc(0, err), "noalloc after a refused call")
