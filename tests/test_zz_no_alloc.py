"""pa_paged_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers may not allocate device memory: a plugin whose host runtime owns
every allocation, or a latency-critical loop that must never reach cudaMalloc.
For them, pa_paged_decode_noalloc takes its split-KV scratch from an array
built into the library, so the caller passes only inputs and outputs.

This file is named so that pytest collects it last. The checks, through the C
interface on a GPU:
  * on two calls in a row, the output matches pa_paged_decode with a
    caller-owned workspace, within the parity tolerance used everywhere else;
  * a batch too large for the built-in array is refused with a clear error.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_352_b200 as pa
from paged_kv_cache_352_b200 import _lib as L
from tests.parity import assert_close, out_to_f64

pytestmark = pytest.mark.gpu


def _case(ctx, hq=8, hkv=2, d=128, dtype=torch.float16, nb=512, seed=3):
    g = torch.Generator().manual_seed(seed)
    kc = torch.randn(nb, hkv, 16, d, generator=g).to(dtype).cuda()
    vc = torch.randn(nb, hkv, 16, d, generator=g).to(dtype).cuda()
    q = torch.randn(len(ctx), hq, d, generator=g).to(dtype).cuda()
    perm = torch.randperm(nb, generator=g)
    mb = max(-(-c // 16) for c in ctx)
    tables = torch.full((len(ctx), mb), -1, dtype=torch.int32)
    used = 0
    for s, c in enumerate(ctx):
        n = -(-c // 16)
        tables[s, :n] = perm[used:used + n].to(torch.int32)
        used += n
    return q, kc, vc, tables.cuda(), torch.tensor(ctx, dtype=torch.int32).cuda()


def test_noalloc_matches_workspace_decode_twice_in_a_row():
    ctx = [3000, 17, 1200, 700, 2049, 1]          # several sequences split into partitions
    q, kc, vc, tables, cl = _case(ctx)
    pt, scale = 256, 0.088
    ref = torch.empty_like(q)
    ws = pa.decode_workspace(len(ctx), 8, 2, 128, max(ctx), pt)
    assert ws is not None and ws.numel() <= L.NOALLOC_WORKSPACE_BYTES
    pa.pa_paged_decode(ref, q, kc, vc, tables, cl, max(ctx), scale, pt, ws)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        L.pa_paged_decode_noalloc(out, q, kc, vc, tables, cl, max(ctx), scale, pt, err)
        torch.cuda.synchronize()
        assert err.item() == 0
        assert_close(out_to_f64(out, "f16"), out_to_f64(ref, "f16"), "noalloc vs workspace")


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
