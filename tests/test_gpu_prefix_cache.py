"""Prefix caching across requests on a B200: a later request sharing a prompt
prefix reuses the cached blocks, writes only its own tokens, and decodes to the
oracle's result over its logical keys and values; tables match the oracle's
block manager bit for bit."""

import math

import numpy as np
import pytest
import torch

from oracle import block_manager as OBM
from oracle.attention import softmax_attention
from oracle.fpbits import bits_to_f64
import paged_kv_cache_352_b200 as pa
from tests.parity import assert_close, out_to_f64
from workloads import gen

pytestmark = pytest.mark.gpu


def test_cached_prefix_requests_decode_like_full_prompts():
    rng = np.random.default_rng(31)
    nb, hkv, hq, d, dt = 512, 8, 32, 128, "bf16"
    torch_dt = torch.bfloat16
    kc = torch.zeros(nb, hkv, 16, d, dtype=torch_dt, device="cuda")
    vc = torch.zeros_like(kc)
    order = rng.permutation(nb)
    cbm = pa.BlockManager(nb, 16, order)
    obm = OBM.BlockManager(nb, 16, order)
    system = rng.integers(0, 32000, 600).tolist()        # shared system prompt
    # K/V of a token depend on its whole prefix; with the same prefix they are the
    # same, so request r's keys/values = the system prompt's followed by its own
    sys_k, sys_v = gen.seq_kv_bits(77, 0, 600, hkv, d, dt)
    reqs, written = [], 0
    for r in range(5):
        own = rng.integers(0, 32000, int(rng.integers(1, 90))).tolist()
        toks = system + own
        ok, ov = gen.seq_kv_bits(77, 1 + r, len(own), hkv, d, dt)
        K = np.concatenate([sys_k, ok])
        V = np.concatenate([sys_v, ov])
        slots, cached = cbm.add_seq_cached(r, toks)
        oslots, ocached = obm.add_seq_cached(r, toks)
        assert list(slots) == oslots and cached == ocached
        assert cached == (0 if r == 0 else 592)          # 37 full blocks of the prompt
        kt = torch.from_numpy(K[cached:]).view(torch_dt).cuda()
        vt = torch.from_numpy(V[cached:]).view(torch_dt).cuda()
        pa.pa_reshape_and_cache(kt, vt, kc, vc, torch.from_numpy(slots[cached:]).cuda())
        written += len(toks) - cached
        reqs.append((toks, K, V))
    ctx = np.array([len(t) for t, _, _ in reqs], np.int32)
    mb = int(max(-(-c // 16) for c in ctx))
    tables = cbm.block_tables(range(5), mb)
    assert np.array_equal(tables, obm.block_tables(range(5), mb))
    q = gen.query_bits(77, 5, hq, d, dt)
    out = torch.empty(5, hq, d, dtype=torch_dt, device="cuda")
    cl = torch.from_numpy(ctx).cuda()
    pa.pa_paged_decode(out, torch.from_numpy(q).view(torch_dt).cuda(), kc, vc,
                       torch.from_numpy(tables).cuda(), cl, int(ctx.max()), 1 / math.sqrt(d), 0,
                       pa.decode_workspace(5, hq, hkv, d, int(ctx.max())),
                       seq_order=torch.from_numpy(pa.pa_longest_first_order(ctx)).cuda())
    torch.cuda.synchronize()
    got = out_to_f64(out, dt)
    for r, (toks, K, V) in enumerate(reqs):
        ref = np.stack([softmax_attention(bits_to_f64(q[r, h], dt),
                                          bits_to_f64(K[:, h // 4], dt),
                                          bits_to_f64(V[:, h // 4], dt), 1 / math.sqrt(d))
                        for h in range(hq)])
        assert_close(got[r], ref, f"request {r}")
    assert written < sum(len(t) for t, _, _ in reqs) - 4 * 592 + 1
