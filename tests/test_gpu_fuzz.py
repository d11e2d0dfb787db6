"""Seeded random shapes through pa_paged_decode, pa_paged_decode_fp8 and
pa_paged_decode_cascade on a B200 against the oracle: every head layout (1..8
query heads per KV head), both head dimensions and query types, 16-bit and E4M3
caches, ragged contexts with the edge lengths (0, 1, 15, 16, 17) mixed in,
caller-chosen and library partitions, with and without a scheduling order, NaN
patterns in the slots past each context; for the cascade, random fork forests
under every supported (group size, query heads per KV head) pair. Each case is
generated from its own seed, so a failure names a reproducible shape."""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_352_b200 as pa
from oracle import fp8 as F
from oracle.attention import paged_decode
from tests.parity import assert_close, out_to_f64
from tests.test_gpu_cascade import _forest, _run
from workloads import gen

pytestmark = pytest.mark.gpu

TDT = {"f16": torch.float16, "bf16": torch.bfloat16}
NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0}


def _dev16(bits, dt):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(TDT[dt]).cuda()


def _shape(seed):
    rng = np.random.default_rng([352, seed])
    d = int(rng.choice([64, 128]))
    dt = str(rng.choice(["f16", "bf16"]))
    G = int(rng.choice([1, 2, 4, 8]))
    hkv = int(rng.choice([1, 2, 4, 8]))
    B = int(rng.integers(1, 13))
    ctx = rng.integers(0, 1300, B)
    edges = np.array([0, 1, 15, 16, 17])
    k = int(rng.integers(0, min(B, 3) + 1))
    ctx[rng.choice(B, size=k, replace=False)] = rng.choice(edges, size=k)
    pt = int(rng.choice([0, 16, 48, 128, 512]))
    order = str(rng.choice(["none", "longest", "random"]))
    fp8 = bool(rng.integers(0, 2))
    return rng, d, dt, G, hkv, B, ctx.astype(np.int32), pt, order, fp8


@pytest.mark.parametrize("seed", range(96))
def test_random_shape_matches_oracle(seed):
    rng, d, dt, G, hkv, B, ctx, pt, order, fp8 = _shape(seed)
    hq = hkv * G
    nblk = [-(-int(c) // 16) for c in ctx]
    mb = max(1, max(nblk))
    nb = sum(nblk) + 3
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((B, mb), -1, np.int32)
    used = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = perm[used:used + n]
        used += n
    q = gen.normal_bits([seed, 1], (B, hq, d), dt)
    scale = 1 / math.sqrt(d)
    maxctx = int(ctx.max())
    seq_order = None
    if order == "longest":
        seq_order = torch.from_numpy(pa.pa_longest_first_order(ctx)).cuda()
    elif order == "random":
        seq_order = torch.from_numpy(rng.permutation(B).astype(np.int32)).cuda()
    out = torch.empty(B, hq, d, dtype=TDT[dt], device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = pa.decode_workspace(B, hq, hkv, d, maxctx, pt)
    td, cd = torch.from_numpy(tables).cuda(), torch.from_numpy(ctx).cuda()
    if fp8:
        codes = rng.integers(0, 256, (2, nb, hkv, 16, d)).astype(np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0x29
        for s, c in enumerate(ctx):      # NaN codes past each context
            if c % 16:
                codes[:, tables[s, c // 16], :, c % 16:, :] = 0x7F
        # The 8-bit path rounds P to half precision (relative 2^-11), so its
        # absolute error grows with |V|; value scales keep |V| <= ~6 (448 x
        # 0.013), the size of value row the tolerance is stated for.
        ks, vs = float(rng.uniform(0.01, 0.1)), float(rng.uniform(0.002, 0.013))
        pa.pa_paged_decode_fp8(out, _dev16(q, dt), torch.from_numpy(codes[0]).cuda(),
                               torch.from_numpy(codes[1]).cuda(), td, cd, maxctx, scale, ks, vs,
                               partition_tokens=pt, workspace=ws, dev_error=err,
                               seq_order=seq_order)
        want = F.paged_decode_fp8(q, codes[0], codes[1], tables, ctx, scale, ks, vs, dt)
    else:
        kb = gen.normal_bits([seed, 2], (nb, hkv, 16, d), dt)
        vb = gen.normal_bits([seed, 3], (nb, hkv, 16, d), dt)
        for s, c in enumerate(ctx):      # NaN patterns past each context
            if c % 16:
                kb[tables[s, c // 16], :, c % 16:, :] = NAN_BITS[dt]
                vb[tables[s, c // 16], :, c % 16:, :] = NAN_BITS[dt]
        pa.pa_paged_decode(out, _dev16(q, dt), _dev16(kb, dt), _dev16(vb, dt), td, cd, maxctx,
                           scale, pt, ws, err, seq_order=seq_order)
        want = paged_decode(q, kb, vb, tables, ctx, scale, dt)
    torch.cuda.synchronize()
    what = (f"seed {seed}: d{d} {dt} G{G} hkv{hkv} B{B} pt{pt} order {order} "
            f"{'e4m3' if fp8 else '16-bit'}")
    assert int(err.item()) == 0, what
    got = out_to_f64(out, dt)
    for s in range(B):
        assert_close(got[s], want[s], f"{what} seq {s} ctx {ctx[s]}")


@pytest.mark.parametrize("seed", range(6))
def test_random_warp_split_batch_matches_oracle(seed):
    """Larger random batches that take the warp-per-partition split (short
    partitions over a grid of at least 1024 CTAs; two blocks per loop step over
    E4M3 caches at 8 query heads per KV head), checked on sampled sequences."""
    rng = np.random.default_rng([353, seed])
    d, dt = 128, str(rng.choice(["f16", "bf16"]))
    hkv, G = 4, [1, 4, 8][seed % 3]
    hq, B, pt = hkv * G, 64, 128
    ctx = rng.integers(1000, 2201, B).astype(np.int32)
    fp8 = seed >= 3
    assert pa.pa_paged_decode_plan(B, hq, hkv, d, int(ctx.max()), pt)[2] == 2, "not the warp split"
    nblk = [-(-int(c) // 16) for c in ctx]
    mb, nb = max(nblk), sum(nblk)
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((B, mb), -1, np.int32)
    used = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = perm[used:used + n]
        used += n
    q = gen.normal_bits([seed, 11], (B, hq, d), dt)
    scale = 1 / math.sqrt(d)
    out = torch.empty(B, hq, d, dtype=TDT[dt], device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = pa.decode_workspace(B, hq, hkv, d, int(ctx.max()), pt)
    td, cd = torch.from_numpy(tables).cuda(), torch.from_numpy(ctx).cuda()
    check = sorted(set(rng.choice(B, 4, replace=False).tolist()) | {int(np.argmax(ctx))})
    if fp8:
        codes = np.frombuffer(rng.bytes(2 * nb * hkv * 16 * d), np.uint8).reshape(
            2, nb, hkv, 16, d).copy()
        codes[(codes & 0x7F) == 0x7F] = 0x29
        ks, vs = 0.04, 0.013
        pa.pa_paged_decode_fp8(out, _dev16(q, dt), torch.from_numpy(codes[0]).cuda(),
                               torch.from_numpy(codes[1]).cuda(), td, cd, int(ctx.max()), scale,
                               ks, vs, partition_tokens=pt, workspace=ws, dev_error=err)
        want = F.paged_decode_fp8(q[check], codes[0], codes[1], tables[check], ctx[check], scale,
                                  ks, vs, dt)
    else:
        kb = gen.normal_bits([seed, 12], (nb, hkv, 16, d), dt)
        vb = gen.normal_bits([seed, 13], (nb, hkv, 16, d), dt)
        pa.pa_paged_decode(out, _dev16(q, dt), _dev16(kb, dt), _dev16(vb, dt), td, cd,
                           int(ctx.max()), scale, pt, ws, err)
        want = paged_decode(q[check], kb, vb, tables[check], ctx[check], scale, dt)
    torch.cuda.synchronize()
    what = f"seed {seed}: {dt} G{G} hkv{hkv} {'e4m3' if fp8 else '16-bit'}"
    assert int(err.item()) == 0, what
    got = out_to_f64(out, dt)
    for i, s in enumerate(check):
        assert_close(got[s], want[i], f"{what} seq {s} ctx {ctx[s]}")


# (query heads per KV head, group size): every pair whose stacked rows (their
# product) are 1, 2, 4 or 8; 8 runs both decodes in one launch
CASCADE_LAYOUTS = [(1, 1), (1, 2), (1, 4), (1, 8), (2, 1), (2, 2), (2, 4), (4, 1), (4, 2),
                   (8, 1)]


@pytest.mark.parametrize("seed", range(24))
def test_random_cascade_matches_oracle(seed):
    """Random fork forests (prompts forked into samples that append their own
    tokens, or prompts of whole blocks with no own tokens, plus an empty
    sequence) through the cascade: every output row within tolerance of the
    oracle's decode over the whole context, and no device error."""
    rng = np.random.default_rng([355, seed])
    G, gs = CASCADE_LAYOUTS[seed % len(CASCADE_LAYOUTS)]
    hkv = int(rng.choice([1, 2, 4, 8]))
    d = int(rng.choice([64, 128]))
    dt = str(rng.choice(["f16", "bf16"]))
    exact = bool(rng.integers(0, 4) == 0)
    order = [None, "cascade", "random"][int(rng.integers(0, 3))]
    fp8 = None
    if rng.integers(0, 2):
        fp8 = (float(rng.uniform(0.02, 0.08)), float(rng.uniform(0.004, 0.013)))
    nb = 1200
    bm, batch, ctx = _forest(int(rng.integers(1 << 30)), nb, exact=exact)
    err, groups = _run(bm, batch, ctx, hkv * G, hkv, d, dt, nb, seed, gs, fp8=fp8, order=order)
    assert err == 0, (f"seed {seed}: G{G} group size {gs} hkv{hkv} d{d} {dt} order {order} "
                      f"fp8 {fp8}: device error {err}")
