"""E4M3 (8-bit) KV cache on a B200 against the oracle: cache-write codes bit for
bit (every finite 16-bit input value, scales where float32 division matters,
saturation), decode over the 8-bit cache within the float tolerance on every
arithmetic path (1, 2 query heads per KV head on CUDA cores; 4, 8 on tensor
cores), split-KV and ragged contexts, NaN codes past the context ignored, and
whole-block copies and swaps of 8-bit pools bit for bit."""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_352_b200 as pa
from oracle import cache_ops as OC
from oracle import fp8 as F
from tests.parity import assert_close, out_to_f64
from workloads import gen

pytestmark = pytest.mark.gpu

TDT = {"f16": torch.float16, "bf16": torch.bfloat16}


def _dev16(bits, dt):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(TDT[dt]).cuda()


@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("scales", [(1.0, 1.0), (0.11, 1.3), (0.02, 7.5)])
def test_cache_write_codes_every_value(dt, scales):
    hkv, d = 2, 64
    top = 0x7C00 if dt == "f16" else 0x7F80
    pos = np.arange(0, top, dtype=np.uint16)
    vals = np.concatenate([pos, pos | 0x8000])            # every finite value, both signs
    per = hkv * d
    vals = np.concatenate([vals, np.zeros((-len(vals)) % per, np.uint16)])
    T = len(vals) // per
    key = vals.reshape(T, hkv, d)
    value = np.roll(vals, 777).reshape(T, hkv, d)
    nb = -(-T // 16) + 3
    rng = np.random.default_rng(5)
    slots = rng.permutation(nb * 16)[:T].astype(np.int64)
    slots[::97] = -1                                      # some tokens are not stored
    kc = torch.full((nb, hkv, 16, d), 0x55, dtype=torch.uint8, device="cuda")
    vc = torch.full_like(kc, 0x55)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_reshape_and_cache_fp8(_dev16(key, dt), _dev16(value, dt), kc, vc,
                                torch.from_numpy(slots).cuda(), scales[0], scales[1], dev_error=err)
    torch.cuda.synchronize()
    ok = np.full((nb, hkv, 16, d), 0x55, np.uint8)
    ov = ok.copy()
    F.reshape_and_cache_fp8(ok, ov, key, value, slots, 16, dt, scales[0], scales[1])
    assert int(err.item()) == 0
    assert np.array_equal(kc.cpu().numpy(), ok) and np.array_equal(vc.cpu().numpy(), ov)


def _case(seed, B, hq, hkv, d, dt, max_ctx, nb, nan_fill=True):
    rng = np.random.default_rng(seed)
    ctx = rng.integers(1, max_ctx + 1, B).astype(np.int32)
    ctx[0] = 0 if B > 2 else ctx[0]
    ctx[1 % B] = 1
    mb = max(1, int(max(-(-c // 16) for c in ctx)))
    order = rng.permutation(nb)
    tables = np.full((B, mb), -1, np.int32)
    k = 0
    for s in range(B):
        n = -(-int(ctx[s]) // 16)
        tables[s, :n] = order[k:k + n]
        k += n
    assert k <= nb
    codes = rng.integers(0, 256, (2, nb, hkv, 16, d)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x31
    if nan_fill:
        # slots past each context hold NaN codes: decode must never read them
        for s in range(B):
            n = int(ctx[s])
            if n % 16:
                codes[:, tables[s, n // 16], :, n % 16:, :] = 0x7F
    q = gen.normal_bits([seed, 2], (B, hq, d), dt)
    return ctx, tables, codes[0], codes[1], q


@pytest.mark.parametrize("hq,hkv,d,dt", [(4, 4, 64, "f16"), (8, 4, 128, "bf16"),
                                          (6, 6, 128, "bf16"), (8, 4, 64, "bf16"),
                                          (6, 3, 128, "f16"),
                                          (16, 4, 128, "bf16"), (16, 2, 64, "f16"),
                                          (32, 4, 128, "f16")])
@pytest.mark.parametrize("partition_tokens", [0, 64])
def test_decode_fp8_matches_oracle(hq, hkv, d, dt, partition_tokens):
    B, nb = 7, 220
    ctx, tables, kc8, vc8, q = _case(hq * 31 + d, B, hq, hkv, d, dt, 400, nb)
    ks, vs = 0.07, 0.013
    scale = 1 / math.sqrt(d)
    want = F.paged_decode_fp8(q, kc8, vc8, tables, ctx, scale, ks, vs, dt)
    out = torch.empty(B, hq, d, dtype=TDT[dt], device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = pa.decode_workspace(B, hq, hkv, d, int(ctx.max()), partition_tokens)
    order = torch.from_numpy(pa.pa_longest_first_order(ctx)).cuda()
    pa.pa_paged_decode_fp8(out, _dev16(q, dt), torch.from_numpy(kc8).cuda(),
                           torch.from_numpy(vc8).cuda(), torch.from_numpy(tables).cuda(),
                           torch.from_numpy(ctx).cuda(), int(ctx.max()), scale, ks, vs,
                           partition_tokens=partition_tokens, workspace=ws, dev_error=err,
                           seq_order=order)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = out_to_f64(out, dt)
    for s in range(B):
        assert_close(got[s], want[s], f"seq {s} ctx {ctx[s]}")


@pytest.mark.parametrize("hq,hkv", [(8, 4), (16, 4)])
def test_decode_fp8_bf16_queries_beyond_half_range(hq, hkv):
    """bf16 query rows whose largest magnitude is far above 2^15 (N(0,1) times
    2^16, exact in bf16) with the softmax scale shrunk by 2^-16: both 8-bit paths
    (2 query heads per KV head on CUDA cores, 4 on tensor cores) hold the query
    in half precision and must bring such rows into range by a power of two. The
    logits equal those of the unscaled queries, so the oracle's values are of
    ordinary size."""
    B, nb, d, dt = 5, 160, 128, "bf16"
    ctx, tables, kc8, vc8, q = _case(917 + hq, B, hq, hkv, d, dt, 300, nb)
    qf = torch.from_numpy(np.ascontiguousarray(q).view(np.int16)).view(torch.bfloat16).float()
    big = (qf * 65536.0).to(torch.bfloat16)
    assert float(big.float().abs().amax(dim=-1).min()) >= 32768.0
    q_big = big.view(torch.int16).numpy().view(np.uint16)
    ks, vs = 0.05, 0.02
    scale = 1 / math.sqrt(d) / 65536.0
    want = F.paged_decode_fp8(q_big, kc8, vc8, tables, ctx, scale, ks, vs, dt)
    out = torch.empty(B, hq, d, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = pa.decode_workspace(B, hq, hkv, d, int(ctx.max()), 0)
    pa.pa_paged_decode_fp8(out, big.cuda(), torch.from_numpy(kc8).cuda(),
                           torch.from_numpy(vc8).cuda(), torch.from_numpy(tables).cuda(),
                           torch.from_numpy(ctx).cuda(), int(ctx.max()), scale, ks, vs,
                           workspace=ws, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = out_to_f64(out, dt)
    for s in range(B):
        assert_close(got[s], want[s], f"seq {s} ctx {ctx[s]}")


def test_quantize_then_decode_end_to_end():
    """Keys/values written by the fp8 cache write, then decoded, against the oracle's
    write and decode of the same 16-bit inputs; also the quantization error of the
    whole path against 16-bit decode stays small."""
    hq, hkv, d, dt = 32, 8, 128, "bf16"
    B, nb = 5, 300
    rng = np.random.default_rng(8)
    ctx = rng.integers(50, 700, B).astype(np.int32)
    order = rng.permutation(nb)
    mb = int(max(-(-c // 16) for c in ctx))
    tables = np.full((B, mb), -1, np.int32)
    slots, k = [], 0
    for s in range(B):
        n = -(-int(ctx[s]) // 16)
        tables[s, :n] = order[k:k + n]
        k += n
        slots += [int(tables[s, p // 16]) * 16 + p % 16 for p in range(int(ctx[s]))]
    T = len(slots)
    key = gen.normal_bits([81, 1], (T, hkv, d), dt)
    val = gen.normal_bits([81, 2], (T, hkv, d), dt)
    ks = vs = 4.0 / 448
    sl = torch.tensor(slots, dtype=torch.int64, device="cuda")
    kc = torch.zeros(nb, hkv, 16, d, dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    pa.pa_reshape_and_cache_fp8(_dev16(key, dt), _dev16(val, dt), kc, vc, sl, ks, vs)
    ok = np.zeros((nb, hkv, 16, d), np.uint8)
    ov = np.zeros_like(ok)
    F.reshape_and_cache_fp8(ok, ov, key, val, np.array(slots), 16, dt, ks, vs)
    q = gen.normal_bits([81, 3], (B, hq, d), dt)
    out = torch.empty(B, hq, d, dtype=TDT[dt], device="cuda")
    scale = 1 / math.sqrt(d)
    pa.pa_paged_decode_fp8(out, _dev16(q, dt), kc, vc, torch.from_numpy(tables).cuda(),
                           torch.from_numpy(ctx).cuda(), int(ctx.max()), scale, ks, vs,
                           workspace=pa.decode_workspace(B, hq, hkv, d, int(ctx.max())))
    torch.cuda.synchronize()
    assert np.array_equal(kc.cpu().numpy(), ok) and np.array_equal(vc.cpu().numpy(), ov)
    want = F.paged_decode_fp8(q, ok, ov, tables, ctx, scale, ks, vs, dt)
    got = out_to_f64(out, dt)
    for s in range(B):
        assert_close(got[s], want[s], f"seq {s}")
    # the 16-bit cache of the same inputs, for the size of the quantization error
    k16 = np.zeros((nb, hkv, 16, d), np.uint16)
    v16 = np.zeros_like(k16)
    OC.reshape_and_cache(k16, v16, key, val, np.array(slots), 16)
    from oracle.attention import paged_decode
    exact = paged_decode(q, k16, v16, tables, ctx, scale, dt)
    rel = np.linalg.norm(got - exact) / np.linalg.norm(exact)
    assert rel < 0.1, rel


def test_copy_and_swap_fp8_pools():
    nb, hkv, d = 40, 4, 128
    rng = np.random.default_rng(2)
    kc = torch.from_numpy(rng.integers(0, 256, (nb, hkv, 16, d)).astype(np.uint8)).cuda()
    vc = torch.from_numpy(rng.integers(0, 256, (nb, hkv, 16, d)).astype(np.uint8)).cuda()
    ok, ov = kc.cpu().numpy(), vc.cpu().numpy()
    pairs = [(3, 30), (7, 8), (0, 39)]
    pa.pa_copy_blocks(kc, vc, pairs)
    OC.copy_blocks(ok, ov, pairs)
    hk = torch.zeros(10, hkv, 16, d, dtype=torch.uint8).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    pa.pa_swap_blocks(kc, vc, hk, hv, [(30, 2), (39, 9)])
    torch.cuda.synchronize()
    assert np.array_equal(kc.cpu().numpy(), ok) and np.array_equal(vc.cpu().numpy(), ov)
    assert np.array_equal(hk[2].numpy(), ok[30]) and np.array_equal(hv[9].numpy(), ov[39])
    pa.pa_swap_blocks(hk, hv, kc, vc, [(2, 11)])
    torch.cuda.synchronize()
    assert np.array_equal(kc[11].cpu().numpy(), ok[30])


def test_fp8_argument_checks():
    kc = torch.zeros(4, 2, 16, 64, dtype=torch.uint8, device="cuda")
    key = torch.zeros(3, 2, 64, dtype=torch.float16, device="cuda")
    sl = torch.zeros(3, dtype=torch.int64, device="cuda")
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(pa.PAError):
            pa.pa_reshape_and_cache_fp8(key, key, kc, kc.clone(), sl, bad, 1.0)
    with pytest.raises(pa.PAError):
        pa.pa_reshape_and_cache(key, key, kc, kc.clone(), sl)   # 16-bit entry, 8-bit cache


def test_warp_split_two_block_steps_with_bad_ids():
    """A batch that takes the warp-per-partition split over 8 query heads per KV
    head, whose loop takes two blocks per step: contexts of 3841..4096 tokens
    (16 partitions of 256 tokens, the last ones ragged), one out-of-range block id
    as the second block of a pair and one as the first. The bad ids are flagged,
    nothing faults, and every other sequence matches the oracle."""
    B, hq, hkv, d, dt, pt = 64, 32, 4, 128, "bf16", 256
    rng = np.random.default_rng(21)
    ctx = rng.integers(3841, 4097, B).astype(np.int32)
    _, parts, launches = pa.pa_paged_decode_plan(B, hq, hkv, d, int(ctx.max()), pt)
    assert parts == 16 and launches == 2, "this batch should take the warp-per-partition split"
    mb = int(-(-ctx.max() // 16))
    nb = int(sum(-(-int(c) // 16) for c in ctx))
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((B, mb), -1, np.int32)
    used = 0
    for s in range(B):
        n = -(-int(ctx[s]) // 16)
        tables[s, :n] = perm[used:used + n]
        used += n
    codes = rng.integers(0, 256, (2, nb, hkv, 16, d)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3A
    q = gen.normal_bits([21, 2], (B, hq, d), dt)
    bad = tables.copy()
    bad[5, 3] = nb + 7         # the second block of a pair (blocks 2 and 3)
    bad[6, 18] = 1 << 30       # the first block of a pair in the second partition
    ks, vs, scale = 0.04, 0.015, 1 / math.sqrt(d)
    out = torch.empty(B, hq, d, dtype=TDT[dt], device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = pa.decode_workspace(B, hq, hkv, d, int(ctx.max()), pt)
    pa.pa_paged_decode_fp8(out, _dev16(q, dt), torch.from_numpy(codes[0]).cuda(),
                           torch.from_numpy(codes[1]).cuda(), torch.from_numpy(bad).cuda(),
                           torch.from_numpy(ctx).cuda(), int(ctx.max()), scale, ks, vs,
                           partition_tokens=pt, workspace=ws, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_BLOCK_RANGE
    got = out_to_f64(out, dt)
    check = [0, 1, 4, 7, 63]
    want = F.paged_decode_fp8(q[check], codes[0], codes[1], tables[check], ctx[check], scale,
                              ks, vs, dt)
    for i, s in enumerate(check):
        assert_close(got[s], want[i], f"seq {s} ctx {ctx[s]}")
