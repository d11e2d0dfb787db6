"""CUDA path (through the C interface) against the oracle, on a B200.

Small versions of every workload are compared in full: block tables, slot
mappings and copy pairs bit for bit, the whole key and value pools bit for bit
(untouched slots included), and every attention output within tolerance.
Full-size workloads run in the launch configuration the benchmark times and
are checked on sampled outputs and sampled cache slots, over 16-bit caches and
(GQA and long contexts) over E4M3 caches.
"""

import math

import numpy as np
import pytest
import torch

from oracle import step as OS
import paged_kv_cache_352_b200 as pa
from paged_kv_cache_352_b200.runner import DecodeRunner
from tests.parity import assert_close, out_to_f64, tensor_bits
import workloads

pytestmark = pytest.mark.gpu

NAMES = ["tiny_mha_d64", "mha_7b_fp16", "gqa_32_8_bf16", "prefix_share_cow", "long_ctx_split_kv"]


def _sync():
    torch.cuda.synchronize()


@pytest.mark.parametrize("name", NAMES)
def test_small_workload_full_parity(name):
    wl = workloads.workload(name, small=True)
    ref = OS.oracle_step(wl)
    r = DecodeRunner(wl)
    out = r.step()
    _sync()
    assert r.error_bits() == 0
    assert np.array_equal(r.block_tables_host, ref.block_tables)
    assert np.array_equal(np.concatenate(r.prefill_slots), ref.prefill_slots)
    assert np.array_equal(r.step_slots_host, ref.step_slots)
    assert np.array_equal(r.cow_pairs, ref.cow_pairs)
    assert np.array_equal(tensor_bits(r.k_cache), ref.k_cache)
    assert np.array_equal(tensor_bits(r.v_cache), ref.v_cache)
    assert_close(out_to_f64(out, wl.dtype), ref.out, name)


def test_context_of_one_is_the_value_row_exactly():
    wl = workloads.workload("tiny_mha_d64")
    assert wl.context_lens[0] == 1
    r = DecodeRunner(wl)
    out = r.step()
    _sync()
    got = tensor_bits(out)[0]                       # [Hq, d]
    v_row = r.step_v_host[0]                        # token 0 of sequence 0, [Hkv, d]
    assert np.array_equal(got, v_row)


@pytest.mark.parametrize("name", ["mha_7b_fp16", "gqa_32_8_bf16", "long_ctx_split_kv"])
def test_physical_placement_is_invisible_bitwise(name):
    wl = workloads.workload(name, small=True)
    a = DecodeRunner(wl).step().clone()
    wl2 = workloads.workload(name, small=True)
    wl2.free_order = np.random.default_rng(77).permutation(wl2.num_blocks).astype(np.int32)
    r2 = DecodeRunner(wl2)
    assert not np.array_equal(r2.block_tables_host, DecodeRunner(wl).block_tables_host)
    b = r2.step()
    _sync()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_shared_blocks_equal_duplicated_blocks_bitwise():
    """pa_paged_decode gives the same bits whether samples share the prompt's
    blocks or hold private copies. (The shared runner's step decodes through the
    cascade, which sums in another order: equal within tolerance.)"""
    wl = workloads.workload("prefix_share_cow", small=True)
    shared = DecodeRunner(wl)
    dup = DecodeRunner(wl, duplicate=True)
    assert len(shared.cow_pairs) > 0 and len(dup.cow_pairs) == 0
    assert shared.bm.num_free() > dup.bm.num_free()
    assert shared.groups is not None and dup.groups is None
    cascade = shared.step().clone()
    a = shared.decode().clone()
    b = dup.step()
    _sync()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert_close(out_to_f64(cascade, wl.dtype), out_to_f64(b, wl.dtype), "cascade vs duplicated")


@pytest.mark.parametrize("name", ["mha_7b_fp16", "gqa_32_8_bf16", "long_ctx_split_kv"])
def test_split_kv_partition_sizes(name):
    wl = workloads.workload(name, small=True)
    ref = OS.oracle_step(wl).out
    r = DecodeRunner(wl)
    r.step()
    outs = {}
    for pt in (16, 48, 128, 512, 8192):
        out = torch.empty_like(r.out)
        r.decode(out, partition_tokens=pt)
        _sync()
        assert_close(out_to_f64(out, wl.dtype), ref, f"{name} partition {pt}")
        outs[pt] = out
    # one partition covering everything: no merge at all; must equal any single-partition run
    single = torch.empty_like(r.out)
    r.decode(single, partition_tokens=16 * 1024)
    _sync()
    assert torch.equal(single.view(torch.int16), outs[8192].view(torch.int16))
    assert r.error_bits() == 0


def _manual_case(ctx, hq=8, hkv=2, d=128, dtype=torch.bfloat16, nb=64, seed=0):
    """Caches filled with N(0,1), a seeded permutation placement, explicit contexts."""
    g = torch.Generator().manual_seed(seed)
    kc = torch.randn(nb, hkv, 16, d, generator=g).to(dtype).cuda()
    vc = torch.randn(nb, hkv, 16, d, generator=g).to(dtype).cuda()
    q = torch.randn(len(ctx), hq, d, generator=g).to(dtype).cuda()
    perm = torch.randperm(nb, generator=g)
    mb = max(1, max(-(-c // 16) for c in ctx))
    tables = torch.full((len(ctx), mb), -1, dtype=torch.int32)
    used = 0
    for s, c in enumerate(ctx):
        n = -(-c // 16)
        tables[s, :n] = perm[used:used + n].to(torch.int32)
        used += n
    return q, kc, vc, tables.cuda(), torch.tensor(ctx, dtype=torch.int32).cuda()


def _oracle_manual(q, kc, vc, tables, ctx, scale, dtype):
    from oracle.attention import paged_decode
    name = "bf16" if dtype == torch.bfloat16 else "f16"
    return paged_decode(tensor_bits(q), tensor_bits(kc), tensor_bits(vc), tables.cpu().numpy(),
                        ctx.cpu().numpy(), scale, name)


def test_zero_and_tiny_contexts():
    ctx = [0, 1, 2, 15, 16, 17, 0, 33]
    q, kc, vc, tables, cl = _manual_case(ctx)
    out = torch.full_like(q, 7.0)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_paged_decode(out, q, kc, vc, tables, cl, max(ctx), 1 / math.sqrt(128), 0,
                       pa.decode_workspace(len(ctx), 8, 2, 128, max(ctx)), err)
    _sync()
    assert err.item() == 0
    got = out_to_f64(out, "bf16")
    assert (got[0] == 0).all() and (got[6] == 0).all()
    assert_close(got, _oracle_manual(q, kc, vc, tables, cl, 1 / math.sqrt(128), torch.bfloat16))


@pytest.mark.parametrize("G,d,dtype", [(1, 64, torch.float16), (2, 128, torch.bfloat16),
                                       (4, 64, torch.bfloat16), (8, 128, torch.float16)])
def test_every_group_size_and_head_dim(G, d, dtype):
    ctx = [5, 40, 300, 700, 1]
    hkv = 2
    q, kc, vc, tables, cl = _manual_case(ctx, hq=G * hkv, hkv=hkv, d=d, dtype=dtype, nb=128,
                                         seed=G)
    for pt in (0, 32):
        out = torch.empty_like(q)
        ws = pa.decode_workspace(len(ctx), G * hkv, hkv, d, max(ctx), pt)
        pa.pa_paged_decode(out, q, kc, vc, tables, cl, max(ctx), 0.3, pt, ws)
        _sync()
        name = "bf16" if dtype == torch.bfloat16 else "f16"
        assert_close(out_to_f64(out, name),
                     _oracle_manual(q, kc, vc, tables, cl, 0.3, dtype), f"G{G} d{d} pt{pt}")


def test_workspace_is_reusable_without_clearing():
    ctx = [900, 1500, 33]
    q, kc, vc, tables, cl = _manual_case(ctx, nb=256)
    ws = pa.decode_workspace(3, 8, 2, 128, max(ctx), 64)
    outs = []
    for _ in range(3):
        out = torch.empty_like(q)
        pa.pa_paged_decode(out, q, kc, vc, tables, cl, max(ctx), 0.1, 64, ws)
        outs.append(out)
    _sync()
    assert all(torch.equal(outs[0].view(torch.int16), o.view(torch.int16)) for o in outs[1:])
    assert int(ws[:3 * 2 * 4].view(torch.int32).abs().sum()) == 0   # counters back at zero


def test_bad_ids_are_flagged_not_faulted():
    ctx = [40, 40]
    q, kc, vc, tables, cl = _manual_case(ctx)
    tables[1, 1] = 10_000          # outside the 64-block pool
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    pa.pa_paged_decode(out, q, kc, vc, tables, cl, 40, 0.1, 0, None, err)
    _sync()
    assert err.item() & pa.PA_DEVERR_BLOCK_RANGE
    ref = _oracle_manual(q[:1], kc, vc, tables[:1], cl[:1], 0.1, torch.bfloat16)
    assert_close(out_to_f64(out[:1], "bf16"), ref)   # the healthy sequence is unaffected

    err.zero_()
    cl2 = torch.tensor([40, 500], dtype=torch.int32, device="cuda")   # longer than its table
    pa.pa_paged_decode(out, q, kc, vc, tables, cl2, 500, 0.1, 0,
                       pa.decode_workspace(2, 8, 2, 128, 500), err)
    _sync()
    assert err.item() & pa.PA_DEVERR_CONTEXT_RANGE
    assert (out_to_f64(out[1:], "bf16") == 0).all()

    err.zero_()
    key = torch.randn(3, 2, 128, dtype=torch.bfloat16, device="cuda")
    before = kc.clone()
    slots = torch.tensor([5, 64 * 16, -1], dtype=torch.int64, device="cuda")
    pa.pa_reshape_and_cache(key, key, kc, vc, slots, err)
    _sync()
    assert err.item() & pa.PA_DEVERR_SLOT_RANGE
    assert torch.equal(kc[0, :, 5], key[0])
    kc[0, :, 5] = before[0, :, 5]
    assert torch.equal(kc, before)


def test_empty_calls_are_noops():
    kc = torch.zeros(4, 2, 16, 64, dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    e = torch.empty(0, 2, 64, dtype=torch.float16, device="cuda")
    pa.pa_reshape_and_cache(e, e, kc, vc, torch.empty(0, dtype=torch.int64, device="cuda"))
    pa.pa_copy_blocks(kc, vc, np.zeros((0, 2), np.int64))
    q = torch.empty(0, 2, 64, dtype=torch.float16, device="cuda")
    pa.pa_paged_decode(q, q, kc, vc, torch.empty(0, 1, dtype=torch.int32, device="cuda"),
                       torch.empty(0, dtype=torch.int32, device="cuda"), 0, 0.1)
    _sync()
    assert not kc.any()


def test_reshape_with_token_stride_and_copy_blocks_bitwise():
    rng = np.random.default_rng(9)
    nb, hkv, d = 40, 4, 128
    kc0 = rng.integers(0, 1 << 15, (nb, hkv, 16, d)).astype(np.uint16)
    vc0 = rng.integers(0, 1 << 15, (nb, hkv, 16, d)).astype(np.uint16)
    kc = torch.from_numpy(kc0.copy()).view(torch.float16).cuda()
    vc = torch.from_numpy(vc0.copy()).view(torch.float16).cuda()
    # keys/values as slices of a fused [T, 3, Hkv, d] buffer (token stride 3*Hkv*d)
    T = 37
    fused = rng.integers(0, 1 << 15, (T, 3, hkv, d)).astype(np.uint16)
    fz = torch.from_numpy(fused).view(torch.float16).cuda()
    slots = rng.choice(nb * 16, size=T, replace=False).astype(np.int64)
    slots[3] = -1
    pa.pa_reshape_and_cache(fz[:, 1], fz[:, 2], kc, vc, torch.from_numpy(slots).cuda())
    pairs = np.array([(0, 7), (3, 1), (39, 38)], np.int64)
    pa.pa_copy_blocks(kc, vc, pairs)
    _sync()
    from oracle.cache_ops import copy_blocks, reshape_and_cache
    reshape_and_cache(kc0, vc0, fused[:, 1], fused[:, 2], slots, 16)
    copy_blocks(kc0, vc0, pairs)
    assert np.array_equal(tensor_bits(kc), kc0)
    assert np.array_equal(tensor_bits(vc), vc0)


def test_many_copy_pairs_span_launches():
    nb, hkv, d = 3000, 1, 64
    rng = np.random.default_rng(2)
    kc0 = rng.integers(0, 1 << 15, (nb, hkv, 16, d)).astype(np.uint16)
    vc0 = rng.integers(0, 1 << 15, (nb, hkv, 16, d)).astype(np.uint16)
    kc = torch.from_numpy(kc0.copy()).view(torch.bfloat16).cuda()
    vc = torch.from_numpy(vc0.copy()).view(torch.bfloat16).cuda()
    perm = rng.permutation(nb)
    pairs = np.stack([perm[:1400], perm[1400:2800]], 1).astype(np.int64)   # > 1024 pairs
    pa.pa_copy_blocks(kc, vc, pairs)
    _sync()
    from oracle.cache_ops import copy_blocks
    copy_blocks(kc0, vc0, pairs)
    assert np.array_equal(tensor_bits(kc), kc0) and np.array_equal(tensor_bits(vc), vc0)


# ---- full-size workloads, checked on samples ------------------------------------

def _sample_rows(wl, rng, nseq=4, nhead=3):
    seqs = sorted(set(rng.choice(wl.num_seqs, size=min(nseq, wl.num_seqs), replace=False)) |
                  {int(np.argmax(wl.context_lens))})
    rows = []
    for s in seqs:
        for h in sorted(set(rng.choice(wl.num_q_heads, size=nhead, replace=False)) |
                        {wl.num_q_heads - 1}):
            rows.append((int(s), int(h)))
    return rows


@pytest.mark.parametrize("name", NAMES)
def test_full_size_sampled_parity(name):
    wl = workloads.workload(name)
    r = DecodeRunner(wl)
    out = r.step()
    _sync()
    assert r.error_bits() == 0
    rng = np.random.default_rng(352)
    rows = _sample_rows(wl, rng)
    ref = OS.sampled_outputs(wl, rows, r.q_host)
    got = out_to_f64(out, wl.dtype)
    assert_close(np.stack([got[s, h] for s, h in rows]), ref, f"{name} sampled")
    # the cache holds each sampled sequence's logical rows at the slots of its table
    for s in sorted({s for s, _ in rows})[:2]:
        kb, vb = OS.logical_kv_bits(wl, s)
        table = r.block_tables_host[s]
        pos = np.unique(np.concatenate([[0, len(kb) - 1], rng.integers(0, len(kb), 16)]))
        blocks = torch.from_numpy(table[pos // 16].astype(np.int64)).cuda()
        offs = torch.from_numpy(pos % 16).cuda()
        gk = tensor_bits(r.k_cache[blocks, :, offs, :])
        gv = tensor_bits(r.v_cache[blocks, :, offs, :])
        assert np.array_equal(gk, kb[pos]) and np.array_equal(gv, vb[pos])
    # every output row is finite and the whole output changes nothing on a second step
    again = r.step().clone()
    _sync()
    assert torch.equal(again.view(torch.int16), out.view(torch.int16))


@pytest.mark.parametrize("name", ["gqa_32_8_bf16", "long_ctx_split_kv", "mha_7b_fp16"])
def test_scheduling_order_does_not_change_results(name):
    wl = workloads.workload(name, small=True)
    r = DecodeRunner(wl)
    r.step()
    outs = []
    for order in (None, "longest", "random"):
        out = torch.empty_like(r.out)
        if order is None:
            r.decode(out, ordered=False)
        else:
            if order == "random":
                perm = np.random.default_rng(5).permutation(wl.num_seqs).astype(np.int32)
                r.seq_order.copy_(torch.from_numpy(perm))
            r.decode(out, ordered=True)
        outs.append(out)
    _sync()
    assert r.error_bits() == 0
    for o in outs[1:]:
        assert torch.equal(outs[0].view(torch.int16), o.view(torch.int16))


def test_bad_order_entries_are_flagged():
    ctx = [40, 70]
    q, kc, vc, tables, cl = _manual_case(ctx)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros_like(q)
    order = torch.tensor([1, 7], dtype=torch.int32, device="cuda")
    pa.pa_paged_decode(out, q, kc, vc, tables, cl, 70, 0.1, 0, None, err, seq_order=order)
    _sync()
    assert err.item() & pa.PA_DEVERR_CONTEXT_RANGE
    ref = _oracle_manual(q, kc, vc, tables, cl, 0.1, torch.bfloat16)
    assert_close(out_to_f64(out[1:], "bf16"), ref[1:])   # sequence 1 was still computed


def test_host_pipeline_returns_each_steps_output():
    from paged_kv_cache_352_b200.runner import HostPipeline
    wl = workloads.workload("gqa_32_8_bf16", small=True)
    r = DecodeRunner(wl)
    ref = r.step().clone()
    hp = HostPipeline(r)
    outs = [hp() for _ in range(4)]
    _sync()
    for o in outs[-2:]:
        assert torch.equal(o.view(torch.int16), ref.cpu().view(torch.int16))
    assert hp.h2d_bytes >= (r.q.numel() + r.step_k.numel() + r.step_v.numel()) * 2


@pytest.mark.parametrize("name", ["mha_7b_fp16", "gqa_32_8_bf16", "long_ctx_split_kv"])
@pytest.mark.parametrize("factor", [8.0, 32.0])
def test_peaked_softmax(name, factor):
    """N(0,1) queries and keys give nearly flat weights, which an absolute
    tolerance passes too easily. Queries scaled by 8 and 32 (exact in 16-bit
    floats) make the weights peaked: one or a few tokens dominate, and every
    rescale of the online softmax and every split-KV merge shows up in the
    output. Unsplit and split (64-token partitions) decodes against the oracle."""
    from oracle.attention import paged_decode
    wl = workloads.workload(name, small=True)
    r = DecodeRunner(wl)
    r.step()
    _sync()
    r.q = (r.q.float() * factor).to(r.q.dtype)
    ref = paged_decode(tensor_bits(r.q), tensor_bits(r.k_cache), tensor_bits(r.v_cache),
                       r.block_tables_host, r.context_lens_host, wl.scale, wl.dtype)
    for pt in (0, 64):
        out = torch.empty_like(r.out)
        r.decode(out, partition_tokens=pt)
        _sync()
        assert_close(out_to_f64(out, wl.dtype), ref, f"{name} q x{factor} partition {pt}")
    assert r.error_bits() == 0


@pytest.mark.parametrize("name", ["mha_7b_fp16", "gqa_32_8_bf16", "long_ctx_split_kv"])
def test_planted_key(name):
    """One key per (sequence, KV head) replaced by 4 x the group's first query
    head: that token's logit is about 4 |q|^2 / sqrt(d) ~ 45 above the rest, so
    its weight is ~1 and the output is ~its value row, wherever in the context
    (first token, a block boundary, the last token, a random position) it sits.
    A kernel that loses a token, a block or a partition misses it by O(1)."""
    from oracle.attention import paged_decode
    wl = workloads.workload(name, small=True)
    r = DecodeRunner(wl)
    r.step()
    _sync()
    g = wl.num_q_heads // wl.num_kv_heads
    rng = np.random.default_rng(wl.seed + 77)
    tables = r.block_tables_host
    for s, c in enumerate(r.context_lens_host.tolist()):
        t = int([0, min(16, c - 1), c - 1, rng.integers(0, c)][s % 4])
        blk, off = int(tables[s][t // 16]), t % 16
        for h in range(wl.num_kv_heads):
            r.k_cache[blk, h, off] = (r.q[s, h * g].float() * 4.0).to(r.k_cache.dtype)
    _sync()
    ref = paged_decode(tensor_bits(r.q), tensor_bits(r.k_cache), tensor_bits(r.v_cache),
                       tables, r.context_lens_host, wl.scale, wl.dtype)
    for pt in (0, 64):
        out = torch.empty_like(r.out)
        r.decode(out, partition_tokens=pt)
        _sync()
        assert_close(out_to_f64(out, wl.dtype), ref, f"{name} planted key, partition {pt}")
    assert r.error_bits() == 0


@pytest.mark.parametrize("name", ["gqa_32_8_bf16", "long_ctx_split_kv"])
def test_full_size_fp8_sampled_parity(name):
    """The same batches over E4M3 caches of random valid codes, in the launch
    configuration the benchmark's 8-bit figure times (the runner's tables,
    lengths, order and partitions: CTA mode for GQA, the warp-per-partition split
    with two blocks per loop step for long contexts), checked on sampled rows
    against the oracle's attention over the dequantized codes."""
    from oracle import fp8 as F
    from oracle.attention import softmax_attention
    from oracle.fpbits import bits_to_f64
    wl = workloads.workload(name)
    r = DecodeRunner(wl)
    g = torch.Generator(device="cuda").manual_seed(353)
    shape = tuple(r.k_cache.shape)

    def codes():
        c = torch.randint(0, 0x7E, shape, generator=g, device="cuda", dtype=torch.uint8)
        return c | (torch.randint(0, 2, shape, generator=g, device="cuda",
                                  dtype=torch.uint8) << 7)
    kc, vc = codes(), codes()
    del r.k_cache, r.v_cache
    torch.cuda.empty_cache()
    ks, vs = 0.05, 0.02
    out = torch.empty_like(r.q)
    pa.pa_paged_decode_fp8(out, r.q, kc, vc, r.block_tables, r.context_lens,
                           wl.max_context_len, wl.scale, ks, vs,
                           partition_tokens=r.partition_tokens or 0, workspace=r.workspace,
                           dev_error=r.dev_error, seq_order=r.seq_order)
    _sync()
    assert r.error_bits() == 0
    got = out_to_f64(out, wl.dtype)
    rows = _sample_rows(wl, np.random.default_rng(353))
    G = wl.num_q_heads // wl.num_kv_heads
    ref = np.zeros((len(rows), wl.head_dim))
    for i, (s, h) in enumerate(rows):
        ctx = int(wl.context_lens[s])
        n = -(-ctx // 16)
        blocks = torch.from_numpy(r.block_tables_host[s, :n].astype(np.int64)).cuda()
        kvh = h // G
        kb = kc[blocks, kvh].reshape(n * 16, -1)[:ctx].cpu().numpy()
        vb = vc[blocks, kvh].reshape(n * 16, -1)[:ctx].cpu().numpy()
        ref[i] = softmax_attention(bits_to_f64(r.q_host[s, h], wl.dtype), F.dequantize(kb, ks),
                                   F.dequantize(vb, vs), wl.scale)
    assert_close(np.stack([got[s, h] for s, h in rows]), ref, f"{name} over E4M3 caches")
