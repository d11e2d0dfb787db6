"""Swapping blocks between the device pool and pinned host memory (preemption),
on a B200, against the oracle: the pools bit for bit, and decode outputs of the
swapped sequences unchanged after they come back into different blocks."""

import numpy as np
import pytest
import torch

from oracle import cache_ops as OC
import paged_kv_cache_352_b200 as pa
from paged_kv_cache_352_b200.runner import DecodeRunner
from tests.parity import tensor_bits
import workloads

pytestmark = pytest.mark.gpu


def _host_pool(shape, dtype):
    return torch.zeros(shape, dtype=dtype).pin_memory()


def test_swap_round_trip_matches_oracle_and_keeps_outputs():
    wl = workloads.workload("mha_7b_fp16", small=True)
    r = DecodeRunner(wl)
    r.step()
    before = r.decode().clone()
    torch.cuda.synchronize()
    nh = 200
    hk = _host_pool((nh,) + tuple(r.k_cache.shape[1:]), r.dtype)
    hv = _host_pool((nh,) + tuple(r.k_cache.shape[1:]), r.dtype)
    r.bm.set_host_pool(nh)
    # oracle mirror of both pools and of the manager
    ok_, ov_ = tensor_bits(r.k_cache).copy(), tensor_bits(r.v_cache).copy()
    ohk = np.zeros((nh,) + ok_.shape[1:], np.uint16)
    ohv = np.zeros_like(ohk)
    victims = [1, 3, 4]
    out_pairs = {}
    for s in victims:
        pairs = r.bm.swap_out(s)
        out_pairs[s] = pairs
        pa.pa_swap_blocks(r.k_cache, r.v_cache, hk, hv, pairs)
        OC.swap_blocks(ok_, ov_, ohk, ohv, pairs)
    torch.cuda.synchronize()
    assert np.array_equal(tensor_bits(hk), ohk) and np.array_equal(tensor_bits(hv), ohv)
    # another sequence takes every free device block and overwrites it
    free = r.bm.num_free()
    r.bm.add_seq(999, free * 16)
    noise = torch.randn(free * 16, wl.num_kv_heads, wl.head_dim, device="cuda").to(r.dtype)
    table999 = r.bm.table(999)
    slots = torch.tensor([b * 16 + o for b in table999 for o in range(16)], dtype=torch.int64,
                         device="cuda")
    pa.pa_reshape_and_cache(noise, noise, r.k_cache, r.v_cache, slots)
    r.bm.free_seq(999)
    for s in victims:
        pairs = r.bm.swap_in(s)
        pa.pa_swap_blocks(hk, hv, r.k_cache, r.v_cache, pairs)
    torch.cuda.synchronize()
    # decode again through the new tables: outputs bit-identical to before
    tables = r.bm.block_tables(range(wl.num_seqs), r.max_blocks)
    r.block_tables.copy_(torch.from_numpy(tables))
    after = r.decode().clone()
    torch.cuda.synchronize()
    assert r.error_bits() == 0
    assert torch.equal(before.view(torch.int16), after.view(torch.int16))
    # and the swapped-in blocks hold exactly what the oracle's pools say
    for s in victims:
        for (_, h), b in zip(out_pairs[s], r.bm.table(s)):
            assert np.array_equal(tensor_bits(r.k_cache[b]), ohk[h])
            assert np.array_equal(tensor_bits(r.v_cache[b]), ohv[h])


def test_swap_refuses_pageable_host_memory():
    dk = torch.zeros(4, 2, 16, 64, dtype=torch.float16, device="cuda")
    hk = torch.zeros(4, 2, 16, 64, dtype=torch.float16)       # not pinned
    with pytest.raises(pa.PAError):
        pa.pa_swap_blocks(dk, dk.clone(), hk, hk.clone(), [(0, 1)])
    lib = pa.lib()
    pairs = np.array([[0, 1]], np.int64)
    st = lib.pa_swap_blocks(dk.data_ptr(), dk.data_ptr() + 16, 4, hk.data_ptr(),
                            hk.data_ptr() + 4096, 4, pairs.ctypes.data, 1, 2, 64, 16, 0, None)
    assert st == pa._lib.PA_ERR_INVALID_ARG and "pinned" in pa.last_error()


def test_swap_many_pairs_device_to_host_to_device():
    nb, hkv, d = 2500, 2, 128
    rng = np.random.default_rng(4)
    src = rng.integers(0, 1 << 15, (nb, hkv, 16, d)).astype(np.uint16)
    dk = torch.from_numpy(src).view(torch.bfloat16).cuda()
    dv = torch.from_numpy(src[::-1].copy()).view(torch.bfloat16).cuda()
    hk = _host_pool((nb, hkv, 16, d), torch.bfloat16)
    hv = _host_pool((nb, hkv, 16, d), torch.bfloat16)
    perm = rng.permutation(nb)
    pairs = np.stack([np.arange(2100), perm[:2100]], 1)   # > 1024 pairs: several launches
    pa.pa_swap_blocks(dk, dv, hk, hv, pairs)
    back_k = torch.zeros_like(dk)
    back_v = torch.zeros_like(dv)
    pa.pa_swap_blocks(hk, hv, back_k, back_v, pairs[:, ::-1].copy())
    torch.cuda.synchronize()
    assert torch.equal(back_k[:2100].view(torch.int16), dk[:2100].view(torch.int16))
    assert torch.equal(back_v[:2100].view(torch.int16), dv[:2100].view(torch.int16))
    assert not back_k[2100:].view(torch.int16).any()
