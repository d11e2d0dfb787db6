"""The C interface without a GPU: exported symbols, host-side argument checks, and
the C++ block manager against the oracle's block manager (bit-exact)."""

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import block_manager as OBM
import paged_kv_cache_352_b200 as pa
from paged_kv_cache_352_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    h = L.lib()
    names = _declared_symbols()
    assert len(names) >= 18
    missing = [n for n in names if not hasattr(h, n)]
    assert not missing, missing
    assert h.pa_version() == 111


def test_binding_covers_every_declared_symbol():
    assert set(_declared_symbols()) <= set(L._SIGS)


def test_stall_hook_rejects_limits_out_of_range():
    # (a valid limit would arm the next decode launch of this process: not done here)
    assert L.lib().pa_test_stall_next_decode(0) == L.PA_ERR_INVALID_ARG
    assert L.lib().pa_test_stall_next_decode(999) == L.PA_ERR_INVALID_ARG
    assert L.lib().pa_test_stall_next_decode(10**9) == L.PA_ERR_INVALID_ARG
    assert "wait_limit_ns" in L.last_error()


# ---- host-side argument checks (return before any CUDA call) --------------------

FAKE = ctypes.c_void_p(4096)  # never dereferenced: every call below fails validation first


def _status(call):
    st = call()
    return st, L.last_error()


@pytest.mark.parametrize("head_dim,block_size,dtype,code", [
    (96, 16, L.PA_F16, L.PA_ERR_UNSUPPORTED),
    (128, 32, L.PA_F16, L.PA_ERR_UNSUPPORTED),
    (128, 16, 7, L.PA_ERR_UNSUPPORTED),
])
def test_reshape_rejects_unsupported_shapes(head_dim, block_size, dtype, code):
    st, msg = _status(lambda: L.lib().pa_reshape_and_cache(
        FAKE, FAKE, 8 * head_dim, 8 * head_dim, FAKE, FAKE, FAKE, 4, 8, head_dim, block_size, 64,
        dtype, None, None))
    assert st == code and msg


def test_reshape_rejects_bad_strides_and_alignment():
    lib = L.lib()
    st = lib.pa_reshape_and_cache(FAKE, FAKE, 100, 1024, FAKE, FAKE, FAKE, 4, 8, 128, 16, 64,
                                  L.PA_F16, None, None)
    assert st == L.PA_ERR_INVALID_ARG and "stride" in L.last_error()
    st = lib.pa_reshape_and_cache(ctypes.c_void_p(4098), FAKE, 1024, 1024, FAKE, FAKE, FAKE, 4, 8,
                                  128, 16, 64, L.PA_F16, None, None)
    assert st == L.PA_ERR_INVALID_ARG and "aligned" in L.last_error()
    assert lib.pa_reshape_and_cache(FAKE, FAKE, 1024, 1024, FAKE, FAKE, FAKE, 0, 8, 128, 16, 64,
                                    L.PA_F16, None, None) == L.PA_OK   # T = 0: no-op


def _pairs(p):
    a = np.ascontiguousarray(np.asarray(p, np.int64).reshape(-1, 2))
    return a, a.ctypes.data


@pytest.mark.parametrize("pairs,why", [
    ([(0, 64)], "outside"),
    ([(-1, 3)], "outside"),
    ([(0, 3), (1, 3)], "twice"),
    ([(0, 3), (3, 5)], "both"),
])
def test_copy_blocks_rejects_bad_pairs(pairs, why):
    arr, ptr = _pairs(pairs)
    st = L.lib().pa_copy_blocks(FAKE, FAKE, ptr, len(arr), 8, 128, 16, 64, L.PA_F16, None)
    assert st == L.PA_ERR_INVALID_ARG and why in L.last_error()


@pytest.mark.parametrize("pairs,why", [
    ([(0, 10)], "outside"),        # destination pool has 10 blocks
    ([(64, 1)], "outside"),        # source pool has 64 blocks
    ([(0, 3), (1, 3)], "twice"),
])
def test_swap_blocks_rejects_bad_pairs(pairs, why):
    arr, ptr = _pairs(pairs)
    other = ctypes.c_void_p(8192)
    st = L.lib().pa_swap_blocks(FAKE, FAKE, 64, other, other, 10, ptr, len(arr), 8, 128, 16,
                                L.PA_F16, None)
    assert st == L.PA_ERR_INVALID_ARG and why in L.last_error()


def test_swap_blocks_refuses_same_pool():
    arr, ptr = _pairs([(0, 1)])
    st = L.lib().pa_swap_blocks(FAKE, FAKE, 64, FAKE, FAKE, 64, ptr, 1, 8, 128, 16, L.PA_F16,
                                None)
    assert st == L.PA_ERR_INVALID_ARG and "different pools" in L.last_error()


def test_block_manager_swap_errors():
    bm = pa.BlockManager(8, 16)
    bm.set_host_pool(2)
    bm.add_seq(1, 40)                      # 3 blocks > 2 host blocks
    with pytest.raises(pa.PAError) as e:
        bm.swap_out(1)
    assert e.value.code == L.PA_ERR_NO_FREE_BLOCKS and not bm.is_swapped(1)
    bm.add_seq(2, 20)
    bm.swap_out(2)
    for op in (lambda: bm.append_slots(2, 1), lambda: bm.fork(2, 3),
               lambda: bm.block_tables([2], 4), lambda: bm.swap_out(2)):
        with pytest.raises(pa.PAError) as e:
            op()
        assert e.value.code == L.PA_ERR_SEQ_SWAPPED
    with pytest.raises(pa.PAError):
        bm.set_host_pool(8)                # host blocks in use
    bm.free_seq(2)
    assert bm.num_free_host() == 2


def test_copy_blocks_zero_pairs_is_noop():
    assert L.lib().pa_copy_blocks(FAKE, FAKE, None, 0, 8, 128, 16, 64, L.PA_F16, None) == L.PA_OK


def test_decode_argument_checks():
    lib = L.lib()

    def call(**kw):
        a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, mb=8, ctx=FAKE, B=4, maxctx=100,
                 hq=32, hkv=8, d=128, bs=16, nb=64, scale=0.1, pt=0, ws=None, wsb=0,
                 err=None, dt=L.PA_BF16)
        a.update(kw)
        return lib.pa_paged_decode(a["out"], a["q"], a["k"], a["v"], a["bt"], a["mb"], a["ctx"],
                                   None, a["B"], a["maxctx"], a["hq"], a["hkv"], a["d"], a["bs"],
                                   a["nb"], a["scale"], a["pt"], a["ws"], a["wsb"], a["err"],
                                   a["dt"], None)

    assert call(hq=24) == L.PA_ERR_UNSUPPORTED          # G = 3
    assert call(hq=30) == L.PA_ERR_INVALID_ARG          # not a multiple
    assert call(hq=128) == L.PA_ERR_UNSUPPORTED         # G = 16
    assert call(d=80) == L.PA_ERR_UNSUPPORTED
    assert call(pt=24) == L.PA_ERR_INVALID_ARG          # not a multiple of 16
    assert call(maxctx=5000) == L.PA_ERR_INVALID_ARG    # needs a workspace, none given
    assert "workspace" in L.last_error()
    assert call(q=ctypes.c_void_p(4100)) == L.PA_ERR_INVALID_ARG
    assert call(B=0) == L.PA_OK                         # nothing to do
    assert call(scale=float("nan")) == L.PA_ERR_INVALID_ARG


def test_longest_first_order():
    ctx = [5, 90, 90, 1, 300, 0]
    assert pa.pa_longest_first_order(ctx).tolist() == [4, 1, 2, 0, 3, 5]
    assert pa.pa_longest_first_order([]).tolist() == []


def test_workspace_size_formula():
    # 8 seqs x 8 KV heads, 4 query heads each, up to 2000 tokens in 512-token partitions
    n = pa.pa_paged_decode_workspace_size(8, 32, 8, 128, 2000, 16, 512)
    parts = 4
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    ml_off = up(64 * 4)
    acc_off = up(ml_off + 64 * parts * 4 * 2 * 4)
    assert n == up(acc_off + 64 * parts * 4 * 128 * 4)
    assert pa.pa_paged_decode_workspace_size(8, 32, 8, 128, 512, 16, 512) == 0  # one partition
    with pytest.raises(pa.PAError):
        pa.pa_paged_decode_workspace_size(8, 32, 8, 128, 512, 16, 100)


# ---- C++ block manager == oracle block manager ---------------------------------

def _same_state(cbm, obm, seqs):
    assert cbm.num_free() == obm.num_free()
    assert cbm.free_list() == obm.free_list()
    assert cbm.num_free_host() == obm.num_free_host()
    assert cbm.num_cached() == obm.num_cached()
    assert cbm.evictable_list() == obm.evictable_list()
    assert cbm.host_free_list() == obm.host_free_list()
    for s in seqs:
        assert cbm.is_swapped(s) == obm.is_swapped(s)
    for b in range(obm.num_blocks):
        assert cbm.refcount(b) == obm.refcount(b)
    for s in seqs:
        assert cbm.seq_len(s) == obm.seq_len(s)
        assert cbm.table(s) == obm.table(s)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_block_manager_matches_oracle(seed):
    rng = np.random.default_rng(seed)
    nb, bs = 80, 16
    order = rng.permutation(nb)
    cbm = pa.BlockManager(nb, bs, order)
    obm = OBM.BlockManager(nb, bs, order)
    cbm.set_host_pool(40)
    obm.set_host_pool(40)
    live, nid = [], 1000
    prefixes = [rng.integers(0, 50, 64).tolist() for _ in range(3)]
    for it in range(1500):
        op = int(rng.integers(0, 8))
        if op == 7:
            base = prefixes[int(rng.integers(0, 3))]
            keep = int(rng.integers(0, 65))
            toks = base[:keep] + rng.integers(0, 50, int(rng.integers(0, 40))).tolist()
            args = ("add_seq_cached", nid, toks)
            assert cbm.cached_prefix(toks) == obm.cached_prefix(toks)
        elif op == 0 or not live:
            n = int(rng.integers(0, 70))
            args = ("add_seq", nid, n)
        elif op == 1:
            args = ("fork", live[int(rng.integers(len(live)))], nid)
        elif op in (2, 3):
            args = ("append_slots", live[int(rng.integers(len(live)))], int(rng.integers(0, 25)))
        elif op == 4:
            args = ("free_seq", live[int(rng.integers(len(live)))])
        elif op == 5:
            args = ("swap_out", live[int(rng.integers(len(live)))])
        else:
            args = ("swap_in", live[int(rng.integers(len(live)))])
        oerr = cerr = None
        try:
            ores = getattr(obm, args[0])(*args[1:])
        except OBM.BlockManagerError as e:
            oerr = e.code
        try:
            cres = getattr(cbm, args[0])(*args[1:])
        except pa.PAError as e:
            cerr = e.code
        assert oerr == cerr, (it, args, oerr, cerr)
        if oerr is None:
            if args[0] == "add_seq":
                assert list(cres) == ores
                live.append(nid)
                nid += 1
            elif args[0] == "add_seq_cached":
                assert list(cres[0]) == ores[0] and cres[1] == ores[1]
                live.append(nid)
                nid += 1
            elif args[0] == "fork":
                live.append(nid)
                nid += 1
            elif args[0] == "append_slots":
                assert list(cres[0]) == ores[0]
                assert [tuple(p) for p in cres[1].tolist()] == [tuple(p) for p in ores[1]]
            elif args[0] == "free_seq":
                live.remove(args[1])
            elif args[0] in ("swap_out", "swap_in"):
                assert [tuple(p) for p in cres.tolist()] == [tuple(p) for p in ores]
        _same_state(cbm, obm, live)
    resident = [s for s in live if not obm.is_swapped(s)]
    mb = max([len(obm.table(s)) for s in resident] + [1])
    assert np.array_equal(cbm.block_tables(resident, mb + 2), obm.block_tables(resident, mb + 2))


def test_prefix_cache_reuse_counts():
    bm = pa.BlockManager(64, 16)
    prompt = list(range(1000, 1100))                 # 6 full blocks + 4 tokens
    _, c1 = bm.add_seq_cached(1, prompt)
    _, c2 = bm.add_seq_cached(2, prompt + [5, 6])
    assert (c1, c2) == (0, 96) and bm.table(2)[:6] == bm.table(1)[:6]
    assert bm.num_cached() == 6
    bm.free_seq(1)
    bm.free_seq(2)
    assert bm.num_free() == 64 and len(bm.evictable_list()) == 6


def test_block_manager_errors_and_queries():
    bm = pa.BlockManager(4, 16)
    with pytest.raises(pa.PAError) as e:
        bm.fork(1, 2)
    assert e.value.code == L.PA_ERR_UNKNOWN_SEQ
    bm.add_seq(1, 20)
    with pytest.raises(pa.PAError) as e:
        bm.add_seq(1, 3)
    assert e.value.code == L.PA_ERR_SEQ_EXISTS
    with pytest.raises(pa.PAError) as e:
        bm.append_slots(1, 100)
    assert e.value.code == L.PA_ERR_NO_FREE_BLOCKS
    assert bm.seq_len(1) == 20 and bm.num_free() == 2
    with pytest.raises(pa.PAError):
        bm.block_tables([1], 1)          # table longer than max_blocks
    with pytest.raises(pa.PAError):
        bm.refcount(9)
    with pytest.raises(pa.PAError):
        pa.BlockManager(4, 16, [0, 1, 1, 2])
    assert bm.num_seqs() == 1
    bm.free_seq(1)
    assert bm.num_free() == 4 and bm.num_seqs() == 0


def test_block_manager_reproduces_figure(golden):
    g = golden("block_table_figure.json")
    bm = pa.BlockManager(g["pool_blocks"], g["block_size"])
    bs = g["block_size"]
    bm.add_seq(10, bs)
    bm.add_seq(11, bs)
    bm.append_slots(10, bs)
    bm.add_seq(12, bs)
    bm.append_slots(11, bs)
    bm.add_seq(13, bs)
    bm.append_slots(10, bs)
    bm.append_slots(11, bs)
    bm.free_seq(12)
    bm.free_seq(13)
    assert bm.table(10) == g["tables"]["A"] and bm.table(11) == g["tables"]["B"]
    assert sorted(bm.free_list()) == g["free"]


def test_block_manager_seventy_tokens(golden):
    g = golden("seventy_tokens.json")
    bm = pa.BlockManager(64, g["block_size"])
    slots = bm.add_seq(0, g["tokens"])
    t = bm.table(0)
    assert len(t) == g["blocks"]
    assert sum(1 for s in slots if s // 16 == t[-1]) == g["last_block_used"]


def test_decode_plan_split_modes():
    """Short caller-chosen partitions over a large grid run one warp per partition
    plus a merge launch; small batches and unsplit calls keep one launch."""
    if os.environ.get("PA_DECODE_SPLIT"):
        pytest.skip("split mode forced by the environment")
    # the long-context configuration: 8 sequences up to 128k tokens, 512-token partitions
    assert L.pa_paged_decode_plan(8, 64, 8, 128, 131072, 512, ordered=True) == (32, 256, 2)
    # one long sequence: too few CTAs for one warp per partition
    assert L.pa_paged_decode_plan(1, 64, 8, 128, 32768, 512, ordered=True) == (32, 64, 1)
    # long partitions stay one CTA per partition
    assert L.pa_paged_decode_plan(8, 64, 8, 128, 131072, 2048, ordered=True)[2] == 1
    # short partitions of short sequences (few partitions each) too
    assert L.pa_paged_decode_plan(256, 32, 8, 128, 4096, 1024, ordered=True) == (64, 4, 1)
    # no split at all, and an empty batch
    assert L.pa_paged_decode_plan(64, 32, 32, 128, 2048, 0, ordered=True) == (128, 1, 1)
    assert L.pa_paged_decode_plan(0, 32, 32, 128, 2048, 0)[2] == 0
    with pytest.raises(L.PAError):
        L.pa_paged_decode_plan(4, 30, 8, 128, 100, 0)          # heads not a multiple
    with pytest.raises(L.PAError):
        L.pa_paged_decode_plan(4, 32, 8, 128, 100, 24)         # partition not whole blocks
