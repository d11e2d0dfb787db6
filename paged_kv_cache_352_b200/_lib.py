"""ctypes binding to libpa.so: the C interface's calls under the same names.

Only argument marshalling happens here: tensors become device pointers, the
current PyTorch CUDA stream becomes the launch stream, and non-zero statuses
become ``PAError``. Every step of the decode path runs in libpa's kernels.
The library must be built (``python -m paged_kv_cache_352_b200.build``); there
is no fallback when it is missing.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpa.so")

PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_NO_FREE_BLOCKS = 2
PA_ERR_UNKNOWN_SEQ = 3
PA_ERR_CUDA = 4
PA_ERR_UNSUPPORTED = 5
PA_ERR_SEQ_EXISTS = 6
PA_ERR_SEQ_SWAPPED = 7

PA_F16 = 0
PA_BF16 = 1
PA_FP8_E4M3 = 2

PA_DEVERR_SLOT_RANGE = 1
PA_DEVERR_BLOCK_RANGE = 2
PA_DEVERR_CONTEXT_RANGE = 4
PA_DEVERR_WAIT_TIMEOUT = 8
PA_DEVERR_GROUP = 16

BLOCK_SIZE = 16


class PAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libpa status {code}: {msg}")
        self.code = code


_c_int = ctypes.c_int
_c_i64 = ctypes.c_int64
_vp = ctypes.c_void_p
_SIGS = {
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_version": (_c_int, []),
    "pa_test_stall_next_decode": (_c_int, [ctypes.c_ulonglong]),
    "pa_reshape_and_cache": (_c_int, [_vp, _vp, _c_i64, _c_i64, _vp, _vp, _vp, _c_int, _c_int,
                                      _c_int, _c_int, _c_int, _c_int, _vp, _vp]),
    "pa_copy_blocks": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                _vp]),
    "pa_paged_decode_workspace_size": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                                _c_int, ctypes.POINTER(ctypes.c_size_t)]),
    "pa_paged_decode": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp, _c_int, _c_int,
                                 _c_int, _c_int, _c_int, _c_int, _c_int, ctypes.c_float, _c_int,
                                 _vp, ctypes.c_size_t, _vp, _c_int, _vp]),
    "pa_paged_decode_noalloc": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp, _c_int,
                                         _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                         ctypes.c_float, _c_int, _vp, _c_int, _vp]),
    "pa_longest_first_order": (_c_int, [_vp, _c_int, _vp]),
    "pa_paged_decode_plan": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                      _c_int, ctypes.POINTER(_c_int), ctypes.POINTER(_c_int),
                                      ctypes.POINTER(_c_int)]),
    "pa_paged_decode_cascade_plan": (_c_int, [_c_int] * 12 + [ctypes.POINTER(_c_int)] * 5),
    "pa_reshape_and_cache_fp8": (_c_int, [_vp, _vp, _c_i64, _c_i64, _vp, _vp, _vp, _c_int, _c_int,
                                          _c_int, _c_int, _c_int, _c_int, ctypes.c_float,
                                          ctypes.c_float, _vp, _vp]),
    "pa_paged_decode_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp, _c_int, _c_int,
                                     _c_int, _c_int, _c_int, _c_int, _c_int, ctypes.c_float,
                                     ctypes.c_float, ctypes.c_float, _c_int, _vp, ctypes.c_size_t,
                                     _vp, _c_int, _vp]),
    "pa_paged_decode_cascade_workspace_size": (_c_int, [_c_int] * 10 +
                                                [ctypes.POINTER(ctypes.c_size_t)]),
    "pa_paged_decode_cascade": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp, _c_int,
                                         _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                         ctypes.c_float, _vp, _vp, _vp, _vp, _c_int, _c_int,
                                         _c_int, _vp, ctypes.c_size_t, _vp, _c_int, _vp]),
    "pa_paged_decode_cascade_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp, _c_int,
                                             _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                             ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                             _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _vp,
                                             ctypes.c_size_t, _vp, _c_int, _vp]),
    "pa_cascade_order": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _vp]),
    "pa_bm_prefix_groups": (_c_int, [_vp, _vp, _c_int, _c_int, _vp, _vp, _vp, _vp,
                                     ctypes.POINTER(_c_int), ctypes.POINTER(_c_int)]),
    "pa_bm_create": (_c_int, [_c_int, _c_int, _vp, ctypes.POINTER(_vp)]),
    "pa_bm_destroy": (None, [_vp]),
    "pa_bm_add_seq": (_c_int, [_vp, _c_i64, _c_int, _vp]),
    "pa_bm_fork": (_c_int, [_vp, _c_i64, _c_i64]),
    "pa_bm_append_slots": (_c_int, [_vp, _c_i64, _c_int, _vp, _vp, ctypes.POINTER(_c_int)]),
    "pa_bm_free_seq": (_c_int, [_vp, _c_i64]),
    "pa_bm_block_tables": (_c_int, [_vp, _vp, _c_int, _vp, _c_int]),
    "pa_bm_num_free": (_c_int, [_vp]),
    "pa_bm_refcount": (_c_int, [_vp, ctypes.c_int32]),
    "pa_bm_seq_len": (_c_int, [_vp, _c_i64]),
    "pa_bm_num_seqs": (_c_int, [_vp]),
    "pa_bm_free_list": (_c_int, [_vp, _vp, _c_int]),
    "pa_swap_blocks": (_c_int, [_vp, _vp, _c_int, _vp, _vp, _c_int, _vp, _c_int, _c_int, _c_int,
                                _c_int, _c_int, _vp]),
    "pa_bm_set_host_pool": (_c_int, [_vp, _c_int]),
    "pa_bm_swap_out": (_c_int, [_vp, _c_i64, _vp, _c_int, ctypes.POINTER(_c_int)]),
    "pa_bm_swap_in": (_c_int, [_vp, _c_i64, _vp, _c_int, ctypes.POINTER(_c_int)]),
    "pa_bm_is_swapped": (_c_int, [_vp, _c_i64]),
    "pa_bm_num_free_host": (_c_int, [_vp]),
    "pa_bm_host_free_list": (_c_int, [_vp, _vp, _c_int]),
    "pa_bm_add_seq_cached": (_c_int, [_vp, _c_i64, _vp, _c_int, _vp, ctypes.POINTER(_c_int)]),
    "pa_bm_num_cached": (_c_int, [_vp]),
    "pa_bm_cached_prefix": (_c_int, [_vp, _vp, _c_int, ctypes.POINTER(_c_int),
                                     ctypes.POINTER(_c_int)]),
    "pa_bm_evictable_list": (_c_int, [_vp, _vp, _c_int]),
    "pa_sched_create": (_c_int, [_c_int, _c_int, _vp, _c_int, _c_int, _c_int, ctypes.POINTER(_vp)]),
    "pa_sched_destroy": (None, [_vp]),
    "pa_sched_submit": (_c_int, [_vp, _c_i64, _c_int, _c_int, _c_int, _c_i64]),
    "pa_sched_submit_tokens": (_c_int, [_vp, _c_i64, _vp, _c_int, _c_int, _c_int, _c_i64]),
    "pa_sched_step": (_c_int, [_vp, _vp]),
    "pa_sched_idle": (_c_int, [_vp]),
    "pa_sched_plan_requests": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp]),
    "pa_sched_plan_pairs": (_c_int, [_vp, _vp, _vp, _vp]),
    "pa_sched_plan_writes": (_c_int, [_vp, _c_int, _vp, _vp, _vp, _vp]),
    "pa_sched_plan_batch": (_c_int, [_vp, _vp, _vp, _vp, _vp]),
    "pa_sched_kv_usage": (_c_int, [_vp, ctypes.POINTER(_c_i64), ctypes.POINTER(_c_i64)]),
    "pa_sched_block_manager": (_vp, [_vp]),
    "pa_sched_attach": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _c_int]),
    "pa_sched_attach_fp8": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _c_int, ctypes.c_float,
                                     ctypes.c_float]),
    "pa_sched_set_cascade": (_c_int, [_vp, _c_int]),
    "pa_sched_last_cascade": (_c_int, [_vp, ctypes.POINTER(_c_int),
                                       ctypes.POINTER(ctypes.c_int64)]),
    "pa_sched_execute": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                  ctypes.c_float, _vp, _vp]),
}

_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded libpa (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m paged_kv_cache_352_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = h
    return _LIB


def last_error() -> str:
    return lib().pa_last_error().decode()


def _check(status: int):
    if status != PA_OK:
        raise PAError(status, last_error())


# --------------------------------------------------------------------------
# tensor marshalling
# --------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float16:
        return PA_F16
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return PA_FP8_E4M3
    raise PAError(PA_ERR_UNSUPPORTED, f"storage type {t.dtype}: expected float16 or bfloat16")


def _dev_ptr(t, name, dtype=None, contiguous=True):
    if t is None:
        return None
    if not t.is_cuda:
        raise PAError(PA_ERR_INVALID_ARG, f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise PAError(PA_ERR_INVALID_ARG, f"{name} must be {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise PAError(PA_ERR_INVALID_ARG, f"{name} must be contiguous")
    return t.data_ptr()


def _device(*tensors):
    """Context in which a call runs: the device of the first CUDA tensor given,
    made current, so that the library's kernels launch on the GPU that holds the
    data and the default stream is that GPU's current stream."""
    import contextlib
    for t in tensors:
        if t is not None and t.is_cuda:
            return _torch().cuda.device(t.device)
    return contextlib.nullcontext()


def _stream(stream):
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _cache_dims(k_cache, v_cache):
    if k_cache.shape != v_cache.shape or k_cache.dtype != v_cache.dtype or k_cache.dim() != 4:
        raise PAError(PA_ERR_INVALID_ARG,
                      "k_cache and v_cache must both be [num_blocks, num_kv_heads, block_size, "
                      "head_dim] with one dtype")
    nb, hkv, bs, d = k_cache.shape
    return nb, hkv, bs, d


# --------------------------------------------------------------------------
# device calls
# --------------------------------------------------------------------------

def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, dev_error=None, stream=None):
    """Store ``key``/``value`` ``[T, num_kv_heads, head_dim]`` at ``slot_mapping`` (int64 [T])."""
    torch = _torch()
    nb, hkv, bs, d = _cache_dims(k_cache, v_cache)
    T = key.shape[0]
    if key.shape[1:] != (hkv, d) or value.shape[1:] != (hkv, d) or value.shape[0] != T:
        raise PAError(PA_ERR_INVALID_ARG, "key/value must be [T, num_kv_heads, head_dim]")
    if key.stride(2) != 1 or key.stride(1) != d or value.stride(2) != 1 or value.stride(1) != d:
        raise PAError(PA_ERR_INVALID_ARG, "key/value rows must be dense per token")
    if slot_mapping.shape != (T,):
        raise PAError(PA_ERR_INVALID_ARG, "slot_mapping must be [T]")
    with _device(k_cache):
        _check(lib().pa_reshape_and_cache(
            _dev_ptr(key, "key", k_cache.dtype, contiguous=False),
            _dev_ptr(value, "value", k_cache.dtype, contiguous=False),
            key.stride(0), value.stride(0),
            _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
            _dev_ptr(slot_mapping, "slot_mapping", torch.int64), T, hkv, d, bs, nb,
            dtype_code(k_cache), _dev_ptr(dev_error, "dev_error", torch.int32), _stream(stream)))


def pa_copy_blocks(k_cache, v_cache, pairs, stream=None):
    """Copy blocks ``pairs[i, 0] -> pairs[i, 1]`` (host int64 array ``[n, 2]``)."""
    nb, hkv, bs, d = _cache_dims(k_cache, v_cache)
    p = np.ascontiguousarray(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
    with _device(k_cache):
        _check(lib().pa_copy_blocks(_dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
                                    p.ctypes.data if len(p) else None, len(p), hkv, d, bs, nb,
                                    dtype_code(k_cache), _stream(stream)))


def _pool_ptr(t, name):
    """Address of a pool tensor on the GPU or in pinned host memory."""
    if not t.is_contiguous():
        raise PAError(PA_ERR_INVALID_ARG, f"{name} must be contiguous")
    if not t.is_cuda and not t.is_pinned():
        raise PAError(PA_ERR_INVALID_ARG, f"{name} must be a CUDA tensor or pinned host memory")
    return t.data_ptr()


def pa_swap_blocks(src_k, src_v, dst_k, dst_v, pairs, stream=None):
    """Copy blocks ``pairs[i, 0]`` of the source pool over ``pairs[i, 1]`` of the
    destination pool; pools are CUDA tensors or pinned host tensors."""
    s_nb, hkv, bs, d = _cache_dims(src_k, src_v)
    d_nb, hkv2, bs2, d2 = _cache_dims(dst_k, dst_v)
    if (hkv, bs, d) != (hkv2, bs2, d2) or src_k.dtype != dst_k.dtype:
        raise PAError(PA_ERR_INVALID_ARG, "source and destination pools differ in layout")
    p = np.ascontiguousarray(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
    with _device(src_k, dst_k):
        _check(lib().pa_swap_blocks(_pool_ptr(src_k, "src_k"), _pool_ptr(src_v, "src_v"), s_nb,
                                    _pool_ptr(dst_k, "dst_k"), _pool_ptr(dst_v, "dst_v"), d_nb,
                                    p.ctypes.data if len(p) else None, len(p), hkv, d, bs,
                                    dtype_code(src_k), _stream(stream)))


def pa_paged_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                   max_context_len, block_size=BLOCK_SIZE, partition_tokens=0):
    out = ctypes.c_size_t(0)
    _check(lib().pa_paged_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                max_context_len, block_size, partition_tokens,
                                                ctypes.byref(out)))
    return out.value


def pa_paged_decode_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                         partition_tokens=0, ordered=False, block_size=BLOCK_SIZE):
    """(blocks per partition, partitions per sequence, kernel launches) of a decode."""
    pb, mp, nl = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().pa_paged_decode_plan(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                      max_context_len, block_size, partition_tokens, int(ordered),
                                      ctypes.byref(pb), ctypes.byref(mp), ctypes.byref(nl)))
    return pb.value, mp.value, nl.value


def pa_paged_decode_cascade_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                 max_blocks_per_seq, num_groups, group_size, max_prefix_blocks,
                                 dtype="f16", fp8_cache=False, block_size=BLOCK_SIZE):
    """The plan of a cascade call with these host bounds: a dict with the prefix's
    blocks per partition and partitions, the own blocks' blocks per partition and
    partitions, and the kernel launches."""
    code = {"f16": PA_F16, "bf16": PA_BF16}[dtype]
    out = [ctypes.c_int(0) for _ in range(5)]
    _check(lib().pa_paged_decode_cascade_plan(
        num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, max_blocks_per_seq,
        block_size, num_groups, group_size, max_prefix_blocks, code, int(bool(fp8_cache)),
        *[ctypes.byref(x) for x in out]))
    keys = ("prefix_part_blocks", "prefix_parts", "own_part_blocks", "own_parts", "launches")
    return dict(zip(keys, (x.value for x in out)))


def decode_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                     partition_tokens=0, device=None):
    """A zero-filled workspace tensor of the size pa_paged_decode needs (None if 0)."""
    torch = _torch()
    n = pa_paged_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                       max_context_len, BLOCK_SIZE, partition_tokens)
    if n == 0:
        return None
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def pa_longest_first_order(context_lens) -> np.ndarray:
    """Host int32 order of sequences by decreasing context length (ties by index)."""
    ctx = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
    order = np.empty(len(ctx), np.int32)
    _check(lib().pa_longest_first_order(ctx.ctypes.data if len(ctx) else None, len(ctx),
                                        order.ctypes.data if len(ctx) else None))
    return order


def pa_cascade_order(context_lens, groups: "PrefixGroups") -> np.ndarray:
    """Host int32 order of sequences by decreasing tokens after their group's
    prefix (ties by index): the recommended ``seq_order`` of
    ``pa_paged_decode_cascade``."""
    ctx = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
    sg = np.ascontiguousarray(groups.seq_group, dtype=np.int32)
    gp = np.ascontiguousarray(groups.prefix_blocks, dtype=np.int32)
    if sg.shape != ctx.shape:
        raise PAError(PA_ERR_INVALID_ARG, "groups must describe this batch")
    order = np.empty(len(ctx), np.int32)
    ng = groups.num_groups
    _check(lib().pa_cascade_order(ctx.ctypes.data if len(ctx) else None,
                                  sg.ctypes.data if ng else None, gp.ctypes.data if ng else None,
                                  ng, len(ctx), order.ctypes.data if len(ctx) else None))
    return order


def pa_paged_decode(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len,
                    scale, partition_tokens=0, workspace=None, dev_error=None, stream=None,
                    seq_order=None):
    """Decode attention through block tables; writes ``out`` ``[B, Hq, d]``.

    ``workspace`` must be a zero-filled uint8 CUDA tensor of at least
    ``pa_paged_decode_workspace_size(...)`` bytes when that size is non-zero.
    ``seq_order`` (int32 CUDA tensor, a permutation) schedules sequences in that
    order; longest first (``pa_longest_first_order``) shortens the launch's tail.
    """
    torch = _torch()
    nb, hkv, bs, d = _cache_dims(k_cache, v_cache)
    B, hq, dq = q.shape
    if dq != d or out.shape != q.shape or out.dtype != k_cache.dtype or q.dtype != k_cache.dtype:
        raise PAError(PA_ERR_INVALID_ARG, "q/out must be [B, num_q_heads, head_dim] in the "
                                          "cache's dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise PAError(PA_ERR_INVALID_ARG, "block_tables must be [B, max_blocks], context_lens [B]")
    ws_bytes = 0
    if workspace is not None:
        ws_bytes = workspace.numel() * workspace.element_size()
    with _device(q):
        _check(lib().pa_paged_decode(
            _dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"),
            _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables", torch.int32),
            block_tables.shape[1], _dev_ptr(context_lens, "context_lens", torch.int32),
            _order_ptr(seq_order, B), B, int(max_context_len), hq, hkv, d, bs, nb, float(scale),
            int(partition_tokens), _dev_ptr(workspace, "workspace"), ws_bytes,
            _dev_ptr(dev_error, "dev_error", torch.int32), dtype_code(k_cache), _stream(stream)))


def pa_reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale,
                             dev_error=None, stream=None):
    """Quantize ``key``/``value`` ``[T, num_kv_heads, head_dim]`` (float16/bfloat16)
    into the E4M3 caches (uint8 or float8_e4m3fn tensors) at ``slot_mapping``."""
    torch = _torch()
    nb, hkv, bs, d = _cache_dims(k_cache, v_cache)
    if dtype_code(k_cache) != PA_FP8_E4M3:
        raise PAError(PA_ERR_INVALID_ARG, "k_cache/v_cache must be uint8 or float8_e4m3fn")
    T = key.shape[0]
    if key.shape[1:] != (hkv, d) or value.shape[1:] != (hkv, d) or value.shape[0] != T:
        raise PAError(PA_ERR_INVALID_ARG, "key/value must be [T, num_kv_heads, head_dim]")
    if key.stride(2) != 1 or key.stride(1) != d or value.stride(2) != 1 or value.stride(1) != d:
        raise PAError(PA_ERR_INVALID_ARG, "key/value rows must be dense per token")
    if value.dtype != key.dtype or slot_mapping.shape != (T,):
        raise PAError(PA_ERR_INVALID_ARG, "value must match key; slot_mapping must be [T]")
    with _device(k_cache):
        _check(lib().pa_reshape_and_cache_fp8(
            _dev_ptr(key, "key", contiguous=False), _dev_ptr(value, "value", contiguous=False),
            key.stride(0), value.stride(0), _dev_ptr(k_cache, "k_cache"),
            _dev_ptr(v_cache, "v_cache"),
            _dev_ptr(slot_mapping, "slot_mapping", torch.int64), T, hkv, d, bs, nb, dtype_code(key),
            float(k_scale), float(v_scale), _dev_ptr(dev_error, "dev_error", torch.int32),
            _stream(stream)))


def pa_paged_decode_fp8(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len,
                        scale, k_scale, v_scale, partition_tokens=0, workspace=None,
                        dev_error=None, stream=None, seq_order=None):
    """pa_paged_decode over E4M3 caches (uint8 / float8_e4m3fn) with key and value
    scales; ``q``/``out`` are float16 or bfloat16."""
    torch = _torch()
    nb, hkv, bs, d = _cache_dims(k_cache, v_cache)
    if dtype_code(k_cache) != PA_FP8_E4M3:
        raise PAError(PA_ERR_INVALID_ARG, "k_cache/v_cache must be uint8 or float8_e4m3fn")
    B, hq, dq = q.shape
    if dq != d or out.shape != q.shape or out.dtype != q.dtype:
        raise PAError(PA_ERR_INVALID_ARG, "q/out must be [B, num_q_heads, head_dim], one dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise PAError(PA_ERR_INVALID_ARG, "block_tables must be [B, max_blocks], context_lens [B]")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _device(q):
        _check(lib().pa_paged_decode_fp8(
            _dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"),
            _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables", torch.int32),
            block_tables.shape[1], _dev_ptr(context_lens, "context_lens", torch.int32),
            _order_ptr(seq_order, B), B, int(max_context_len), hq, hkv, d, bs, nb, float(scale),
            float(k_scale), float(v_scale), int(partition_tokens), _dev_ptr(workspace, "workspace"),
            ws_bytes, _dev_ptr(dev_error, "dev_error", torch.int32), dtype_code(q),
            _stream(stream)))


def pa_paged_decode_cascade_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                           max_context_len, max_blocks_per_seq, num_groups,
                                           group_size, max_prefix_blocks) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().pa_paged_decode_cascade_workspace_size(
        num_seqs, num_q_heads, num_kv_heads, head_dim, int(max_context_len),
        int(max_blocks_per_seq), BLOCK_SIZE, int(num_groups), int(group_size),
        int(max_prefix_blocks), ctypes.byref(n)))
    return n.value


class PrefixGroups:
    """Groups of a batch that share leading blocks (``BlockManager.prefix_groups``),
    as host arrays and, after ``to(device)``, as the device tensors
    ``pa_paged_decode_cascade`` reads."""

    def __init__(self, members, prefix_blocks, seq_group, seq_member, group_size,
                 max_prefix_blocks):
        self.members = members                # int32 [num_groups, group_size], -1 pads
        self.prefix_blocks = prefix_blocks    # int32 [num_groups]
        self.seq_group = seq_group            # int32 [num_seqs]
        self.seq_member = seq_member          # int32 [num_seqs]
        self.group_size = group_size
        self.max_prefix_blocks = max_prefix_blocks
        self.dev = None

    @property
    def num_groups(self) -> int:
        return len(self.prefix_blocks)

    def to(self, device):
        torch = _torch()
        members = self.members if self.num_groups else np.full((1, self.group_size), -1, np.int32)
        prefix = self.prefix_blocks if self.num_groups else np.zeros(1, np.int32)
        self.dev = tuple(torch.from_numpy(np.ascontiguousarray(x)).to(device)
                         for x in (members, prefix, self.seq_group, self.seq_member))
        return self


def cascade_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                      max_blocks_per_seq, groups: PrefixGroups, device=None):
    """A workspace tensor for pa_paged_decode_cascade (each call rewrites it)."""
    torch = _torch()
    n = pa_paged_decode_cascade_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                               max_context_len, max_blocks_per_seq,
                                               groups.num_groups, groups.group_size,
                                               groups.max_prefix_blocks)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def pa_paged_decode_cascade(out, q, k_cache, v_cache, block_tables, context_lens,
                            max_context_len, scale, groups: PrefixGroups, workspace,
                            dev_error=None, stream=None, k_scale=None, v_scale=None,
                            seq_order=None):
    """Decode attention that reads blocks shared by a group's members once; writes
    ``out`` ``[B, Hq, d]``. ``groups`` comes from ``BlockManager.prefix_groups`` for
    the same batch order, moved to the device (``groups.to(device)``). E4M3 caches
    take ``k_scale`` and ``v_scale``. ``seq_order`` (int32 CUDA tensor, a
    permutation) schedules the own-block decode; ``pa_cascade_order`` gives the
    recommended one."""
    torch = _torch()
    nb, hkv, bs, d = _cache_dims(k_cache, v_cache)
    B, hq, dq = q.shape
    fp8 = dtype_code(k_cache) == PA_FP8_E4M3
    if dq != d or out.shape != q.shape or out.dtype != q.dtype or \
            (not fp8 and q.dtype != k_cache.dtype):
        raise PAError(PA_ERR_INVALID_ARG, "q/out must be [B, num_q_heads, head_dim] in the "
                                          "query dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise PAError(PA_ERR_INVALID_ARG, "block_tables must be [B, max_blocks], context_lens [B]")
    if groups.dev is None or groups.seq_group.shape != (B,):
        raise PAError(PA_ERR_INVALID_ARG, "groups must describe this batch and be on the device")
    with _device(q):
        members, prefix, sgroup, smember = groups.dev
        i32 = torch.int32
        head = [_dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"),
                _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables", i32),
                block_tables.shape[1], _dev_ptr(context_lens, "context_lens", i32),
                _order_ptr(seq_order, B), B, int(max_context_len), hq, hkv, d, bs, nb,
                float(scale)]
        tail = [_dev_ptr(members, "group_members", i32),
                _dev_ptr(prefix, "group_prefix_blocks", i32), _dev_ptr(sgroup, "seq_group", i32),
                _dev_ptr(smember, "seq_member", i32),
                groups.num_groups, groups.group_size, groups.max_prefix_blocks,
                _dev_ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                _dev_ptr(dev_error, "dev_error", i32), dtype_code(q), _stream(stream)]
        if fp8:
            if k_scale is None or v_scale is None:
                raise PAError(PA_ERR_INVALID_ARG, "E4M3 caches need k_scale and v_scale")
            _check(lib().pa_paged_decode_cascade_fp8(*head, float(k_scale), float(v_scale), *tail))
        else:
            _check(lib().pa_paged_decode_cascade(*head, *tail))


NOALLOC_WORKSPACE_BYTES = 16 << 20


def _order_ptr(seq_order, B):
    if seq_order is None:
        return None
    if seq_order.shape != (B,):
        raise PAError(PA_ERR_INVALID_ARG, "seq_order must be [num_seqs]")
    return _dev_ptr(seq_order, "seq_order", _torch().int32)


def pa_paged_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens,
                            max_context_len, scale, partition_tokens=0, dev_error=None,
                            stream=None, seq_order=None):
    """Like ``pa_paged_decode`` but without a workspace argument.

    For callers that cannot allocate device memory: the split-KV scratch comes
    from a fixed array built into libpa (``NOALLOC_WORKSPACE_BYTES`` per GPU).
    Calls share that array, so calls that overlap on the GPU must not be issued
    (use one stream). Batches that need more scratch raise ``PAError``. The call
    runs on the device of ``q`` (made current for it), and the library refuses
    tensors or a stream of any other device.
    """
    torch = _torch()
    nb, hkv, bs, d = _cache_dims(k_cache, v_cache)
    B, hq, dq = q.shape
    if dq != d or out.shape != q.shape or out.dtype != k_cache.dtype or q.dtype != k_cache.dtype:
        raise PAError(PA_ERR_INVALID_ARG, "q/out must be [B, num_q_heads, head_dim] in the "
                                          "cache's dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise PAError(PA_ERR_INVALID_ARG, "block_tables must be [B, max_blocks], context_lens [B]")
    with _device(q):
        _check(lib().pa_paged_decode_noalloc(
            _dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"),
            _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables", torch.int32),
            block_tables.shape[1], _dev_ptr(context_lens, "context_lens", torch.int32),
            _order_ptr(seq_order, B), B, int(max_context_len), hq, hkv, d, bs, nb, float(scale),
            int(partition_tokens), _dev_ptr(dev_error, "dev_error", torch.int32),
            dtype_code(k_cache), _stream(stream)))


# --------------------------------------------------------------------------
# host block manager
# --------------------------------------------------------------------------

def _i64p(a):
    return a.ctypes.data if a is not None and a.size else None


class BlockManager:
    """Owner of one ``pa_bm`` handle (the pa_bm_* calls as methods)."""

    @classmethod
    def _borrow(cls, handle, num_blocks: int, block_size: int):
        """A view of a manager owned elsewhere (never destroyed by this object)."""
        self = cls.__new__(cls)
        self._lib = lib()
        self._h = ctypes.c_void_p(handle)
        self._owned = False
        self.num_blocks = num_blocks
        self.block_size = block_size
        return self

    def __init__(self, num_blocks: int, block_size: int = BLOCK_SIZE, initial_free_order=None):
        self._lib = lib()
        order = None
        if initial_free_order is not None:
            order = np.ascontiguousarray(np.asarray(initial_free_order, dtype=np.int32))
            if order.shape != (num_blocks,):
                raise PAError(PA_ERR_INVALID_ARG, "initial_free_order must have num_blocks ids")
        h = ctypes.c_void_p()
        _check(self._lib.pa_bm_create(num_blocks, block_size,
                                      order.ctypes.data if order is not None else None,
                                      ctypes.byref(h)))
        self._h = h
        self._owned = True
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if getattr(self, "_owned", False) and self._h:
            self._lib.pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_seq(self, seq_id: int, num_tokens: int) -> np.ndarray:
        slots = np.empty(max(num_tokens, 0), np.int64)
        _check(self._lib.pa_bm_add_seq(self._h, seq_id, num_tokens, _i64p(slots)))
        return slots

    def fork(self, parent: int, child: int) -> None:
        _check(self._lib.pa_bm_fork(self._h, parent, child))

    def append_slots(self, seq_id: int, n: int):
        slots = np.empty(max(n, 0), np.int64)
        pairs = np.empty(2, np.int64)
        ncow = ctypes.c_int(0)
        _check(self._lib.pa_bm_append_slots(self._h, seq_id, n, _i64p(slots), pairs.ctypes.data,
                                            ctypes.byref(ncow)))
        return slots, pairs[:2 * ncow.value].reshape(-1, 2).copy()

    def free_seq(self, seq_id: int) -> None:
        _check(self._lib.pa_bm_free_seq(self._h, seq_id))

    def block_tables(self, seq_ids, max_blocks: int) -> np.ndarray:
        ids = np.ascontiguousarray(np.asarray(list(seq_ids), dtype=np.int64))
        out = np.empty((len(ids), max_blocks), np.int32)
        _check(self._lib.pa_bm_block_tables(self._h, _i64p(ids), len(ids),
                                            out.ctypes.data if out.size else None, max_blocks))
        return out

    def prefix_groups(self, seq_ids, group_size: int) -> "PrefixGroups":
        """Groups of the batch ``seq_ids`` that hold the same leading blocks
        (``pa_bm_prefix_groups``); members are batch indices."""
        ids = np.ascontiguousarray(np.asarray(list(seq_ids), dtype=np.int64))
        n = len(ids)
        members = np.empty((max(n, 1), group_size), np.int32)
        prefix = np.empty(max(n, 1), np.int32)
        sgroup = np.empty(max(n, 1), np.int32)
        smember = np.empty(max(n, 1), np.int32)
        ng, mp = _c_int(0), _c_int(0)
        _check(self._lib.pa_bm_prefix_groups(self._h, _i64p(ids), n, group_size,
                                             members.ctypes.data, prefix.ctypes.data,
                                             sgroup.ctypes.data, smember.ctypes.data,
                                             ctypes.byref(ng), ctypes.byref(mp)))
        k = ng.value
        return PrefixGroups(members[:k].copy(), prefix[:k].copy(), sgroup[:n].copy(),
                            smember[:n].copy(), group_size, mp.value)

    def num_free(self) -> int:
        return self._lib.pa_bm_num_free(self._h)

    def refcount(self, block: int) -> int:
        r = self._lib.pa_bm_refcount(self._h, block)
        if r < 0:
            raise PAError(PA_ERR_INVALID_ARG, last_error())
        return r

    def seq_len(self, seq_id: int) -> int:
        r = self._lib.pa_bm_seq_len(self._h, seq_id)
        if r < 0:
            raise PAError(PA_ERR_UNKNOWN_SEQ, last_error())
        return r

    def num_seqs(self) -> int:
        return self._lib.pa_bm_num_seqs(self._h)

    def free_list(self) -> list:
        out = np.empty(self.num_blocks, np.int32)
        n = self._lib.pa_bm_free_list(self._h, out.ctypes.data, self.num_blocks)
        return out[:n].tolist()

    def table(self, seq_id: int) -> list:
        if self.is_swapped(seq_id):
            return []
        n = -(-self.seq_len(seq_id) // self.block_size)
        return self.block_tables([seq_id], max(n, 1))[0, :n].tolist()

    # -- prefix caching ----------------------------------------------------------
    def add_seq_cached(self, seq_id: int, token_ids):
        """Register from prompt token ids; returns (slots, num_cached_tokens)."""
        toks = np.ascontiguousarray(np.asarray(list(token_ids), dtype=np.int32))
        slots = np.empty(max(len(toks), 1), np.int64)
        cached = ctypes.c_int(0)
        _check(self._lib.pa_bm_add_seq_cached(self._h, seq_id, toks.ctypes.data, len(toks),
                                              slots.ctypes.data, ctypes.byref(cached)))
        return slots[:len(toks)].copy(), cached.value

    def num_cached(self) -> int:
        return self._lib.pa_bm_num_cached(self._h)

    def cached_prefix(self, token_ids):
        """(leading full blocks found in the cache, how many of them are evictable)."""
        toks = np.ascontiguousarray(np.asarray(list(token_ids), dtype=np.int32))
        hits, revived = ctypes.c_int(0), ctypes.c_int(0)
        _check(self._lib.pa_bm_cached_prefix(self._h, toks.ctypes.data if len(toks) else None,
                                             len(toks), ctypes.byref(hits), ctypes.byref(revived)))
        return hits.value, revived.value

    def evictable_list(self) -> list:
        out = np.empty(max(self.num_blocks, 1), np.int32)
        n = self._lib.pa_bm_evictable_list(self._h, out.ctypes.data, self.num_blocks)
        return out[:n].tolist()

    # -- swapping ----------------------------------------------------------------
    def set_host_pool(self, num_host_blocks: int) -> None:
        _check(self._lib.pa_bm_set_host_pool(self._h, num_host_blocks))
        self.num_host_blocks = num_host_blocks

    def _swap(self, fn, seq_id):
        n = -(-self.seq_len(seq_id) // self.block_size)
        pairs = np.empty((max(n, 1), 2), np.int64)
        cnt = ctypes.c_int(0)
        _check(fn(self._h, seq_id, pairs.ctypes.data, n, ctypes.byref(cnt)))
        return pairs[:cnt.value].copy()

    def swap_out(self, seq_id: int) -> np.ndarray:
        """(device block, host block) copy pairs, in logical order."""
        return self._swap(self._lib.pa_bm_swap_out, seq_id)

    def swap_in(self, seq_id: int) -> np.ndarray:
        """(host block, device block) copy pairs, in logical order."""
        return self._swap(self._lib.pa_bm_swap_in, seq_id)

    def is_swapped(self, seq_id: int) -> bool:
        r = self._lib.pa_bm_is_swapped(self._h, seq_id)
        if r < 0:
            raise PAError(PA_ERR_UNKNOWN_SEQ, last_error())
        return bool(r)

    def num_free_host(self) -> int:
        return self._lib.pa_bm_num_free_host(self._h)

    def host_free_list(self) -> list:
        n = max(self.num_free_host(), 1)
        out = np.empty(n, np.int32)
        m = self._lib.pa_bm_host_free_list(self._h, out.ctypes.data, n)
        return out[:m].tolist()


# --------------------------------------------------------------------------
# continuous batching
# --------------------------------------------------------------------------

PA_SCHED_MAX_SAMPLES = 64
PA_SCHED_CASCADE_OFF = 0
PA_SCHED_CASCADE_ON = 1
PA_SCHED_CASCADE_AUTO = 2
PA_PREEMPT_SWAP = 0
PA_PREEMPT_RECOMPUTE = 1


class SchedPlanCounts(ctypes.Structure):
    _fields_ = [("step", ctypes.c_int64), ("num_finished", ctypes.c_int),
                ("num_preempted", ctypes.c_int), ("num_resumed", ctypes.c_int),
                ("num_admitted", ctypes.c_int), ("num_swap_out", ctypes.c_int),
                ("num_swap_in", ctypes.c_int), ("num_copies", ctypes.c_int),
                ("num_prefill", ctypes.c_int), ("num_writes", ctypes.c_int),
                ("num_seqs", ctypes.c_int), ("max_blocks_per_seq", ctypes.c_int),
                ("max_context_len", ctypes.c_int), ("total_context", ctypes.c_int64),
                ("num_cached_tokens", ctypes.c_int64)]


def _p(a):
    return a.ctypes.data if a is not None and a.size else None


class Scheduler:
    """Owner of one ``pa_sched`` handle: iteration-level batching over a block
    manager (pa_sched_* calls as methods) and the executor of planned steps."""

    def __init__(self, num_blocks: int, block_size: int = BLOCK_SIZE, initial_free_order=None,
                 max_num_seqs: int = 256, num_host_blocks: int = 0,
                 preempt_mode: int = PA_PREEMPT_SWAP):
        self._lib = lib()
        order = None
        if initial_free_order is not None:
            order = np.ascontiguousarray(np.asarray(initial_free_order, dtype=np.int32))
            if order.shape != (num_blocks,):
                raise PAError(PA_ERR_INVALID_ARG, "initial_free_order must have num_blocks ids")
        h = ctypes.c_void_p()
        _check(self._lib.pa_sched_create(num_blocks, block_size,
                                         order.ctypes.data if order is not None else None,
                                         max_num_seqs, num_host_blocks, preempt_mode,
                                         ctypes.byref(h)))
        self._h = h
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.max_num_seqs = max_num_seqs
        self.num_host_blocks = num_host_blocks
        self.bm = BlockManager._borrow(self._lib.pa_sched_block_manager(h), num_blocks,
                                       block_size)
        self.counts = None

    def close(self):
        if getattr(self, "_h", None):
            self._lib.pa_sched_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def submit(self, request_id: int, prompt_len: int, output_len: int, num_samples: int = 1,
               arrival: int = 0, tokens=None) -> None:
        """Queue a request; with ``tokens`` (the prompt's token ids) it is admitted
        through the prefix cache."""
        if tokens is None:
            _check(self._lib.pa_sched_submit(self._h, request_id, prompt_len, output_len,
                                             num_samples, arrival))
            return
        toks = np.ascontiguousarray(np.asarray(list(tokens), dtype=np.int32))
        if len(toks) != prompt_len:
            raise PAError(PA_ERR_INVALID_ARG, "one token id per prompt position")
        _check(self._lib.pa_sched_submit_tokens(self._h, request_id,
                                                toks.ctypes.data if len(toks) else None,
                                                prompt_len, output_len, num_samples, arrival))

    def step(self) -> SchedPlanCounts:
        c = SchedPlanCounts()
        _check(self._lib.pa_sched_step(self._h, ctypes.byref(c)))
        self.counts = c
        return c

    def idle(self) -> bool:
        return bool(self._lib.pa_sched_idle(self._h))

    def kv_usage(self):
        f, a = ctypes.c_int64(0), ctypes.c_int64(0)
        _check(self._lib.pa_sched_kv_usage(self._h, ctypes.byref(f), ctypes.byref(a)))
        return f.value, a.value

    def plan(self) -> dict:
        """The last planned step in full, as plain lists (the oracle's Plan fields)."""
        c = self.counts
        fin = np.empty(c.num_finished, np.int64)
        pre = np.empty(c.num_preempted, np.int64)
        mode = np.empty(c.num_preempted, np.int32)
        res = np.empty(c.num_resumed, np.int64)
        adm = np.empty(c.num_admitted, np.int64)
        _check(self._lib.pa_sched_plan_requests(self._h, _p(fin), _p(pre), _p(mode), _p(res),
                                                _p(adm)))
        so = np.empty((c.num_swap_out, 2), np.int64)
        si = np.empty((c.num_swap_in, 2), np.int64)
        cp = np.empty((c.num_copies, 2), np.int64)
        _check(self._lib.pa_sched_plan_pairs(self._h, _p(so), _p(si), _p(cp)))
        writes = {}
        for which, n in ((0, c.num_prefill), (1, c.num_writes)):
            r = np.empty(n, np.int64)
            sm = np.empty(n, np.int32)
            pos = np.empty(n, np.int32)
            sl = np.empty(n, np.int64)
            _check(self._lib.pa_sched_plan_writes(self._h, which, _p(r), _p(sm), _p(pos), _p(sl)))
            writes[which] = [tuple(int(x) for x in t) for t in zip(r, sm, pos, sl)]
        br = np.empty(c.num_seqs, np.int64)
        bsm = np.empty(c.num_seqs, np.int32)
        ctx = np.empty(c.num_seqs, np.int32)
        tables = np.empty((c.num_seqs, c.max_blocks_per_seq), np.int32)
        _check(self._lib.pa_sched_plan_batch(self._h, _p(br), _p(bsm), _p(ctx), _p(tables)))
        pairs = lambda a: [tuple(int(x) for x in row) for row in a]
        return {
            "step": int(c.step),
            "finished": fin.tolist(),
            "preempted": list(zip(pre.tolist(), mode.tolist())),
            "resumed": res.tolist(),
            "admitted": adm.tolist(),
            "swap_out": pairs(so), "swap_in": pairs(si), "copies": pairs(cp),
            "prefill": writes[0], "writes": writes[1],
            "batch": list(zip(br.tolist(), bsm.tolist(), ctx.tolist())),
            "cached": int(c.num_cached_tokens),
            "tables": tables,
        }

    def attach(self, num_q_heads: int, num_kv_heads: int, head_dim: int, dtype,
               max_context_len: int, fp8_scales=None) -> None:
        """Allocate the executor for queries/inputs of ``dtype``; with
        ``fp8_scales=(k_scale, v_scale)`` the pools are 8-bit E4M3 caches."""
        code = dtype if isinstance(dtype, int) else (
            PA_F16 if dtype == _torch().float16 else PA_BF16)
        if fp8_scales is None:
            _check(self._lib.pa_sched_attach(self._h, num_q_heads, num_kv_heads, head_dim, code,
                                             max_context_len))
        else:
            _check(self._lib.pa_sched_attach_fp8(self._h, num_q_heads, num_kv_heads, head_dim,
                                                 code, max_context_len, float(fp8_scales[0]),
                                                 float(fp8_scales[1])))
        self.io_dtype = code
        self.fp8 = fp8_scales is not None

    def set_cascade(self, mode: int) -> None:
        """When the executor decodes sequences that share leading blocks through
        the cascade: PA_SCHED_CASCADE_OFF, _ON or _AUTO (the default)."""
        _check(self._lib.pa_sched_set_cascade(self._h, int(mode)))

    def last_cascade(self):
        """(groups decoded through the cascade in the last executed step, block
        reads that saved); (0, 0) when that step used the plain decode."""
        ng, saved = _c_int(0), ctypes.c_int64(0)
        _check(self._lib.pa_sched_last_cascade(self._h, ctypes.byref(ng), ctypes.byref(saved)))
        return ng.value, saved.value

    def execute(self, k_cache, v_cache, host_k, host_v, prefill_key, prefill_value, key, value,
                q, out, scale: float, dev_error=None, stream=None) -> None:
        """Run the last planned step (pa_sched_execute). Inputs are device tensors
        whose leading dimension covers the plan's counts; host_k/host_v are the
        pinned host pool (or None)."""
        torch = _torch()
        if (dtype_code(k_cache) == PA_FP8_E4M3) != getattr(self, "fp8", False):
            raise PAError(PA_ERR_INVALID_ARG, "cache element type differs from the attached one")
        cdt = k_cache.dtype
        dt = q.dtype
        host = lambda t, n: None if t is None else _pool_ptr(t, n)
        with _device(k_cache):
            _check(self._lib.pa_sched_execute(
                self._h, _dev_ptr(k_cache, "k_cache", cdt), _dev_ptr(v_cache, "v_cache", cdt),
                host(host_k, "host_k"), host(host_v, "host_v"),
                _dev_ptr(prefill_key, "prefill_key", dt),
                _dev_ptr(prefill_value, "prefill_value", dt),
                _dev_ptr(key, "key", dt), _dev_ptr(value, "value", dt), _dev_ptr(q, "q", dt),
                _dev_ptr(out, "out", dt), scale, _dev_ptr(dev_error, "dev_error", torch.int32),
                _stream(stream)))
