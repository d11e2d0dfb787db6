"""Writing new tokens into the paged cache, and whole-block copies (oracle side).

Both are plain copies of bit patterns, written as loops over tokens and pairs.

Cache layout (fixed by the C interface; the pages fix none): one array for
keys and one for values, each ``[num_blocks, num_kv_heads, block_size,
head_dim]``. Slot ``s`` is offset ``s % block_size`` of physical block
``s // block_size``, the same numbering the block manager uses when it maps a
token position through the block table ("PagedAttention and Continuous
Batching", "Pages, from operating systems").
"""

import numpy as np


def reshape_and_cache(k_cache, v_cache, key, value, slot_mapping, block_size: int):
    """Store token ``t``'s keys/values ``[num_kv_heads, head_dim]`` at its slot.

    ``slot_mapping[t] < 0`` means the token is not stored. Modifies the caches
    in place (they are uint16 bit-pattern arrays).
    """
    key = np.asarray(key)
    value = np.asarray(value)
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64).tolist()):
        if slot < 0:
            continue
        block, offset = divmod(slot, block_size)
        k_cache[block, :, offset, :] = key[t]
        v_cache[block, :, offset, :] = value[t]


def copy_blocks(k_cache, v_cache, pairs):
    """Copy physical block ``src`` over ``dst`` in both caches, for each pair.

    This is the copy half of copy-on-write: the block manager has already
    pointed the writer's table at ``dst`` ("Pages, from operating systems";
    "The OS paging analogy", page sharing by fork and copy-on-write).
    """
    for src, dst in np.asarray(pairs, dtype=np.int64).reshape(-1, 2).tolist():
        k_cache[dst] = k_cache[src].copy()
        v_cache[dst] = v_cache[src].copy()


def swap_blocks(src_k, src_v, dst_k, dst_v, pairs):
    """Copy block ``src`` of the source pool over block ``dst`` of the destination
    pool (device -> host on swap-out, host -> device on swap-in), K and V."""
    for src, dst in np.asarray(pairs, dtype=np.int64).reshape(-1, 2).tolist():
        dst_k[dst] = src_k[src].copy()
        dst_v[dst] = src_v[src].copy()
