"""Block manager of the paged KV cache, restated in plain Python (oracle side).

What the pages fix:
  * The cache is a pool of equal fixed-size blocks, each holding the keys and
    values of 16 tokens, allocated once up front ("PagedAttention: The vLLM
    Paper", "The Core Idea" figure and "Implementation Essentials").
  * Each sequence has a block table mapping its logical blocks to physical
    ones; blocks are taken on demand as tokens arrive and only the last block
    of a sequence can be partly filled ("PagedAttention and Continuous
    Batching", "Pages, from operating systems"; "PagedAttention: The vLLM
    Paper", "The design yields three immediate wins", item 1).
  * Blocks are reference counted so sequences can share them; a shared block
    is copied only when one sequence has to write into it, as with fork and
    copy-on-write in an operating system ("Pages, from operating systems";
    "The OS paging analogy" table; "Implementation Essentials").
  * Finished sequences return their blocks to the pool for any request to use
    ("The Core Idea" figure caption).

Readings where the pages are silent (the CUDA-side library follows the same
rules so that tables can be compared bit for bit):
  * The free list is a stack. ``initial_free_order[0]`` is handed out first;
    freed blocks go on top and are reused first.
  * ``free_seq`` releases a sequence's blocks from its last logical block to
    its first.
  * Copy-on-write happens when an append writes into a partly filled last
    block whose refcount is above one: the appending sequence gets a fresh
    block, a ``(old, new)`` copy pair is emitted and the old block's count
    drops by one. A sequence whose last block has refcount one writes in place.
  * Every call is all-or-nothing: when the pool cannot cover it, nothing changes.
  * Block tables are padded with -1.

Swapping (preemption when the pool runs short: a request's blocks move to CPU
memory and come back later — "PagedAttention: The vLLM Paper", "Implementation
Essentials" and "The OS paging analogy", swapping), read as:
  * A host pool of equal blocks with its own stack free list, set once.
  * ``swap_out`` gives each of the sequence's blocks a host block, in logical
    order, and emits ``(device block, host block)`` pairs; the device
    refcounts drop by one and blocks reaching zero return to the device free
    list, last logical block first (as ``free_seq``). A block still shared with
    resident sequences stays on the device for them; the swapped sequence takes
    its own host copy. The caller copies the pairs before the freed device
    blocks are written again.
  * ``swap_in`` gives each host block a fresh device block, in logical order,
    emits ``(host block, device block)`` pairs, and returns the host blocks to
    the host free list, last logical block first.
  * A swapped sequence cannot append, fork, be swapped out again or appear in
    block tables; ``free_seq`` releases its host blocks.

Prefix caching across requests (the KV of shared prompt prefixes is kept and
reused by later requests, so a hit makes prefill nearly free — "PagedAttention:
The vLLM Paper", "Impact and Follow-Ups", item 1), read as:
  * ``add_seq_cached`` takes the prompt's token ids. Every full block of the
    prompt is identified exactly by (physical block of the previous logical
    block, or -1 for the first; the block's 16 token ids). Leading full blocks
    found in the cache are shared (refcount + 1); the first miss and everything
    after it get fresh blocks, and the new full blocks join the cache. The
    partly filled last block is never cached, so writes never touch a cached
    block. The call reports how many leading tokens need no write.
  * A cached block whose refcount falls to 0 is not freed but kept for reuse,
    queued least recently released first. Blocks are taken from the free list
    first and, when it is empty, by evicting the head of that queue. Tables are
    released last block first and a table holding a block holds its whole
    prefix, so a block is never queued before its cached descendants and
    eviction takes leaves first; evicting a block nevertheless also evicts any
    cached descendant, so no cache key can name a block that now holds other
    tokens.
  * ``num_free`` counts free plus evictable blocks.
"""

from __future__ import annotations

import numpy as np

# Status codes shared in meaning with the C interface.
OK = 0
ERR_INVALID_ARG = 1
ERR_NO_FREE_BLOCKS = 2
ERR_UNKNOWN_SEQ = 3
ERR_SEQ_EXISTS = 6
ERR_SEQ_SWAPPED = 7


class BlockManagerError(Exception):
    def __init__(self, code: int, msg: str):
        super().__init__(msg)
        self.code = code


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int, initial_free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise BlockManagerError(ERR_INVALID_ARG, "num_blocks and block_size must be positive")
        if initial_free_order is None:
            order = list(range(num_blocks))
        else:
            order = [int(b) for b in initial_free_order]
            if sorted(order) != list(range(num_blocks)):
                raise BlockManagerError(ERR_INVALID_ARG,
                                        "initial_free_order must be a permutation of the pool")
        self.num_blocks = num_blocks
        self.block_size = block_size
        # Top of the stack is the end of the list, so order[0] is popped first.
        self._free = list(reversed(order))
        self._ref = [0] * num_blocks
        self._tables: dict[int, list[int]] = {}
        self._lens: dict[int, int] = {}
        self._host_free: list[int] = []
        self.num_host_blocks = 0
        self._swapped: dict[int, list[int]] = {}   # seq -> host blocks in logical order
        self._cache: dict = {}          # (parent block, tokens) -> block
        self._key_of: dict = {}         # cached block -> its key
        self._children: dict = {}       # cached block -> set of cached child blocks
        self._evictable: list[int] = [] # cached blocks with refcount 0, oldest first

    def set_host_pool(self, num_host_blocks: int) -> None:
        if num_host_blocks < 0:
            raise BlockManagerError(ERR_INVALID_ARG, "num_host_blocks must be >= 0")
        if self._swapped:
            raise BlockManagerError(ERR_INVALID_ARG, "host blocks are in use")
        self.num_host_blocks = num_host_blocks
        self._host_free = list(reversed(range(num_host_blocks)))

    def num_free_host(self) -> int:
        return len(self._host_free)

    def is_swapped(self, seq_id: int) -> bool:
        self._need(seq_id)
        return seq_id in self._swapped

    def swap_out(self, seq_id: int):
        """Move the sequence to host blocks; return ``(device, host)`` copy pairs."""
        self._need(seq_id)
        self._resident(seq_id)
        table = self._tables[seq_id]
        if len(table) > len(self._host_free):
            raise BlockManagerError(ERR_NO_FREE_BLOCKS, "host pool exhausted")
        host = [self._host_free.pop() for _ in table]
        pairs = list(zip(table, host))
        for b in reversed(table):
            self._release(b)
        self._tables[seq_id] = []
        self._swapped[seq_id] = host
        return pairs

    def swap_in(self, seq_id: int):
        """Bring a swapped sequence back; return ``(host, device)`` copy pairs."""
        self._need(seq_id)
        if seq_id not in self._swapped:
            raise BlockManagerError(ERR_SEQ_SWAPPED, f"sequence {seq_id} is not swapped out")
        host = self._swapped[seq_id]
        if len(host) > self.num_free():
            raise BlockManagerError(ERR_NO_FREE_BLOCKS, "pool exhausted")
        table = [self._take() for _ in host]
        pairs = list(zip(host, table))
        for h in reversed(host):
            self._host_free.append(h)
        del self._swapped[seq_id]
        self._tables[seq_id] = table
        return pairs

    def _resident(self, seq_id):
        if seq_id in self._swapped:
            raise BlockManagerError(ERR_SEQ_SWAPPED, f"sequence {seq_id} is swapped out")

    # -- queries ---------------------------------------------------------
    def num_free(self) -> int:
        return len(self._free) + len(self._evictable)

    def num_cached(self) -> int:
        return len(self._key_of)

    def evictable_list(self) -> list[int]:
        return list(self._evictable)

    def refcount(self, block: int) -> int:
        if not 0 <= block < self.num_blocks:
            raise BlockManagerError(ERR_INVALID_ARG, "block id out of range")
        return self._ref[block]

    def seq_len(self, seq_id: int) -> int:
        self._need(seq_id)
        return self._lens[seq_id]

    def table(self, seq_id: int) -> list[int]:
        self._need(seq_id)
        return list(self._tables[seq_id])

    def host_table(self, seq_id: int) -> list[int]:
        self._need(seq_id)
        return list(self._swapped.get(seq_id, []))

    def host_free_list(self) -> list[int]:
        return list(reversed(self._host_free))

    def seq_ids(self):
        return list(self._tables)

    def free_list(self) -> list[int]:
        """Free blocks in the order they would be handed out."""
        return list(reversed(self._free))

    # -- helpers ---------------------------------------------------------
    def _need(self, seq_id):
        if seq_id not in self._tables:
            raise BlockManagerError(ERR_UNKNOWN_SEQ, f"unknown sequence {seq_id}")

    def _take(self) -> int:
        """A block for new tokens: the free list first, else evict the oldest
        released cached block (with its cached descendants)."""
        if not self._free:
            self._evict(self._evictable[0])
        b = self._free.pop()
        self._ref[b] = 1
        return b

    def _evict(self, b: int) -> None:
        for c in sorted(self._children.pop(b, ())):
            self._evict(c)
        key = self._key_of.pop(b)
        del self._cache[key]
        if key[0] >= 0:
            self._children[key[0]].discard(b)
        self._evictable.remove(b)
        self._free.append(b)

    def _release(self, b: int) -> None:
        self._ref[b] -= 1
        if self._ref[b] == 0:
            if b in self._key_of:
                self._evictable.append(b)
            else:
                self._free.append(b)

    def _slot(self, table, pos):
        return table[pos // self.block_size] * self.block_size + pos % self.block_size

    # -- mutations -------------------------------------------------------
    def add_seq(self, seq_id: int, num_tokens: int) -> list[int]:
        """Register a sequence holding ``num_tokens`` tokens; return their slots."""
        if num_tokens < 0:
            raise BlockManagerError(ERR_INVALID_ARG, "num_tokens must be >= 0")
        if seq_id in self._tables:
            raise BlockManagerError(ERR_SEQ_EXISTS, f"sequence {seq_id} exists")
        need = _ceil_div(num_tokens, self.block_size)
        if need > self.num_free():
            raise BlockManagerError(ERR_NO_FREE_BLOCKS, "pool exhausted")
        table = [self._take() for _ in range(need)]
        self._tables[seq_id] = table
        self._lens[seq_id] = num_tokens
        return [self._slot(table, p) for p in range(num_tokens)]

    def cached_prefix(self, token_ids):
        """(leading full blocks of these prompt tokens found in the cache, how many
        of them are evictable, i.e. held by no sequence); changes nothing."""
        tokens = [int(t) for t in token_ids]
        bs = self.block_size
        hits = revived = 0
        parent = -1
        for i in range(len(tokens) // bs):
            b = self._cache.get((parent, tuple(tokens[i * bs:(i + 1) * bs])))
            if b is None:
                break
            hits += 1
            revived += self._ref[b] == 0
            parent = b
        return hits, revived

    def add_seq_cached(self, seq_id: int, token_ids):
        """Register a sequence from its prompt's token ids, sharing the leading
        full blocks already cached. Returns ``(slots, num_cached_tokens)``; the
        first ``num_cached_tokens`` tokens' keys and values are already in place."""
        tokens = [int(t) for t in token_ids]
        n = len(tokens)
        if seq_id in self._tables:
            raise BlockManagerError(ERR_SEQ_EXISTS, f"sequence {seq_id} exists")
        bs = self.block_size
        full = n // bs
        hits, parent = [], -1
        for i in range(full):
            b = self._cache.get((parent, tuple(tokens[i * bs:(i + 1) * bs])))
            if b is None:
                break
            hits.append(b)
            parent = b
        need = _ceil_div(n, bs) - len(hits)
        revived = sum(1 for b in hits if self._ref[b] == 0)
        if need > self.num_free() - revived:
            raise BlockManagerError(ERR_NO_FREE_BLOCKS, "pool exhausted")
        for b in hits:
            if self._ref[b] == 0:
                self._evictable.remove(b)
            self._ref[b] += 1
        table = list(hits)
        for i in range(len(hits), _ceil_div(n, bs)):
            b = self._take()
            table.append(b)
            if i < full:
                key = (parent, tuple(tokens[i * bs:(i + 1) * bs]))
                self._cache[key] = b
                self._key_of[b] = key
                if parent >= 0:
                    self._children.setdefault(parent, set()).add(b)
                parent = b
        self._tables[seq_id] = table
        self._lens[seq_id] = n
        return [self._slot(table, p) for p in range(n)], len(hits) * bs

    def fork(self, parent: int, child: int) -> None:
        """Child starts as a copy of the parent's table; every block is shared."""
        self._need(parent)
        self._resident(parent)
        if child in self._tables:
            raise BlockManagerError(ERR_SEQ_EXISTS, f"sequence {child} exists")
        table = list(self._tables[parent])
        for b in table:
            self._ref[b] += 1
        self._tables[child] = table
        self._lens[child] = self._lens[parent]

    def append_slots(self, seq_id: int, n: int):
        """Append ``n`` tokens; return ``(slots, cow_pairs)``."""
        self._need(seq_id)
        self._resident(seq_id)
        if n < 0:
            raise BlockManagerError(ERR_INVALID_ARG, "n must be >= 0")
        table = self._tables[seq_id]
        length = self._lens[seq_id]
        bs = self.block_size
        new_blocks = _ceil_div(length + n, bs) - len(table)
        cow = n > 0 and length % bs != 0 and self._ref[table[-1]] > 1
        if new_blocks + int(cow) > self.num_free():
            raise BlockManagerError(ERR_NO_FREE_BLOCKS, "pool exhausted")
        pairs = []
        if cow:
            old = table[-1]
            new = self._take()
            self._ref[old] -= 1   # still held by its other sharers
            table[-1] = new
            pairs.append((old, new))
        slots = []
        for p in range(length, length + n):
            if p % bs == 0:
                table.append(self._take())
            slots.append(self._slot(table, p))
        self._lens[seq_id] = length + n
        return slots, pairs

    def free_seq(self, seq_id: int) -> None:
        self._need(seq_id)
        for h in reversed(self._swapped.pop(seq_id, [])):
            self._host_free.append(h)
        for b in reversed(self._tables[seq_id]):
            self._release(b)
        del self._tables[seq_id]
        del self._lens[seq_id]

    def block_tables(self, seq_ids, max_blocks: int) -> np.ndarray:
        """Tables of ``seq_ids`` as int32 ``[n, max_blocks]``, padded with -1."""
        seq_ids = list(seq_ids)
        out = np.full((len(seq_ids), max_blocks), -1, dtype=np.int32)
        for i, s in enumerate(seq_ids):
            self._need(s)
            self._resident(s)
            t = self._tables[s]
            if len(t) > max_blocks:
                raise BlockManagerError(ERR_INVALID_ARG, "table longer than max_blocks")
            out[i, :len(t)] = t
        return out

    def prefix_groups(self, seq_ids, group_size: int):
        """Groups of the batch ``seq_ids`` whose members hold the same leading
        blocks, for decoding a shared prefix once (a reading of this build: the
        pages share a prompt's blocks among forks, "Implementation Essentials",
        prefix sharing, but name no grouping rule).

        Sequences with at least one full block are bucketed by their first block
        id; buckets keep the order in which their first member appears, members
        keep batch order. Each bucket is cut into consecutive runs of
        ``group_size``; a run of two or more is a group whose prefix is the
        number of leading block ids shared by all its members, capped at every
        member's count of full blocks; a run whose prefix is 0 is no group.

        Returns ``(members, prefix_blocks, seq_group, seq_member)``: a list of
        member lists (batch indices), a list of prefix lengths, and per batch
        index its group and slot (-1 when it has none).
        """
        seq_ids = list(seq_ids)
        for s in seq_ids:
            self._need(s)
            self._resident(s)
        full = [self._lens[s] // self.block_size for s in seq_ids]
        buckets: dict[int, list[int]] = {}
        for i, s in enumerate(seq_ids):
            if full[i] >= 1:
                buckets.setdefault(self._tables[s][0], []).append(i)
        members, prefix = [], []
        seq_group = [-1] * len(seq_ids)
        seq_member = [-1] * len(seq_ids)
        for run_source in buckets.values():
            for c in range(0, len(run_source), group_size):
                run = run_source[c:c + group_size]
                if len(run) < 2:
                    continue
                tables = [self._tables[seq_ids[i]] for i in run]
                p = min(full[i] for i in run)
                shared = 0
                while shared < p and all(t[shared] == tables[0][shared] for t in tables):
                    shared += 1
                if shared == 0:
                    continue
                for slot, i in enumerate(run):
                    seq_group[i] = len(members)
                    seq_member[i] = slot
                members.append(run)
                prefix.append(shared)
        return members, prefix, seq_group, seq_member
