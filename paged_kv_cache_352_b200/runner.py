"""Drives decode steps of a workload through libpa (block manager + kernels).

The order of a step is the method's: the block manager hands out the new
tokens' slots (and copy-on-write pairs), shared blocks are copied, the new
tokens' keys and values are written into their slots, and decode attention
reads the cache through the block tables ("PagedAttention and Continuous
Batching", "Pages, from operating systems"; "PagedAttention: The vLLM Paper",
"Implementation Essentials").

Two kinds of workloads are supported, matching ``workloads.configs``:
  * independent sequences: sequence s holds ctx_s - 1 earlier tokens (written
    with pa_reshape_and_cache once, at set-up); each step writes token ctx_s - 1
    and decodes over ctx_s tokens;
  * prompts forked into samples: each prompt is written once and forked; the
    step applies the samples' copy-on-write pairs, writes their own tokens and
    decodes every sample. With ``duplicate=True`` every sample instead gets a
    private copy of the prompt (same logical sequences, no sharing).

The pool is allocated once, at set-up, with PyTorch; steps allocate nothing.
Re-running a step rewrites the same slots with the same values, so steps can be
repeated for timing.
"""

from __future__ import annotations

import numpy as np
import torch

from workloads import gen

from . import _lib as L

_TORCH_DTYPE = {"f16": torch.float16, "bf16": torch.bfloat16}


def _to_dev(bits: np.ndarray, dtype: str, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits)).view(_TORCH_DTYPE[dtype])
    return t.to(device, non_blocking=False)


class DecodeRunner:
    def __init__(self, wl, device="cuda", partition_tokens=None, duplicate=False):
        self.wl = wl
        self.duplicate = duplicate
        self.device = torch.device(device)
        self.dtype = _TORCH_DTYPE[wl.dtype]
        self.partition_tokens = wl.partition_tokens if partition_tokens is None else partition_tokens
        shape = (wl.num_blocks, wl.num_kv_heads, wl.block_size, wl.head_dim)
        self.k_cache = torch.zeros(shape, dtype=self.dtype, device=self.device)
        self.v_cache = torch.zeros(shape, dtype=self.dtype, device=self.device)
        self.bm = L.BlockManager(wl.num_blocks, wl.block_size, wl.free_order)
        self.dev_error = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.prefill_slots = []
        if wl.kind == "shared_prefix":
            self._setup_shared()
        else:
            self._setup_decode()
        self.max_blocks = wl.max_blocks_per_seq
        self.block_tables_host = self.bm.block_tables(range(wl.num_seqs), self.max_blocks)
        self.block_tables = torch.from_numpy(self.block_tables_host).to(self.device)
        self.context_lens_host = wl.context_lens.astype(np.int32)
        self.context_lens = torch.from_numpy(self.context_lens_host).to(self.device)
        # Schedule the longest sequences first, so they do not finish last. Samples
        # that share a prompt's blocks stay in fork order instead: scheduled side
        # by side they read the shared blocks while those are still in L2.
        if wl.kind == "shared_prefix":
            self.seq_order_host = np.arange(wl.num_seqs, dtype=np.int32)
        else:
            self.seq_order_host = L.pa_longest_first_order(self.context_lens_host)
        self.seq_order = torch.from_numpy(self.seq_order_host).to(self.device)
        self.q_host = gen.query_bits(wl.seed, wl.num_seqs, wl.num_q_heads, wl.head_dim, wl.dtype)
        self.q = _to_dev(self.q_host, wl.dtype, self.device)
        self.out = torch.empty_like(self.q)
        self.workspace = L.decode_workspace(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                            wl.head_dim, wl.max_context_len,
                                            self.partition_tokens, self.device)
        # Samples forked from one prompt hold its full blocks in common: the step
        # decodes them through pa_paged_decode_cascade, which reads each shared
        # block once per group of samples (8 / G samples stacked per KV head).
        self.groups = None
        self.cascade_ws = None
        self.cascade_order = None
        g = wl.num_q_heads // wl.num_kv_heads
        if wl.kind == "shared_prefix" and not duplicate and g <= 4:
            groups = self.bm.prefix_groups(range(wl.num_seqs), 8 // g)
            if groups.num_groups:
                self.groups = groups.to(self.device)
                # own blocks longest first (tokens after each sample's prefix)
                self.cascade_order = torch.from_numpy(
                    L.pa_cascade_order(self.context_lens_host, groups)).to(self.device)
                self.cascade_ws = L.cascade_workspace(
                    wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
                    wl.max_context_len, self.max_blocks, self.groups, self.device)
        torch.cuda.synchronize(self.device)

    # -- set-up -----------------------------------------------------------------
    def _write(self, k_bits, v_bits, slots):
        if len(slots) == 0:
            return
        k = _to_dev(k_bits, self.wl.dtype, self.device)
        v = _to_dev(v_bits, self.wl.dtype, self.device)
        s = torch.from_numpy(np.asarray(slots, np.int64)).to(self.device)
        L.pa_reshape_and_cache(k, v, self.k_cache, self.v_cache, s, self.dev_error)

    def _setup_decode(self):
        wl = self.wl
        ctx = wl.context_lens.astype(np.int64)
        step_k, step_v = [], []
        chunk = 16
        for first in range(0, wl.num_seqs, chunk):
            seqs = list(range(first, min(wl.num_seqs, first + chunk)))
            kvs = gen.many_seq_kv_bits(wl.seed, seqs, ctx[seqs], wl.num_kv_heads, wl.head_dim,
                                       wl.dtype)
            for s, (kb, vb) in zip(seqs, kvs):
                n = int(ctx[s]) - 1
                slots = self.bm.add_seq(s, n)
                self._write(kb[:n], vb[:n], slots)
                self.prefill_slots.append(slots)
                step_k.append(kb[n])
                step_v.append(vb[n])
        slots = []
        for s in range(wl.num_seqs):
            sl, pairs = self.bm.append_slots(s, 1)
            assert len(pairs) == 0
            slots.append(sl)
        self.step_slots_host = np.concatenate(slots).astype(np.int64)
        self.cow_pairs = np.zeros((0, 2), np.int64)
        self.step_k_host = np.stack(step_k)
        self.step_v_host = np.stack(step_v)
        self._finish_step_inputs()

    def _setup_shared(self):
        wl = self.wl
        S, P, Lp = wl.samples, wl.num_prompts, wl.prompt_len
        prompts = gen.many_seq_kv_bits(wl.seed, range(P), [Lp] * P, wl.num_kv_heads, wl.head_dim,
                                       wl.dtype)
        for p in range(P):
            owners = [p * S + i for i in range(S)] if self.duplicate else [p * S]
            for seq in owners:
                slots = self.bm.add_seq(seq, Lp)
                self._write(prompts[p][0], prompts[p][1], slots)
                self.prefill_slots.append(slots)
            if not self.duplicate:
                for i in range(1, S):
                    self.bm.fork(p * S, p * S + i)
        slots, pairs, ks, vs = [], [], [], []
        for seq in range(P * S):
            n = int(wl.own_lens[seq])
            if n == 0:
                continue
            sl, cow = self.bm.append_slots(seq, n)
            k, v = gen.own_token_kv_bits(wl.seed, seq, n, wl.num_kv_heads, wl.head_dim, wl.dtype)
            slots.append(sl)
            pairs.append(cow)
            ks.append(k)
            vs.append(v)
        self.step_slots_host = np.concatenate(slots).astype(np.int64) if slots else \
            np.zeros(0, np.int64)
        self.cow_pairs = np.concatenate(pairs).astype(np.int64).reshape(-1, 2) if pairs else \
            np.zeros((0, 2), np.int64)
        shp = (0, wl.num_kv_heads, wl.head_dim)
        self.step_k_host = np.concatenate(ks) if ks else np.zeros(shp, np.uint16)
        self.step_v_host = np.concatenate(vs) if vs else np.zeros(shp, np.uint16)
        self._finish_step_inputs()

    def _finish_step_inputs(self):
        self.step_k = _to_dev(self.step_k_host, self.wl.dtype, self.device)
        self.step_v = _to_dev(self.step_v_host, self.wl.dtype, self.device)
        self.step_slots = torch.from_numpy(self.step_slots_host).to(self.device)

    # -- the step ---------------------------------------------------------------
    def copy_blocks(self):
        if len(self.cow_pairs):
            L.pa_copy_blocks(self.k_cache, self.v_cache, self.cow_pairs)

    def reshape_and_cache(self):
        if len(self.step_slots_host):
            L.pa_reshape_and_cache(self.step_k, self.step_v, self.k_cache, self.v_cache,
                                   self.step_slots, self.dev_error)

    def decode(self, out=None, partition_tokens=None, ordered=True):
        out = self.out if out is None else out
        pt = self.partition_tokens if partition_tokens is None else partition_tokens
        ws = self.workspace
        if pt != self.partition_tokens:
            ws = L.decode_workspace(self.wl.num_seqs, self.wl.num_q_heads, self.wl.num_kv_heads,
                                    self.wl.head_dim, self.wl.max_context_len, pt, self.device)
        L.pa_paged_decode(out, self.q, self.k_cache, self.v_cache, self.block_tables,
                          self.context_lens, self.wl.max_context_len, self.wl.scale, pt, ws,
                          self.dev_error, seq_order=self.seq_order if ordered else None)
        return out

    def decode_cascade(self, out=None):
        """The decode through pa_paged_decode_cascade (batches with groups only)."""
        out = self.out if out is None else out
        L.pa_paged_decode_cascade(out, self.q, self.k_cache, self.v_cache, self.block_tables,
                                  self.context_lens, self.wl.max_context_len, self.wl.scale,
                                  self.groups, self.cascade_ws, self.dev_error,
                                  seq_order=self.cascade_order)
        return out

    def decode_step(self, out=None):
        """The step's decode: the cascade when sequences share blocks, else plain."""
        if self.groups is not None:
            return self.decode_cascade(out)
        return self.decode(out)

    def step(self):
        """One decode step: copy-on-write copies, cache writes, decode attention."""
        self.copy_blocks()
        self.reshape_and_cache()
        return self.decode_step()

    def decode_launches(self) -> int:
        """Kernel launches of the step's decode call."""
        wl = self.wl
        if self.groups is not None:
            # prepare, both decodes in one launch (8 stacked query heads per KV
            # head; else two launches), merge
            return L.pa_paged_decode_cascade_plan(
                wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.max_context_len,
                self.max_blocks, self.groups.num_groups, self.groups.group_size,
                self.groups.max_prefix_blocks, dtype=wl.dtype)["launches"]
        _, _, n = L.pa_paged_decode_plan(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads,
                                         wl.head_dim, wl.max_context_len,
                                         self.partition_tokens or 0, ordered=True)
        return n

    def launches_per_step(self) -> int:
        decode = self.decode_launches()
        return int(len(self.cow_pairs) > 0) * -(-len(self.cow_pairs) // 1024) + \
            int(len(self.step_slots_host) > 0) + decode

    def error_bits(self) -> int:
        return int(self.dev_error.item())


class HostStep:
    """One step fed from pinned host memory and read back to the host.

    The step's inputs (queries, new keys/values, slot mapping, block tables,
    context lengths, scheduling order) live back to back in one pinned host buffer and one device
    buffer; the runner's input tensors are views of the device buffer. Every
    call copies the whole input buffer host -> device, runs the step's kernels,
    and copies the attention output device -> host, all on the current stream.
    """

    def __init__(self, runner: DecodeRunner):
        r = self.r = runner
        srcs = [("q", r.q), ("step_k", r.step_k), ("step_v", r.step_v),
                ("step_slots", r.step_slots), ("block_tables", r.block_tables),
                ("context_lens", r.context_lens), ("seq_order", r.seq_order)]
        offs, total = [], 0
        for _, t in srcs:
            offs.append(total)
            total += -(-t.numel() * t.element_size() // 256) * 256
        self.h_buf = torch.empty(total, dtype=torch.uint8).pin_memory()
        self.d_buf = torch.empty(total, dtype=torch.uint8, device=r.device)
        for (name, t), off in zip(srcs, offs):
            n = t.numel() * t.element_size()
            dview = self.d_buf[off:off + n].view(t.dtype).view(t.shape)
            hview = self.h_buf[off:off + n].view(t.dtype).view(t.shape)
            hview.copy_(t.cpu())
            dview.copy_(t)
            setattr(r, name, dview)
        self.h_out = torch.empty(r.out.shape, dtype=r.dtype).pin_memory()
        self.h2d_bytes = total
        self.d2h_bytes = self.h_out.numel() * self.h_out.element_size()
        torch.cuda.synchronize(r.device)

    def __call__(self):
        r = self.r
        self.d_buf.copy_(self.h_buf, non_blocking=True)
        r.step()
        self.h_out.copy_(r.out, non_blocking=True)
        return self.h_out


class HostPipeline:
    """Steps fed from pinned host memory with the copies overlapped.

    Two slots each hold a step's inputs (pinned host and device copies) and its
    output. Step k uses slot k % 2: an upload stream copies the slot's inputs
    host -> device, the current stream waits for them and runs the step's
    kernels into the slot's output, and a download stream copies that output
    device -> host. Step k + 1's upload thus runs while step k computes, and
    step k's download while step k + 1 computes. Every step still moves all of
    its inputs and its output across the host link; a slot is reused only after
    its previous output has reached the host.
    """

    FIELDS = ("q", "step_k", "step_v", "step_slots", "block_tables", "context_lens", "seq_order")

    def __init__(self, runner: DecodeRunner):
        r = self.r = runner
        self.compute = torch.cuda.current_stream(r.device)
        self.upload = torch.cuda.Stream(r.device)
        self.download = torch.cuda.Stream(r.device)
        self.slots = []
        for _ in range(2):
            offs, total = [], 0
            for name in self.FIELDS:
                t = getattr(r, name)
                offs.append(total)
                total += -(-t.numel() * t.element_size() // 256) * 256
            h_buf = torch.empty(total, dtype=torch.uint8).pin_memory()
            d_buf = torch.empty(total, dtype=torch.uint8, device=r.device)
            views = {}
            for name, off in zip(self.FIELDS, offs):
                t = getattr(r, name)
                n = t.numel() * t.element_size()
                h_buf[off:off + n].view(t.dtype).view(t.shape).copy_(t.cpu())
                views[name] = d_buf[off:off + n].view(t.dtype).view(t.shape)
            self.slots.append({
                "h_buf": h_buf, "d_buf": d_buf, "views": views,
                "out": torch.empty_like(r.out),
                "h_out": torch.empty(r.out.shape, dtype=r.dtype).pin_memory(),
                "in_ready": torch.cuda.Event(), "out_ready": torch.cuda.Event(),
                "free": torch.cuda.Event(),
            })
            self.h2d_bytes = total
        self.d2h_bytes = self.slots[0]["h_out"].numel() * self.slots[0]["h_out"].element_size()
        for sl in self.slots:
            sl["free"].record(self.download)
        self.k = 0
        torch.cuda.synchronize(r.device)

    def __call__(self):
        r = self.r
        sl = self.slots[self.k % 2]
        self.k += 1
        with torch.cuda.stream(self.upload):
            self.upload.wait_event(sl["free"])
            sl["d_buf"].copy_(sl["h_buf"], non_blocking=True)
            sl["in_ready"].record(self.upload)
        self.compute.wait_event(sl["in_ready"])
        for name, v in sl["views"].items():
            setattr(r, name, v)
        r.copy_blocks()
        r.reshape_and_cache()
        r.decode_step(out=sl["out"])
        sl["out_ready"].record(self.compute)
        with torch.cuda.stream(self.download):
            self.download.wait_event(sl["out_ready"])
            sl["h_out"].copy_(sl["out"], non_blocking=True)
            sl["free"].record(self.download)
        return sl["h_out"]
