"""Iteration-level (continuous) batching over the paged KV cache, oracle side.

Test infrastructure: only the tests, the smoke check and the benchmark's CPU
baseline may use this module. It shares no code with the CUDA-side library.

What the pages fix:
  * Scheduling works per decoding iteration, not per request: after every step
    the requests that finished leave the batch and waiting requests join the
    next step's batch ("PagedAttention and Continuous Batching", "Batch by step,
    not by request"; "PagedAttention: The vLLM Paper", "Continuous Batching:
    Request-Level vs. Iteration-Level Scheduling", figure: batch {A,B,C}, A
    finishes, D joins, batch {B,C,D}).
  * A request joins when the pool has free blocks for it; nothing contiguous is
    reserved ("Batch by step, not by request").
  * When memory runs short a request is preempted, either by swapping its
    blocks to CPU memory or by dropping them and recomputing them later
    ("PagedAttention: The vLLM Paper", "Implementation Essentials", block manager).
  * Parallel samples of one prompt share the prompt's blocks
    ("Implementation Essentials", prefix sharing).

Readings where the pages are silent (the library's scheduler follows the same
rules so that plans can be compared bit for bit):
  * A request has a prompt of ``prompt_len`` tokens, ``num_samples`` parallel
    samples and generates ``output_len`` tokens per sample, one per step; its
    keys and values are inputs (there is no model). Admission writes the whole
    prompt (sample 0's sequence; the other samples are forks of it).
  * Every step, each running sample appends one token (its slot is written and
    the sample is decoded with the new token in its context). A request that
    has generated ``output_len`` tokens is finished after that step and its
    blocks are freed at the start of the next step.
  * Order of one step: (1) free the requests finished last step; (2) append for
    running requests, oldest admission first; before a request appends, the
    exact number of blocks its samples' appends take is checked, and while the
    pool is short the newest running request is preempted (the request itself
    when it is the newest); (3) only if nothing was preempted in this step,
    resume swapped requests in arrival order; (4) only if nothing was
    preempted and none is swapped, admit waiting requests in arrival order.
    Resumed and admitted requests go to the back of the running list and
    append in the same step. Admission stops at the first request that does not
    fit (no skipping); the number of running sequences never exceeds
    ``max_num_seqs``.
  * Preemption swaps the request's samples out (each sample takes a host copy
    of every block of its own table) when the host pool has room; otherwise a
    one-sample request is dropped for recomputation: it rejoins the waiting
    queue at its arrival position and, when admitted again, its prompt and the
    tokens it has generated are written again. A many-sample request that
    cannot be swapped is an error. In recompute mode there is no host pool
    and every request must have one sample.
  * Arrival order is (arrival step, submission order).
  * A request submitted with its prompt's token ids is admitted through the
    block manager's prefix cache (``add_seq_cached``): the leading full prompt
    blocks found cached are shared and only the rest of the prompt is written.
    Its admission need subtracts the blocks found and adds back those of them
    that no sequence holds (they are counted as free). A recomputed request
    re-registers its prompt the same way and then appends its generated tokens.
  * The device executes a step in this order: swap-out pairs, swap-in pairs,
    prefill writes (the prompts, and recomputed tokens, of admitted requests),
    copy-on-write pairs, new-token writes, then decode. Prefill comes before
    the copies because a many-sample request admitted in this step copies its
    own partly filled prompt block on its first append; the new tokens come
    after them because the last holder of a shared block writes into it in place.

Sequence id of sample ``s`` of request ``r``: ``r * MAX_SAMPLES + s``.
"""

from dataclasses import dataclass, field

from oracle.block_manager import BlockManager, BlockManagerError, ERR_INVALID_ARG, \
    ERR_NO_FREE_BLOCKS

MAX_SAMPLES = 64
PREEMPT_SWAP = 0
PREEMPT_RECOMPUTE = 1


def seq_id(request: int, sample: int) -> int:
    return request * MAX_SAMPLES + sample


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


@dataclass
class Request:
    rid: int
    prompt_len: int
    output_len: int
    num_samples: int
    arrival: int
    order: int
    generated: int = 0
    state: str = "pending"      # pending, waiting, running, swapped, finished
    tokens: tuple = None        # prompt token ids (admission through the prefix cache)


@dataclass
class Plan:
    step: int
    finished: list = field(default_factory=list)
    preempted: list = field(default_factory=list)       # (request, 0 swap / 1 recompute)
    resumed: list = field(default_factory=list)
    admitted: list = field(default_factory=list)
    swap_out: list = field(default_factory=list)        # (device block, host block)
    swap_in: list = field(default_factory=list)         # (host block, device block)
    prefill: list = field(default_factory=list)         # (request, sample, position, slot)
    copies: list = field(default_factory=list)          # (src block, dst block)
    writes: list = field(default_factory=list)          # (request, sample, position, slot)
    batch: list = field(default_factory=list)           # (request, sample, context_len)
    cached: int = 0                                     # prompt tokens found in the prefix cache


class Scheduler:
    def __init__(self, num_blocks: int, block_size: int, initial_free_order=None,
                 max_num_seqs: int = 256, num_host_blocks: int = 0,
                 preempt_mode: int = PREEMPT_SWAP):
        if max_num_seqs <= 0 or preempt_mode not in (PREEMPT_SWAP, PREEMPT_RECOMPUTE):
            raise BlockManagerError(ERR_INVALID_ARG, "bad scheduler arguments")
        if preempt_mode == PREEMPT_RECOMPUTE and num_host_blocks:
            raise BlockManagerError(ERR_INVALID_ARG, "recompute mode takes no host pool")
        self.bm = BlockManager(num_blocks, block_size, initial_free_order)
        if num_host_blocks:
            self.bm.set_host_pool(num_host_blocks)
        self.block_size = block_size
        self.max_num_seqs = max_num_seqs
        self.mode = preempt_mode
        self.requests: dict[int, Request] = {}
        self.pending: list[Request] = []     # submitted, not yet arrived
        self.waiting: list[Request] = []
        self.running: list[Request] = []
        self.swapped: list[Request] = []
        self.finishing: list[Request] = []
        self.step_index = 0
        self._submitted = 0

    # -- requests ---------------------------------------------------------
    def submit(self, rid: int, prompt_len: int, output_len: int, num_samples: int = 1,
               arrival: int = 0, tokens=None) -> None:
        if rid in self.requests or rid < 0:
            raise BlockManagerError(ERR_INVALID_ARG, "bad or duplicate request id")
        if prompt_len < 1 or output_len < 1 or not 1 <= num_samples <= MAX_SAMPLES:
            raise BlockManagerError(ERR_INVALID_ARG, "bad request sizes")
        if self.mode == PREEMPT_RECOMPUTE and num_samples != 1:
            raise BlockManagerError(ERR_INVALID_ARG, "recompute mode needs one sample")
        worst = num_samples * _ceil_div(prompt_len + output_len, self.block_size)
        if num_samples > self.max_num_seqs or worst > self.bm.num_blocks:
            raise BlockManagerError(ERR_NO_FREE_BLOCKS, "request can never fit")
        if tokens is not None and len(tokens) != prompt_len:
            raise BlockManagerError(ERR_INVALID_ARG, "one token id per prompt position")
        r = Request(rid, prompt_len, output_len, num_samples, arrival, self._submitted,
                    tokens=None if tokens is None else tuple(int(t) for t in tokens))
        self._submitted += 1
        self.requests[rid] = r
        self.pending.append(r)

    def _running_seqs(self) -> int:
        return sum(r.num_samples for r in self.running)

    @staticmethod
    def _insert_by_arrival(queue: list, r: Request) -> None:
        key = (r.arrival, r.order)
        i = 0
        while i < len(queue) and (queue[i].arrival, queue[i].order) < key:
            i += 1
        queue.insert(i, r)

    # -- block needs ------------------------------------------------------
    def _append_need(self, r: Request) -> int:
        """Blocks that appending one token to every sample takes, in sample
        order, with copy-on-write on shared partly filled last blocks."""
        need, taken = 0, {}
        for s in range(r.num_samples):
            sid = seq_id(r.rid, s)
            length = self.bm.seq_len(sid)
            if length % self.block_size == 0:
                need += 1
                continue
            last = self.bm.table(sid)[-1]
            if self.bm.refcount(last) - taken.get(last, 0) > 1:
                need += 1
                taken[last] = taken.get(last, 0) + 1
        return need

    def _resume_need(self, r: Request) -> int:
        need = 0
        for s in range(r.num_samples):
            sid = seq_id(r.rid, s)
            length = self.bm.seq_len(sid)
            need += len(self.bm.host_table(sid)) + (1 if length % self.block_size == 0 else 0)
        return need

    def _admit_need(self, r: Request) -> int:
        length = r.prompt_len + r.generated
        extra = r.num_samples if length % self.block_size == 0 else r.num_samples - 1
        hits = revived = 0
        if r.tokens is not None:
            hits, revived = self.bm.cached_prefix(r.tokens)
        return _ceil_div(length, self.block_size) - hits + revived + extra

    # -- one iteration ----------------------------------------------------
    def _append(self, r: Request, plan: Plan) -> None:
        for s in range(r.num_samples):
            sid = seq_id(r.rid, s)
            pos = self.bm.seq_len(sid)
            slots, pairs = self.bm.append_slots(sid, 1)
            plan.copies.extend(pairs)
            plan.writes.append((r.rid, s, pos, slots[0]))

    def _preempt(self, r: Request, plan: Plan) -> None:
        host_need = sum(len(self.bm.table(seq_id(r.rid, s))) for s in range(r.num_samples))
        if self.mode == PREEMPT_SWAP and host_need <= self.bm.num_free_host():
            for s in range(r.num_samples):
                plan.swap_out.extend(self.bm.swap_out(seq_id(r.rid, s)))
            r.state = "swapped"
            self._insert_by_arrival(self.swapped, r)
            plan.preempted.append((r.rid, PREEMPT_SWAP))
        elif r.num_samples == 1:
            self.bm.free_seq(seq_id(r.rid, 0))
            r.state = "waiting"
            self._insert_by_arrival(self.waiting, r)
            plan.preempted.append((r.rid, PREEMPT_RECOMPUTE))
        else:
            raise BlockManagerError(ERR_NO_FREE_BLOCKS, "host pool cannot take the request")

    def step(self) -> Plan:
        t = self.step_index
        plan = Plan(step=t)
        # arrivals
        still = []
        for r in self.pending:
            if r.arrival <= t:
                r.state = "waiting"
                self._insert_by_arrival(self.waiting, r)
            else:
                still.append(r)
        self.pending = still
        # (1) free the requests finished last step
        for r in self.finishing:
            for s in range(r.num_samples):
                self.bm.free_seq(seq_id(r.rid, s))
            plan.finished.append(r.rid)
        self.finishing = []
        # (2) running requests append, oldest first; preempt the newest when short
        i = 0
        while i < len(self.running):
            r = self.running[i]
            need = self._append_need(r)
            while need > self.bm.num_free() and self.running[-1] is not r:
                self._preempt(self.running.pop(), plan)
            if need > self.bm.num_free():
                self.running.pop()
                self._preempt(r, plan)
                break
            self._append(r, plan)
            i += 1
        if not plan.preempted:
            # (3) resume swapped requests in arrival order
            while self.swapped:
                r = self.swapped[0]
                if self._running_seqs() + r.num_samples > self.max_num_seqs:
                    break
                if self._resume_need(r) > self.bm.num_free():
                    break
                self.swapped.pop(0)
                for s in range(r.num_samples):
                    plan.swap_in.extend(self.bm.swap_in(seq_id(r.rid, s)))
                r.state = "running"
                self.running.append(r)
                plan.resumed.append(r.rid)
                self._append(r, plan)
            # (4) admit waiting requests in arrival order
            while not self.swapped and self.waiting:
                r = self.waiting[0]
                if self._running_seqs() + r.num_samples > self.max_num_seqs:
                    break
                if self._admit_need(r) > self.bm.num_free():
                    break
                self.waiting.pop(0)
                length = r.prompt_len + r.generated
                if r.tokens is None:
                    slots = self.bm.add_seq(seq_id(r.rid, 0), length)
                    plan.prefill.extend((r.rid, 0, p, slots[p]) for p in range(length))
                else:
                    slots, cached = self.bm.add_seq_cached(seq_id(r.rid, 0), r.tokens)
                    plan.cached += cached
                    plan.prefill.extend((r.rid, 0, p, slots[p])
                                        for p in range(cached, r.prompt_len))
                    if r.generated:
                        gslots, _ = self.bm.append_slots(seq_id(r.rid, 0), r.generated)
                        plan.prefill.extend((r.rid, 0, r.prompt_len + i, gslots[i])
                                            for i in range(r.generated))
                for s in range(1, r.num_samples):
                    self.bm.fork(seq_id(r.rid, 0), seq_id(r.rid, s))
                r.state = "running"
                self.running.append(r)
                plan.admitted.append(r.rid)
                self._append(r, plan)
        # decode batch; requests reaching their output length finish
        for r in self.running:
            for s in range(r.num_samples):
                plan.batch.append((r.rid, s, self.bm.seq_len(seq_id(r.rid, s))))
            r.generated += 1
        done = [r for r in self.running if r.generated == r.output_len]
        for r in done:
            r.state = "finished"
        self.running = [r for r in self.running if r.generated < r.output_len]
        self.finishing = done
        self.step_index += 1
        return plan

    # -- queries ----------------------------------------------------------
    def idle(self) -> bool:
        return not (self.pending or self.waiting or self.running or self.swapped
                    or self.finishing)

    def batch_seq_ids(self, plan: Plan) -> list:
        return [seq_id(r, s) for r, s, _ in plan.batch]

    def kv_usage(self):
        """(filled slots, allocated slots) over the device blocks that resident
        sequences hold (running ones and those finished in the last step); a block shared by several sequences counts once, with
        the fill of its fullest holder."""
        fill = {}
        for r in self.running + self.finishing:
            for s in range(r.num_samples):
                sid = seq_id(r.rid, s)
                length = self.bm.seq_len(sid)
                for i, b in enumerate(self.bm.table(sid)):
                    f = min(self.block_size, length - i * self.block_size)
                    fill[b] = max(fill.get(b, 0), f)
        return sum(fill.values()), len(fill) * self.block_size
