"""Benchmark of the paged-decode step on B200.

One step = the whole decode-step path of one attention layer for a batch:
copy-on-write block copies (when the workload has any), writing each new
token's K/V into its slot, and paged decode attention with the split-KV merge.
The default (headline) workload is the largest single-GPU batch: long-context
split-KV decode (8 sequences, contexts U[32768, 131072], 64 query / 8 KV heads,
head_dim 128, bf16, 512-token split-KV partitions, one new token per sequence).
Every other workload (tiny MHA, 7B-like MHA, GQA 32/8, prompts forked into
samples sharing blocks) is timed at full size with the same protocol in the
line's ``per_config`` object.

Metric: KV-read GB/s (algorithmic bytes of the step / device time of the
step; % of measured HBM peak alongside) and decode tokens/s.

Timing: W untimed warm-up steps; then K steps, each bracketed by one pair of
CUDA events on the launching stream, and K decodes alone the same way (the
roofline); a barrier + synchronize on both sides of the timed region; max over
ranks. Every 32 steps a GPU spin (outside the events) keeps
the stream busy while the host enqueues them, so the steps run back to back
and the events measure device time rather than host issue gaps. Workloads whose inputs exceed 4x the 126 MB L2 run
without a flush (a cyclic scan larger than the cache reuses nothing); smaller
ones flush L2 between steps, outside the events, by reading a 256 MiB buffer
(a write flush would leave dirty lines whose write-back the next kernel pays).
The decode kernel alone is timed the same way for the roofline. ``e2e``
repeats the step through the same C interface fed from pinned host buffers:
every step copies its inputs host -> device and its output device -> host
inside the timed region; the next step's input copy overlaps this step's
kernels (two buffer slots, an upload and a download stream).

Multi-GPU (torchrun, one process per GPU): the decode step has no exchange
between GPUs, so each rank runs an independent replica with its own pool and
its own seeded batch (weak scaling); timing is the max over ranks.

``--impl reference`` times the CPU oracle (float64 NumPy) on a bounded sample
of the same workload on the host cores; only rank 0 does work.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged-decode KV-read GB/s (% of B200 HBM peak); decode tokens/s"
UNIT = "GB/s"
DEFAULT_WORKLOAD = "long_ctx_split_kv"
# every other workload is timed at full size in the line's per_config object
PER_CONFIG = ("tiny_mha_d64", "mha_7b_fp16", "gqa_32_8_bf16", "prefix_share_cow",
              "long_ctx_split_kv")
# head shape of the serving-loop, prefix-cache and batching measurements
LOOP_SHAPE = "mha_7b_fp16"
L2_FLUSH_BYTES = 256 << 20


# --------------------------------------------------------------------------
# byte accounting
# --------------------------------------------------------------------------

def decode_bytes(wl) -> int:
    """Algorithmic bytes of one paged-decode call: each token's K and V once per KV
    head, q read and out written once, the used block-table entries and the
    context lengths."""
    ctx = wl.context_lens.astype(np.int64)
    e = wl.elem_bytes
    kv = int(ctx.sum()) * wl.num_kv_heads * wl.head_dim * e * 2
    qo = 2 * wl.num_seqs * wl.num_q_heads * wl.head_dim * e
    tables = 4 * int(((ctx + wl.block_size - 1) // wl.block_size).sum())
    return kv + qo + tables + 4 * wl.num_seqs


def unique_decode_bytes(wl, runner) -> int:
    """For workloads whose sequences share blocks: K/V bytes of distinct physical
    blocks read (whole used blocks), plus q/out/tables as above."""
    used = set()
    ctx = wl.context_lens.astype(np.int64)
    for s in range(wl.num_seqs):
        n = int((ctx[s] + wl.block_size - 1) // wl.block_size)
        used.update(runner.block_tables_host[s, :n].tolist())
    e = wl.elem_bytes
    kv = len(used) * wl.block_size * wl.num_kv_heads * wl.head_dim * e * 2
    return kv + decode_bytes(wl) - int(ctx.sum()) * wl.num_kv_heads * wl.head_dim * e * 2


def step_bytes(wl, runner) -> int:
    """Algorithmic bytes of one step: decode + new-token writes + block copies."""
    row = wl.num_kv_heads * wl.head_dim * wl.elem_bytes
    t = len(runner.step_slots_host)
    writes = t * (2 * row * 2 + 8)           # read key+value rows, write them, read slot
    blk = wl.block_size * row
    copies = len(runner.cow_pairs) * 2 * blk * 2   # K and V blocks, read + write
    return decode_bytes(wl) + writes + copies


# --------------------------------------------------------------------------
# clocks
# --------------------------------------------------------------------------

_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


_NVML_POLL = r"""
import sys, time, pynvml
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByPciBusId(sys.argv[1]) if sys.argv[1] else \
    pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[2]))
print("max", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
while True:
    try:
        print(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
              pynvml.nvmlDeviceGetCurrentClocksEventReasons(h), flush=True)
    except pynvml.NVMLError:
        pass
    time.sleep(0.005)
"""


class ClockSampler:
    """SM clock and clock-event reasons sampled every 5 ms through NVML (read-only)
    by a separate process, so the sampling does not compete with the launching
    thread; falls back to ``nvidia-smi -lms 100`` without NVML."""

    def __init__(self, torch_device):
        self.dev = torch_device
        self.samples = []
        self.proc = None
        self.thread = None
        self.max_mhz = None
        self.ready = threading.Event()

    def _bus_id(self):
        import torch
        try:
            p = torch.cuda.get_device_properties(self.dev)
            return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        except Exception:
            return ""

    def __enter__(self):
        try:
            import pynvml  # noqa: F401
            cmd = [sys.executable, "-c", _NVML_POLL, self._bus_id(), str(self.dev.index or 0)]
            kind = "nvml"
        except ImportError:
            cmd = ["nvidia-smi", "-i", str(self.dev.index or 0),
                   "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                   "--format=csv,noheader,nounits", "-lms", "100"]
            kind = "smi"
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.thread = threading.Thread(target=self._read, args=(kind,), daemon=True)
            self.thread.start()
            self.ready.wait(timeout=20)   # the poller has started sampling
        except (OSError, ValueError):
            self.proc = None
        return self

    def _read(self, kind):
        for line in self.proc.stdout:
            try:
                if kind == "nvml":
                    parts = line.split()
                    if parts[0] == "max":
                        self.max_mhz = float(parts[1])
                        continue
                    self.samples.append((float(parts[0]), int(parts[1])))
                else:
                    parts = [p.strip() for p in line.split(",")]
                    self.max_mhz = float(parts[1])
                    bits = int(parts[2], 16) if parts[2].startswith("0x") else int(parts[2])
                    self.samples.append((float(parts[0]), bits))
                self.ready.set()
            except (ValueError, IndexError):
                continue

    def __exit__(self, *exc):
        time.sleep(0.02)  # one more sample after the region
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        sm = [m for m, _ in self.samples]
        reasons = set()
        for _, bits in self.samples:
            for b, name in _REASONS.items():
                if bits & b and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------
# helpers
# --------------------------------------------------------------------------

def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


DECODE_SOURCES = ("paged_decode_impl.cuh", "decode_policies.cuh", "decode_common.cuh",
                  "decode_merge.cuh", "pa_device.cuh", "pa_internal.h")
# a cascade figure (":cascade" entries) also depends on the cascade's own kernels
# and its partition layout, an 8-bit figure (":fp8" entries) on the E4M3
# policies, an 8-bit cascade figure (":cascade:fp8") on both
CASCADE_SOURCES = DECODE_SOURCES + ("cascade.cu", "pa_api.cu")
FP8_SOURCES = DECODE_SOURCES + ("decode_policy_fp8.cuh",)
CASCADE_FP8_SOURCES = CASCADE_SOURCES + ("decode_policy_fp8.cuh",)


def decode_source_sha(sources=DECODE_SOURCES) -> str:
    """Hash of the decode kernel's sources (ties a traffic figure to the code profiled)."""
    h = hashlib.sha256()
    for name in sources:
        with open(os.path.join(ROOT, "paged_kv_cache_352_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic_for(workload: str):
    """DRAM bytes per decode call from the committed ncu summary, if it was taken
    on the current kernel sources for this workload (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(workload)
        sha = decode_source_sha(CASCADE_SOURCES if workload.endswith(":cascade")
                                else CASCADE_FP8_SOURCES if workload.endswith(":cascade:fp8")
                                else FP8_SOURCES if workload.endswith(":fp8")
                                else DECODE_SOURCES)
    except (OSError, ValueError, AttributeError):
        return None
    if not rec or rec.get("source_sha") != sha:
        return None
    return rec.get("dram_bytes_per_launch")


def read_stream_gbs(device, nbytes: int = 2 << 30, reps: int = 5):
    """A read-only streaming reference: summing a 2 GiB int64 buffer (torch)."""
    import torch
    x = torch.ones(nbytes // 8, dtype=torch.int64, device=device)
    x.sum()
    torch.cuda.synchronize(device)
    best = None
    for _ in range(reps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        x.sum()
        b.record()
        torch.cuda.synchronize(device)
        t = a.elapsed_time(b) / 1e3
        best = t if best is None else min(best, t)
    del x
    torch.cuda.empty_cache()
    return nbytes / best / 1e9


def _rank_info():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def _max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_workload(name: str, rank: int, num_seqs: int = 0, num_blocks: int = 0):
    """The named workload; rank r > 0 gets an independent batch (seed shifted).

    ``num_seqs``/``num_blocks`` (profiling only) keep the first sequences of the
    batch in a smaller pool; the workload name then says so."""
    import workloads
    from workloads import configs
    if rank == 0:
        wl = workloads.workload(name)
    else:
        base = workloads.workload(name)
        wl = configs.WORKLOADS[name](seed=base.seed + 7919 * rank)
    if num_seqs or num_blocks:
        wl = configs.truncated(wl, num_seqs or wl.num_seqs, num_blocks or wl.num_blocks)
    return wl


# --------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and --impl reference)
# --------------------------------------------------------------------------

def _host_cpus() -> int:
    """CPUs this process may run on (the oracle's BLAS pool is sized from them)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover - non-Linux
        return os.cpu_count() or 1


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()
             if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def time_oracle(wl, budget_s: float = 15.0, max_seq: int | None = None, chunks=None,
                setup_budget_s: float = 20.0):
    """Times the oracle's paged decode on the first sequences of the workload.

    Grows the sample one sequence at a time (in chunks of 1, 2, 4, 8) until
    ``budget_s`` of oracle time is used, or until building the sample's pools has
    taken ``setup_budget_s`` (long contexts); a batch that ends first is decoded
    again, pass after pass, until the budget is spent. ``chunks`` (from an earlier
    call) reuses a built sample instead. Returns (GB/s, tokens/s, description,
    oracle seconds, chunks)."""
    from oracle.attention import paged_decode
    import time as _t
    total_t, total_b, total_seq, total_tok = 0.0, 0, 0, 0
    limit = wl.num_seqs if max_seq is None else min(max_seq, wl.num_seqs)

    def run(sub, st):
        nonlocal total_t, total_b, total_seq, total_tok
        t0 = _t.perf_counter()
        paged_decode(st.q, st.k_cache, st.v_cache, st.block_tables, sub.context_lens, sub.scale,
                     sub.dtype, sub.block_size)
        total_t += _t.perf_counter() - t0
        total_b += decode_bytes(sub)
        total_seq += sub.num_seqs
        total_tok += int(sub.context_lens.sum())

    passes = 1
    if chunks is None:
        chunks = []
        first, chunk, setup_t = 0, 1, 0.0
        while first < limit and (total_seq == 0 or (total_t < budget_s and
                                                    setup_t < setup_budget_s)):
            n = min(chunk, limit - first)
            t0 = _t.perf_counter()
            chunks.append(oracle_sample_setup_range(wl, first, n))
            setup_t += _t.perf_counter() - t0
            run(*chunks[-1])
            first += n
            chunk = min(8, chunk * 2)
    else:
        passes = 0
    unique = sum(sub.num_seqs for sub, _ in chunks)
    while total_t < budget_s and passes < 100000:
        passes += 1
        for c in chunks:
            run(*c)
            if total_t >= budget_s:
                break
    desc = (f"oracle paged_decode (fp64 NumPy) on {unique} of {wl.num_seqs} sequences, "
            f"{total_seq} sequence decodes in {passes} pass(es) ({total_tok} context tokens, "
            f"all {wl.num_q_heads} query heads), {total_t:.1f} s of oracle time")
    return total_b / total_t / 1e9, total_seq / total_t, desc, total_t, chunks


def time_oracle_one_thread(wl, budget_s: float = 5.0, chunks=None):
    """The same oracle sample timing with the BLAS pool limited to one thread,
    so the multi-core figure can be read per core. None without threadpoolctl."""
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:
        return None
    with threadpool_limits(limits=1):
        v, tps, desc, _, _ = time_oracle(wl, budget_s=budget_s, chunks=chunks)
    return {"value": round(v, 4), "unit": UNIT, "cores": 1, "sample": desc,
            "decode_tokens_per_s": round(tps, 3)}


def oracle_sample_setup_range(wl, first: int, n: int):
    from oracle import step as OS
    from workloads.configs import DecodeWorkload
    ctx = wl.context_lens[first:first + n]
    nb = int(sum(-(-int(c) // wl.block_size) for c in ctx)) + 1
    sub = DecodeWorkload(f"{wl.name}[{first}:{first + n}]", wl.seed + first, n, wl.num_q_heads,
                         wl.num_kv_heads, wl.head_dim, wl.dtype, ctx, nb,
                         np.random.default_rng([wl.seed, 5, first]).permutation(nb))
    return sub, OS.decode_step(sub, compute_out=False)


# --------------------------------------------------------------------------
# arms
# --------------------------------------------------------------------------

def measure_swap(wl, r, device, nblocks: int = 2048, reps: int = 5):
    """Host-link rate of pa_swap_blocks: ``nblocks`` whole blocks (all KV heads,
    K and V) from the workload's pool to a pinned host pool and back, in a
    shuffled order, timed with CUDA events (best of ``reps``)."""
    import torch
    from paged_kv_cache_352_b200 import _lib as L
    nblocks = min(nblocks, wl.num_blocks)
    shape = (nblocks,) + tuple(r.k_cache.shape[1:])
    hk = torch.empty(shape, dtype=r.dtype).pin_memory()
    hv = torch.empty(shape, dtype=r.dtype).pin_memory()
    rng = np.random.default_rng(7)
    src = rng.permutation(wl.num_blocks)[:nblocks]
    out_pairs = np.stack([src, np.arange(nblocks)], 1)
    in_pairs = np.stack([np.arange(nblocks), src], 1)
    nbytes = 2 * r.k_cache[0].numel() * r.k_cache.element_size() * nblocks
    res = {}
    for name, fn in (("d2h", lambda: L.pa_swap_blocks(r.k_cache, r.v_cache, hk, hv, out_pairs)),
                     ("h2d", lambda: L.pa_swap_blocks(hk, hv, r.k_cache, r.v_cache, in_pairs))):
        fn()
        torch.cuda.synchronize(device)
        best = None
        for _ in range(reps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize(device)
            t = a.elapsed_time(b) / 1e3
            best = t if best is None else min(best, t)
        res[name + "_gbs"] = round(nbytes / best / 1e9, 2)
    res.update(blocks=int(nblocks), bytes=int(nbytes), unit="GB/s",
               what="pa_swap_blocks, shuffled whole blocks, device pool <-> pinned host pool")
    return res


def measure_prefix_cache(wl, device, requests: int = 64, prompts: int = 4,
                         prompt_len: int = 1024, own_len: int = 256, reps: int = 5):
    """Prefix caching on a synthetic request trace: ``requests`` requests, each a
    ``prompt_len``-token prompt drawn from ``prompts`` shared system prompts plus
    ``own_len`` tokens of its own, admitted through the block manager's prefix
    cache. Reports the share of prompt tokens found cached, and the device time
    of the one cache-write launch that stores every admitted request's new
    tokens, with the cache (suffixes only) and without it (whole prompts)."""
    import torch
    from paged_kv_cache_352_b200 import _lib as L
    rng = np.random.default_rng(11)
    sys_toks = [rng.integers(0, 32000, prompt_len).tolist() for _ in range(prompts)]
    own = [rng.integers(0, 32000, own_len).tolist() for _ in range(requests)]
    nblk = requests * (-(-(prompt_len + own_len) // 16))
    shape = (nblk, wl.num_kv_heads, 16, wl.head_dim)
    dt = torch.float16 if wl.dtype == "f16" else torch.bfloat16
    kc = torch.zeros(shape, dtype=dt, device=device)
    vc = torch.zeros_like(kc)
    row_bytes = wl.num_kv_heads * wl.head_dim * 2

    def admit(cached_mode):
        bm = L.BlockManager(nblk, 16)
        slots_all, total, hit = [], 0, 0
        for r in range(requests):
            toks = sys_toks[r % prompts] + own[r]
            if cached_mode:
                slots, c = bm.add_seq_cached(r, toks)
            else:
                slots, c = bm.add_seq(r, len(toks)), 0
            slots_all.append(np.asarray(slots[c:], np.int64))
            total += len(toks)
            hit += c
        sl = torch.from_numpy(np.concatenate(slots_all)).to(device)
        kv = torch.randn((sl.numel(), wl.num_kv_heads, wl.head_dim), device=device).to(dt)
        L.pa_reshape_and_cache(kv, kv, kc, vc, sl)             # warm-up
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record()
        for _ in range(reps):
            L.pa_reshape_and_cache(kv, kv, kc, vc, sl)
        ev[1].record()
        torch.cuda.synchronize(device)
        ms = ev[0].elapsed_time(ev[1]) / reps
        return hit, total, sl.numel(), ms

    hit, total, n_c, t_c = admit(True)
    _, _, n_p, t_p = admit(False)
    # bytes moved by one write launch: K and V rows read and written once each
    gbs = lambda n, ms: round(4 * n * row_bytes / (ms * 1e6), 1)
    return {"requests": requests, "prompt_tokens": total, "cached_tokens": hit,
            "hit_rate": round(hit / total, 4),
            "written_tokens_with_cache": n_c, "written_tokens_without_cache": n_p,
            "write_ms_with_cache": round(t_c, 4), "write_ms_without_cache": round(t_p, 4),
            "write_gbs_with_cache": gbs(n_c, t_c), "write_gbs_without_cache": gbs(n_p, t_p),
            "what": f"{requests} requests = one of {prompts} shared {prompt_len}-token prompts "
                    f"+ {own_len} own tokens, admitted through pa_bm_add_seq_cached; "
                    f"one pa_reshape_and_cache launch stores all new tokens"}


def continuous_batching_trace(num_requests: int = 1000, seed: int = 352, rate: float = 1.0):
    """Seeded request trace for the continuous-batching loop: Poisson arrivals
    (``rate`` requests per step; at 1.0 the 8192-block pool binds and requests
    are preempted), lognormal prompt (median 400, clipped to 8..1536)
    and output (median 200, clipped to 4..512) lengths, and 1, 2 or 4 parallel
    samples with probabilities 0.85, 0.10, 0.05."""
    rng = np.random.default_rng(seed)
    arrival = np.floor(np.cumsum(rng.exponential(1 / rate, num_requests))).astype(np.int64)
    prompt = np.clip(np.rint(rng.lognormal(np.log(400), 0.8, num_requests)), 8, 1536)
    output = np.clip(np.rint(rng.lognormal(np.log(200), 0.8, num_requests)), 4, 512)
    samples = rng.choice([1, 2, 4], num_requests, p=[0.85, 0.10, 0.05])
    return [(i, int(prompt[i]), int(output[i]), int(samples[i]), int(arrival[i]))
            for i in range(num_requests)]


def shared_prompt_trace(num_requests: int = 1000, seed: int = 353, systems: int = 8,
                        system_len: int = 512, rate: float = 1.0):
    """Seeded trace whose prompts are one of ``systems`` shared ``system_len``-token
    system prompts followed by a lognormal number (median 128, clipped to
    8..1024) of the request's own tokens, with token ids; outputs and samples as
    ``continuous_batching_trace``."""
    rng = np.random.default_rng(seed)
    sys_prompts = [rng.integers(0, 32000, system_len).tolist() for _ in range(systems)]
    arrival = np.floor(np.cumsum(rng.exponential(1 / rate, num_requests))).astype(np.int64)
    own = np.clip(np.rint(rng.lognormal(np.log(128), 0.8, num_requests)), 8, 1024).astype(int)
    output = np.clip(np.rint(rng.lognormal(np.log(200), 0.8, num_requests)), 4, 512)
    samples = rng.choice([1, 2, 4], num_requests, p=[0.85, 0.10, 0.05])
    trace = []
    for i in range(num_requests):
        toks = sys_prompts[int(rng.integers(systems))] + rng.integers(0, 32000, own[i]).tolist()
        trace.append((i, len(toks), int(output[i]), int(samples[i]), int(arrival[i]), toks))
    return trace


def measure_host_planning(num_requests: int = 1000, num_blocks: int = 8192,
                          max_num_seqs: int = 256, host_blocks: int = 4096):
    """The scheduler's planning alone (block manager, slot mappings, copy-on-write
    pairs, swaps, tables; C++ behind one binding call per step) over the
    continuous-batching trace, host wall time: the host share of each step, which
    the loop overlaps with the GPU's work on the previous plans."""
    from paged_kv_cache_352_b200 import _lib as L
    trace = continuous_batching_trace(num_requests)
    sched = L.Scheduler(num_blocks, 16, np.random.default_rng(7).permutation(num_blocks),
                        max_num_seqs=max_num_seqs, num_host_blocks=host_blocks)
    for t in trace:
        sched.submit(*t[:5])
    steps = slots = 0
    t0 = time.perf_counter()
    while not sched.idle():
        c = sched.step()
        steps += 1
        slots += c.num_seqs + c.num_prefill
    el = time.perf_counter() - t0
    return {"us_per_step": round(el / steps * 1e6, 2), "steps": steps, "slots": slots,
            "slots_per_s": round(slots / el, 1),
            "what": "pa_sched_step alone over the continuous-batching trace (1000 requests): "
                    "admission, appends with copy-on-write, preemption by swap, slot mappings "
                    "and tables; host wall time including the binding"}


def measure_continuous_batching(wl, device, num_requests: int = 1000, num_blocks: int = 8192,
                                max_num_seqs: int = 256, host_blocks: int = 4096,
                                max_model_len: int = 2048, fp8_scales=None, trace=None,
                                use_tokens: bool = False, cascade=None):
    """The iteration-level batching loop end to end on one GPU: the library's
    scheduler plans each step and its executor runs swap-out/in, prefill writes,
    copy-on-write, new-token writes and decode (7B-like heads of ``wl``). Keys,
    values and queries are rows of a random device bank (no model). Reports
    generated tokens per second over the whole trace (CUDA events around the
    loop; host planning included), and KV occupancy sampled every 16 steps next
    to what a contiguous ``max_model_len`` reservation per sequence would give.
    ``fp8_scales = (k_scale, v_scale)`` runs the same trace over E4M3 caches;
    ``trace`` replaces the default trace, and ``use_tokens`` submits its token ids
    so that admission goes through the prefix cache. ``cascade`` sets the
    executor's mode for sequences sharing blocks (PA_SCHED_CASCADE_*; default
    auto)."""
    import torch
    from paged_kv_cache_352_b200 import _lib as L
    trace = continuous_batching_trace(num_requests) if trace is None else trace
    num_requests = len(trace)
    dt = torch.float16 if wl.dtype == "f16" else torch.bfloat16
    hq, hkv, d = wl.num_q_heads, wl.num_kv_heads, wl.head_dim
    sched = L.Scheduler(num_blocks, 16, np.random.default_rng(7).permutation(num_blocks),
                        max_num_seqs=max_num_seqs, num_host_blocks=host_blocks)
    for t in trace:
        sched.submit(*t[:5], tokens=t[5] if use_tokens else None)
    sched.attach(hq, hkv, d, dt, max_model_len, fp8_scales=fp8_scales)
    if cascade is not None:
        sched.set_cascade(cascade)
    cdt = torch.uint8 if fp8_scales else dt
    kc = torch.zeros(num_blocks, hkv, 16, d, dtype=cdt, device=device)
    vc = torch.zeros_like(kc)
    hk = torch.zeros(host_blocks, hkv, 16, d, dtype=cdt).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    bank = torch.randn(num_blocks * 16, hkv, d, device=device).to(dt)
    qbank = torch.randn(max_num_seqs, hq, d, device=device).to(dt)
    out = torch.empty(max_num_seqs, hq, d, dtype=dt, device=device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    scale = 1.0 / math.sqrt(d)
    tot = {"steps": 0, "tokens": 0, "prefill_tokens": 0, "preempt": 0, "swap_blocks": 0,
           "cow": 0, "context": 0, "cached": 0, "cascade_steps": 0, "saved_blocks": 0}
    util, contiguous = [], []
    row_bytes = hkv * d * (1 if fp8_scales else 2)   # cached bytes of one (token, K or V) row
    torch.cuda.synchronize(device)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    a.record()
    while not sched.idle():
        c = sched.step()
        sched.execute(kc, vc, hk, hv, bank, bank, bank, bank, qbank, out, scale, dev_error=err)
        ng, saved = sched.last_cascade()
        tot["cascade_steps"] += ng > 0
        tot["saved_blocks"] += saved
        tot["steps"] += 1
        tot["tokens"] += c.num_seqs
        tot["prefill_tokens"] += c.num_prefill
        tot["preempt"] += c.num_preempted
        tot["swap_blocks"] += c.num_swap_out + c.num_swap_in
        tot["cow"] += c.num_copies
        tot["context"] += c.total_context
        tot["cached"] += c.num_cached_tokens
        if tot["steps"] % 16 == 0 and c.num_seqs:
            filled, alloc = sched.kv_usage()
            util.append(filled / alloc)
            contiguous.append(filled / (c.num_seqs * max_model_len))
    b.record()
    torch.cuda.synchronize(device)
    host_s = time.perf_counter() - t0
    ms = a.elapsed_time(b)
    if int(err.item()):
        raise RuntimeError(f"continuous batching: device error bits {int(err.item())}")
    return {
        "metric": "generated_tokens_per_s", "value": round(tot["tokens"] / (ms / 1e3), 1),
        "unit": "tokens/s", "requests": num_requests, "steps": tot["steps"],
        "ms_per_step": round(ms / tot["steps"], 4),
        "host_ms_per_step": round(1e3 * host_s / tot["steps"], 4),
        "mean_batch": round(tot["tokens"] / tot["steps"], 1),
        "mean_context": round(tot["context"] / max(tot["tokens"], 1), 1),
        # K/V bytes the steps' decodes read, over the whole loop's time: how close
        # the loop (host planning, copies, writes and decode together) runs to HBM
        "decode_kv_gbs": round(tot["context"] * row_bytes * 2 / (ms / 1e3) / 1e9, 1),
        "generated_tokens": tot["tokens"], "prefill_tokens": tot["prefill_tokens"],
        "cached_prompt_tokens": tot["cached"],
        "preemptions": tot["preempt"], "swapped_blocks": tot["swap_blocks"],
        "cow_copies": tot["cow"],
        "cascade_steps": tot["cascade_steps"],
        "cascade_saved_block_reads": tot["saved_blocks"],
        "kv_utilization": round(float(np.mean(util)), 4) if util else None,
        "contiguous_reservation_utilization": (round(float(np.mean(contiguous)), 4)
                                               if contiguous else None),
        "cache": "e4m3" if fp8_scales else wl.dtype,
        "what": f"{num_requests} requests (Poisson 1.0/step, lognormal prompts/outputs, "
                f"1/2/4 samples), pool {num_blocks} blocks, batch cap {max_num_seqs}, "
                f"host pool {host_blocks} blocks; utilization vs a {max_model_len}-token "
                f"contiguous reservation per sequence",
    }


HOLD_EVERY = 32           # timed launches queued behind one hold
HOLD_PER_STEP_S = 150e-6  # generous host time to enqueue one timed step


def gpu_hold(seconds: float) -> None:
    """Keep the current stream busy (a spin of about ``seconds`` at <= 2 GHz) while
    the host enqueues the next timed launches, so that they run back to back and
    CUDA events measure device time, not gaps while the host issues the next
    launch. Placed outside every pair of timing events."""
    import torch
    torch.cuda._sleep(int(seconds * 2.0e9))


def fp8_decode_bytes(wl) -> int:
    """Algorithmic bytes of one decode over an E4M3 cache: one byte per cached K
    and V element, 16-bit q and out, the used block-table entries and lengths."""
    ctx = wl.context_lens.astype(np.int64)
    kv = int(ctx.sum()) * wl.num_kv_heads * wl.head_dim * 2
    return kv + decode_bytes(wl) - int(ctx.sum()) * wl.num_kv_heads * wl.head_dim * \
        wl.elem_bytes * 2


def measure_fp8_decode(wl, runner, device, l2_flush, dec16_s, peak, iters: int = 50):
    """The same decode batch (tables, lengths, order, queries) over E4M3 caches
    of random valid codes: per-launch device time (CUDA events, warm-up first,
    the same L2 rule as the 16-bit measurement) and algorithmic bandwidth."""
    import torch
    from paged_kv_cache_352_b200 import _lib as L
    shape = tuple(runner.k_cache.shape)
    g = torch.Generator(device=device).manual_seed(352)

    def codes():
        c = torch.randint(0, 0x7E, shape, generator=g, device=device, dtype=torch.uint8)
        sign = torch.randint(0, 2, shape, generator=g, device=device, dtype=torch.uint8)
        return c | (sign << 7)

    kc, vc = codes(), codes()
    out = torch.empty_like(runner.q)
    ks, vs = 0.05, 0.02
    stream = torch.cuda.current_stream(device)

    def launch():
        if runner.groups is not None:   # blocks shared by forks: read once per group
            L.pa_paged_decode_cascade(out, runner.q, kc, vc, runner.block_tables,
                                      runner.context_lens, wl.max_context_len, wl.scale,
                                      runner.groups, runner.cascade_ws, runner.dev_error,
                                      k_scale=ks, v_scale=vs, seq_order=runner.cascade_order)
            return
        L.pa_paged_decode_fp8(out, runner.q, kc, vc, runner.block_tables, runner.context_lens,
                              wl.max_context_len, wl.scale, ks, vs,
                              partition_tokens=runner.partition_tokens or 0,
                              workspace=runner.workspace, dev_error=runner.dev_error,
                              seq_order=runner.seq_order)

    for _ in range(3):
        launch()
    torch.cuda.synchronize(device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(iters)]
    for i, (a, b) in enumerate(ev):
        if i % HOLD_EVERY == 0:
            gpu_hold(HOLD_EVERY * HOLD_PER_STEP_S)
        l2_flush()
        a.record(stream)
        launch()
        b.record(stream)
    torch.cuda.synchronize(device)
    if runner.error_bits():
        raise RuntimeError(f"fp8 decode: device error bits {runner.error_bits()}")
    t = float(np.mean([a.elapsed_time(b) for a, b in ev])) / 1e3
    nbytes = fp8_decode_bytes(wl)
    kernel = "paged_decode_kernel (E4M3 cache)"
    if runner.groups is not None:
        # distinct blocks at one byte per cached element (half the 16-bit K/V bytes)
        ctx_sum = int(wl.context_lens.astype(np.int64).sum())
        non_kv = decode_bytes(wl) - ctx_sum * wl.num_kv_heads * wl.head_dim * wl.elem_bytes * 2
        nbytes = (unique_decode_bytes(wl, runner) - non_kv) // 2 + non_kv
        kernel = "pa_paged_decode_cascade over E4M3 caches (distinct blocks)"
    achieved = nbytes / t / 1e9
    traffic = _traffic_for(wl.name + (":fp8" if runner.groups is None else ":cascade:fp8"))
    return {"kernel": kernel, "launch_ms": round(t * 1e3, 4),
            "algorithmic_bytes_per_launch": nbytes, "achieved_gbs": round(achieved, 2),
            "frac_of_hbm_peak": round(achieved / peak, 4),
            "traffic": traffic,
            "traffic_over_algorithmic": round(traffic / nbytes, 4) if traffic else None,
            "decode_tokens_per_s": round(wl.num_seqs / t, 1),
            "speedup_vs_16bit_decode": round(dec16_s / t, 3) if dec16_s == dec16_s else None,
            "what": "same batch as the 16-bit decode over E4M3 caches (random valid codes, "
                    "k_scale 0.05, v_scale 0.02), CUDA events per launch"}


def line_config(wl, args) -> dict:
    """The ``config`` object of a bench line: the workload's name and shape. Both
    arms print exactly this for the same arguments."""
    cfg = {"workload": wl.name, **{k: v for k, v in wl.describe().items() if k != "workload"}}
    pt = getattr(args, "partition_tokens", -1)
    if pt is not None and pt >= 0:
        cfg["partition_tokens"] = pt
    return cfg


def run_reference(args):
    rank, world, _ = _rank_info()
    if rank != 0:
        return 0
    import workloads
    wl = workloads.workload(args.workload)
    per_step_budget = max(0.5, 90.0 / max(1, args.steps + args.warmup))
    # calibrate the sample size per step on one sequence
    _, _, _, t1, _ = time_oracle(wl, budget_s=0.0, max_seq=1)
    nseq = int(max(1, min(wl.num_seqs, per_step_budget / max(t1, 1e-3))))
    from oracle.attention import paged_decode
    sub, st = oracle_sample_setup_range(wl, 0, nseq)

    def one():
        paged_decode(st.q, st.k_cache, st.v_cache, st.block_tables, sub.context_lens, sub.scale,
                     sub.dtype, sub.block_size)
    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    el = time.perf_counter() - t0
    bytes_per = decode_bytes(sub)
    value = bytes_per * args.steps / el / 1e9
    desc = (f"oracle paged_decode (fp64 NumPy) per step on {nseq} of {wl.num_seqs} sequences "
            f"({int(sub.context_lens.sum())} context tokens, all {wl.num_q_heads} query heads)")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": line_config(wl, args),
        "decode_tokens_per_s": round(nseq * args.steps / el, 3),
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": _oracle_threads(),
                         "host_cpus": _host_cpus(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _l2_flusher(wl, r, device, mode: str):
    """The L2 rule between timed launches. Inputs several times larger than L2
    need no flush (a cyclic scan larger than the cache leaves nothing to reuse);
    smaller ones get a flush that READS a buffer larger than L2, outside the
    timing events (a write flush would leave dirty lines whose write-back the
    next kernel would pay for). Sequences sharing blocks read only their distinct
    blocks from HBM, so those decide. Returns (flush callable, description)."""
    import torch
    l2_bytes = torch.cuda.get_device_properties(device).L2_cache_size
    read_bytes = unique_decode_bytes(wl, r) if r.groups is not None else decode_bytes(wl)
    needed = read_bytes < 4 * l2_bytes if mode == "auto" else mode == "flush"
    flush = torch.ones(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=device) if needed else None
    sink = torch.empty(1, dtype=torch.int64, device=device)

    def l2_flush():
        if flush is not None:
            torch.sum(flush, dim=0, out=sink)
    desc = ("flushed between steps by reading a 256 MiB buffer, outside the timed events"
            if needed else f"inputs larger than L2 ({read_bytes / 1e6:.0f} MB vs "
                           f"{l2_bytes / 1e6:.0f} MB L2), no flush")
    return l2_flush, desc


def time_steps(r, steps: int, device, l2_flush):
    """Two timed loops of ``steps`` iterations each, launched back to back behind a
    GPU hold every HOLD_EVERY iterations, with the L2 rule applied before each.
    First whole steps (copy-on-write copies, cache writes, decode), one pair of
    CUDA events around each on the launching stream, so that the step's launches
    run as they do in use (the decode may start while the cache write ahead of it
    drains); then the decode alone, for the roofline. Returns per-iteration
    (step seconds, decode seconds)."""
    import torch
    stream = torch.cuda.current_stream(device)

    def loop(body):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for k in range(steps):
            if k % HOLD_EVERY == 0:
                gpu_hold(HOLD_EVERY * HOLD_PER_STEP_S)
            l2_flush()
            ev[k][0].record(stream)
            body()
            ev[k][1].record(stream)
        torch.cuda.synchronize(device)
        return np.array([a.elapsed_time(b) for a, b in ev]) / 1e3

    def step():
        r.copy_blocks()
        r.reshape_and_cache()
        r.decode_step()
    t_step = loop(step)
    t_dec = loop(r.decode_step)
    return t_step, t_dec


def time_copy_blocks(r, wl, device):
    """pa_copy_blocks of the step's copy-on-write pairs alone (idempotent: each pair
    copies the same source), 20 launches back to back behind a GPU hold."""
    import torch
    if len(r.cow_pairs) == 0:
        return None
    stream = torch.cuda.current_stream(device)
    ca, cb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gpu_hold(20 * HOLD_PER_STEP_S)
    ca.record(stream)
    for _ in range(20):
        r.copy_blocks()
    cb.record(stream)
    torch.cuda.synchronize(device)
    tc = ca.elapsed_time(cb) / 20 / 1e3
    nbytes = len(r.cow_pairs) * 2 * 2 * wl.num_kv_heads * 16 * wl.head_dim * wl.elem_bytes
    return {"pairs": len(r.cow_pairs), "ms": round(tc * 1e3, 4), "bytes": nbytes,
            "gbs": round(nbytes / tc / 1e9, 1),
            "what": "pa_copy_blocks of the step's copy-on-write pairs (K and V, read + write), "
                    "CUDA events around 20 back-to-back launches"}


def time_plain_decode(r, device, l2_flush, cascade_s: float):
    """For batches decoded through the cascade: the same batch through
    pa_paged_decode, in which every sequence reads its shared blocks itself."""
    import torch
    stream = torch.cuda.current_stream(device)
    pe = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(20)]
    gpu_hold(20 * HOLD_PER_STEP_S)
    for a_, b_ in pe:
        l2_flush()
        a_.record(stream)
        r.decode()
        b_.record(stream)
    torch.cuda.synchronize(device)
    tp = float(np.mean([a_.elapsed_time(b_) for a_, b_ in pe])) / 1e3
    return {"ms": round(tp * 1e3, 4), "cascade_speedup": round(tp / cascade_s, 3),
            "what": "pa_paged_decode of the same batch (every sequence reads its "
                    "shared blocks itself), CUDA events, mean of 20"}


def decode_roofline(wl, r, dec_s: float, peak: float, peak_kind: str, read_ref):
    """The decode call against the HBM roofline: algorithmic bytes per call (distinct
    blocks for batches whose sequences share blocks) over its mean device time."""
    db = decode_bytes(wl)
    kernel = "paged_decode_kernel"
    if r.groups is None and r.decode_launches() == 2:
        kernel = "paged_decode_warp_parts_kernel + merge_partitions_kernel"
    if r.groups is not None:
        db = unique_decode_bytes(wl, r)
        kernel = ("pa_paged_decode_cascade: cascade_prepare_kernel, cascade_decode_kernel (the "
                  "groups' shared blocks and every sequence's own blocks in one launch), "
                  "cascade_merge_kernel")
    achieved = db / dec_s / 1e9
    roof = {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 2), "peak": peak,
            "unit": "GB/s", "frac": round(achieved / peak, 4),
            "traffic": _traffic_for(wl.name + (":cascade" if r.groups is not None else "")),
            "algorithmic_bytes_per_launch": db, "launch_ms": round(dec_s * 1e3, 4),
            "peak_kind": peak_kind,
            "pct_of_nominal_8tbs": round(100 * achieved / 8000.0, 2)}
    if read_ref:
        # the copy peak counts read + write bytes; a read-only stream measured in
        # the same run is the tighter ceiling for a read-dominated kernel
        roof["read_stream_gbs"] = round(read_ref, 1)
        roof["frac_of_read_stream"] = round(achieved / read_ref, 4)
    return roof


def measure_config(name: str, args, device, peak: float, peak_kind: str, read_ref):
    """One workload's step at full size (set-up, warm-up, ``args.steps`` timed steps
    with the headline's protocol) and its decode against the roofline. For the
    per-workload object of the bench line; everything it allocates is released."""
    import torch
    from paged_kv_cache_352_b200 import _lib as L
    from paged_kv_cache_352_b200.runner import DecodeRunner
    import workloads
    wl = workloads.workload(name)
    r = DecodeRunner(wl, device=device)
    l2_flush, l2_desc = _l2_flusher(wl, r, device, "auto")
    for _ in range(max(3, args.warmup)):
        r.step()
    torch.cuda.synchronize(device)
    if r.error_bits():
        raise RuntimeError(f"{name}: device error bits {r.error_bits()} during warm-up")
    t_step, t_dec = time_steps(r, args.steps, device, l2_flush)
    if r.error_bits():
        raise RuntimeError(f"{name}: device error bits {r.error_bits()} during timing")
    step_s, dec_s = float(t_step.mean()), float(t_dec.mean())
    sb = step_bytes(wl, r)
    if r.groups is not None:
        sb = sb - decode_bytes(wl) + unique_decode_bytes(wl, r)
    roof = decode_roofline(wl, r, dec_s, peak, peak_kind, read_ref)
    res = {
        "decode_us": {"mean": round(1e6 * dec_s, 2),
                      "median": round(1e6 * float(np.median(t_dec)), 2),
                      "min": round(1e6 * float(t_dec.min()), 2)},
        "decode_gbs": roof["achieved"], "frac": roof["frac"],
        "pct_of_nominal_8tbs": roof["pct_of_nominal_8tbs"],
        "frac_of_read_stream": roof.get("frac_of_read_stream"),
        "algorithmic_bytes": roof["algorithmic_bytes_per_launch"], "traffic": roof["traffic"],
        "decode_tokens_per_s": round(wl.num_seqs / dec_s, 1),
        "step_ms": round(1e3 * step_s, 4), "step_gbs": round(sb / step_s / 1e9, 2),
        "step_tokens_per_s": round(wl.num_seqs / step_s, 1),
        "kernel": roof["kernel"], "partition_tokens": r.partition_tokens, "l2": l2_desc,
        "dtype": wl.dtype, "steps": args.steps,
    }
    if name == "tiny_mha_d64":
        res["note"] = ("0.11 MB per launch: one launch latency, so the 70 % bandwidth target "
                       "cannot apply")
    if r.groups is not None:
        res["cascade_plan"] = L.pa_paged_decode_cascade_plan(
            wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.max_context_len,
            r.max_blocks, r.groups.num_groups, r.groups.group_size, r.groups.max_prefix_blocks,
            dtype=wl.dtype)
        res["logical_decode_gbs"] = round(decode_bytes(wl) / dec_s / 1e9, 2)
        res["plain_decode"] = time_plain_decode(r, device, l2_flush, dec_s)
        res["copy_blocks"] = time_copy_blocks(r, wl, device)
    if wl.num_seqs > 4:
        res["fp8_kv"] = measure_fp8_decode(wl, r, device, l2_flush, dec_s, peak,
                                           iters=max(args.steps, 20))
    del r
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    rank, world, local = _rank_info()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(device)

    from paged_kv_cache_352_b200 import build as pabuild
    pabuild.build()
    from paged_kv_cache_352_b200.runner import DecodeRunner, HostPipeline
    import workloads

    wl = rank_workload(args.workload, rank, args.num_seqs, args.num_blocks)
    r = DecodeRunner(wl, device=device,
                     partition_tokens=args.partition_tokens if args.partition_tokens >= 0 else None)
    l2_flush, l2_desc = _l2_flusher(wl, r, device, args.l2)

    for _ in range(max(3, args.warmup)):
        r.step()
    torch.cuda.synchronize(device)
    if r.error_bits():
        raise RuntimeError(f"device error bits {r.error_bits()} during warm-up")
    if args.only == "fp8":
        # profiling only: the 8-bit decode of this batch, nothing else
        line = measure_fp8_decode(wl, r, device, l2_flush, float("nan"), _peaks()[0],
                                  iters=args.steps)
        print(json.dumps({"only": "fp8", "workload": wl.name, **line}), flush=True)
        return 0

    K = args.steps
    _barrier(world)
    torch.cuda.synchronize(device)
    with ClockSampler(device) as clocks:
        t_step, t_dec = time_steps(r, K, device, l2_flush)
    _barrier(world)
    step_s = _max_over_ranks(float(t_step.mean()), world, device)
    dec_s = _max_over_ranks(float(t_dec.mean()), world, device)
    if r.error_bits():
        raise RuntimeError(f"device error bits {r.error_bits()} during timing")
    decode_ms = {"mean": round(1e3 * float(t_dec.mean()), 4),
                 "median": round(1e3 * float(np.median(t_dec)), 4),
                 "min": round(1e3 * float(t_dec.min()), 4)}
    # the step's cache writes (copy-on-write copies + new tokens) before the decode:
    # what the step costs beyond the decode alone
    cache_write_ms = round(1e3 * float(t_step.mean() - t_dec.mean()), 4)
    copy_blocks = time_copy_blocks(r, wl, device) if world == 1 else None
    plain_decode = time_plain_decode(r, device, l2_flush, dec_s) \
        if r.groups is not None and world == 1 else None

    # e2e: the same step fed from pinned host buffers, result read back to the
    # host, with the next step's input copy overlapping this step's kernels
    hs = HostPipeline(r)
    for _ in range(3):
        hs()
    torch.cuda.synchronize(device)
    E = max(10, K // 2)
    _barrier(world)
    torch.cuda.synchronize(device)
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(hs.upload)
    for k in range(E):
        hs()
    hs.compute.wait_stream(hs.download)
    e_end.record(hs.compute)
    torch.cuda.synchronize(device)
    _barrier(world)
    e2e_s = _max_over_ranks(e_start.elapsed_time(e_end) / 1e3 / E, world, device)

    peak, peak_kind = _peaks()
    read_ref = read_stream_gbs(device) if world == 1 else None
    sb = step_bytes(wl, r)
    db = decode_bytes(wl)
    effective = None
    if r.groups is not None:
        # Sequences share blocks: the bytes that must leave HBM are those of the
        # distinct blocks read; the logical rate is reported beside them.
        ub = unique_decode_bytes(wl, r)
        effective = {"decode_gbs_logical": round(db / dec_s / 1e9, 2),
                     "step_gbs_logical": round(world * sb / step_s / 1e9, 2),
                     "logical_decode_bytes": db, "unique_decode_bytes": ub}
        sb = sb - db + ub
    value = world * sb / step_s / 1e9
    roofline = decode_roofline(wl, r, dec_s, peak, peak_kind, read_ref)
    csum = clocks.summary()
    # the timed region holds K whole steps and then K decodes alone
    launches_timed = K * (r.launches_per_step() + r.decode_launches())
    fp8 = measure_fp8_decode(wl, r, device, l2_flush, dec_s, peak) \
        if world == 1 and args.only == "all" and r.groups is None else None
    e2e = {"value": round(world * sb / e2e_s / 1e9, 2), "unit": UNIT,
           "h2d_bytes_per_step": hs.h2d_bytes, "d2h_bytes_per_step": hs.d2h_bytes,
           "ms_per_step": round(e2e_s * 1e3, 4),
           "what": "the step through the C interface fed from pinned host buffers (queries, new "
                   "keys/values, slot mapping, block tables, lengths, order copied host -> device "
                   "every step, output copied back); the block tables and slots are the "
                   "workload's, planned once before timing (host planning per step is measured "
                   "in host_planning)"}
    del hs
    extras = world == 1 and args.only == "all"
    # 512 MiB of whole blocks each way between the pool and pinned host memory
    blk_bytes = 2 * r.k_cache[0].numel() * r.k_cache.element_size()
    swap = measure_swap(wl, r, device, nblocks=(512 << 20) // blk_bytes) if extras else None
    del r
    torch.cuda.empty_cache()

    # every other workload at full size, with the same protocol (one GPU only)
    per_config = None
    if extras:
        per_config = {}
        for name in PER_CONFIG:
            if name != wl.name:
                per_config[name] = measure_config(name, args, device, peak, peak_kind, read_ref)
    # the serving-loop extras run on 7B-like MHA heads (32/32, d 128, fp16)
    loop_wl = workloads.workload(LOOP_SHAPE) if extras else None
    prefix_cache = measure_prefix_cache(loop_wl, device) if extras else None

    def loop(**kw):
        """The loop with the executor's default cascade rule, and the generated
        tokens/s of the same trace with the cascade off beside it."""
        res = measure_continuous_batching(loop_wl, device, **kw)
        import paged_kv_cache_352_b200 as pa
        off = measure_continuous_batching(loop_wl, device, cascade=pa.PA_SCHED_CASCADE_OFF, **kw)
        res["cascade_off"] = {"value": off["value"], "ms_per_step": off["ms_per_step"]}
        return res

    batching = loop() if extras else None
    host_planning = measure_host_planning() if extras else None
    batching_fp8 = loop(fp8_scales=(0.05, 0.02)) if extras else None
    batching_prefix = None
    if extras:
        spt = shared_prompt_trace()
        batching_prefix = {
            "with_cache": loop(trace=spt, use_tokens=True),
            "without_cache": measure_continuous_batching(loop_wl, device, trace=spt),
        }

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": max(3, args.warmup), "ms_per_step": round(step_s * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic",
        "config": line_config(wl, args),
        "l2_policy": l2_desc,
        "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "hbm_peak_gbs": peak, "hbm_peak_kind": peak_kind,
        "pct_of_nominal_8tbs": round(100 * value / world / 8000.0, 2),
        "read_stream_ref_gbs": round(read_ref, 1) if read_ref else None,
        "decode_ms": decode_ms, "cache_write_ms": cache_write_ms, "copy_blocks": copy_blocks,
        "decode_tokens_per_s": round(world * wl.num_seqs / step_s, 1),
        "decode_only_tokens_per_s": round(world * wl.num_seqs / dec_s, 1),
        "bytes_per_step": sb,
        "shared_blocks": effective, "plain_decode": plain_decode,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": launches_timed,
        "per_config": per_config,
        "fp8_kv": fp8,
        "swap": swap,
        "prefix_cache": prefix_cache,
        "continuous_batching": batching,
        "host_planning": host_planning,
        "continuous_batching_fp8": batching_fp8,
        "continuous_batching_shared_prompts": batching_prefix,
        "clocks": csum,
    }
    if world == 1 and not args.no_cpu_baseline:
        v, tps, desc, _, chunks = time_oracle(wl, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": round(v, 4), "unit": UNIT, "cores": _oracle_threads(),
                                "host_cpus": _host_cpus(),
                                "kind": "oracle", "sample": desc,
                                "decode_tokens_per_s": round(tps, 3)}
        one = time_oracle_one_thread(wl, budget_s=min(5.0, args.cpu_budget / 3), chunks=chunks)
        if one is not None:
            line["cpu_baseline"]["one_thread"] = one
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--partition-tokens", type=int, default=-1,
                    help="split-KV partition size (default: the workload's / library default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--l2", choices=["auto", "flush", "none"], default="auto",
                    help="L2 handling between steps: auto = flush (by a read) only when the "
                         "step's inputs are smaller than 4x L2")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="profiling only: keep the first N sequences of the batch")
    ap.add_argument("--num-blocks", type=int, default=0,
                    help="profiling only: pool size for the truncated batch")
    ap.add_argument("--only", choices=["all", "decode", "fp8"], default="all",
                    help="profiling only: 'decode' times the step without the extra "
                         "measurements (swap, prefix cache, batching loop, 8-bit decode); "
                         "'fp8' times only the 8-bit decode of the batch (--steps launches)")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle time for the cpu_baseline sample")
    args = ap.parse_args(argv)
    if args.steps < 1 or args.warmup < 0:
        ap.error("--steps >= 1 and --warmup >= 0")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
