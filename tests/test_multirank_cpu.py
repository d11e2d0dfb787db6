"""The multi-GPU host logic of the benchmark, on CPU with gloo (world size 2).

The decode step has no exchange between GPUs: N GPUs run N independent
replicas, each with its own pool and its own seeded batch, and the reported
time is the maximum over ranks. These tests run that logic on two CPU ranks.
"""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench._max_over_ranks(0.25 + rank, world)
        wl = bench.rank_workload("mha_7b_fp16", rank)
        info = bench._rank_info()
        bench._barrier(world)
        q.put((rank, t, wl.seed, wl.context_lens.tolist()[:4], wl.free_order[:4].tolist(),
               info))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_draw_independent_batches():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert all(r[1] == 1.25 for r in res)                       # max over ranks
    assert res[0][2] != res[1][2]                               # independent batches
    assert res[0][3] != res[1][3] or res[0][4] != res[1][4]
    assert [r[5] for r in res] == [(0, 2, 0), (1, 2, 1)]


def test_rank_zero_batch_is_the_named_workload():
    import workloads
    a = bench.rank_workload("gqa_32_8_bf16", 0)
    b = workloads.workload("gqa_32_8_bf16")
    assert a.seed == b.seed and np.array_equal(a.context_lens, b.context_lens)


def test_reference_arm_other_ranks_do_nothing(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), {"workload": "tiny_mha_d64", "steps": 1, "warmup": 0})
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line(monkeypatch, capsys):
    import json
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    args = type("A", (), {"workload": "tiny_mha_d64", "steps": 2, "warmup": 1})
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"]["workload"] == "tiny_mha_d64"


def test_byte_accounting_matches_definition():
    import workloads
    wl = workloads.workload("tiny_mha_d64")
    # contexts {1, 16, 17, 70}: 104 tokens x 4 heads x 64 x 2 B x (K+V)
    kv = 104 * 4 * 64 * 2 * 2
    qo = 2 * 4 * 4 * 64 * 2
    tables = 4 * (1 + 1 + 2 + 5)
    assert bench.decode_bytes(wl) == kv + qo + tables + 4 * 4


def test_both_arms_print_the_same_config(monkeypatch, capsys):
    """The repo arm and the reference arm describe the workload with one function,
    so the driver sees the same ``config`` for the same arguments."""
    import json
    import workloads
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    args = type("A", (), {"workload": "tiny_mha_d64", "steps": 1, "warmup": 0,
                          "partition_tokens": -1})
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["config"] == bench.line_config(workloads.workload("tiny_mha_d64"), args)
    assert "l2" not in line["config"] and "parallelism" not in line["config"]
    src = open(bench.__file__).read()
    assert src.count('"config": line_config(wl, args)') == 2


def test_default_workload_is_the_largest_single_gpu_batch():
    import workloads
    sizes = {n: bench.decode_bytes(workloads.workload(n)) for n in bench.PER_CONFIG}
    assert bench.DEFAULT_WORKLOAD == max(sizes, key=sizes.get) == "long_ctx_split_kv"
