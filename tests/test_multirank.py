"""The benchmark's multi-rank logic on two CPU ranks (gloo): weak scaling,
each rank drawing its own batch, with the job's time the slowest rank's and
no collective on the data path."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from bit_kv_cache_20_b200 import workloads
    cfg = workloads.CONFIGS["tiny"]
    w = workloads.make("tiny", seed=bench.rank_seed(cfg.seed, rank))
    fake_ms = 10.0 + 5.0 * rank                 # rank 1 is the slow one
    slowest = bench.reduce_max(fake_ms, world, "cpu")
    digest = float(workloads.bf16_bits(w.k_new).astype(np.int64).sum() % 1000003)
    t = torch.tensor([digest], dtype=torch.float64)
    gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(gathered, t)
    results[rank] = (slowest, [float(g.item()) for g in gathered])
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_weak_scaling_logic():
    world = 2
    mgr = mp.get_context("spawn").Manager()  # no fork of a process that has threads
    results = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
    assert results[0][0] == results[1][0] == 15.0          # max over ranks
    d0, d1 = results[0][1]
    assert d0 != d1                                         # independent batches
    import bench
    from bit_kv_cache_20_b200 import workloads
    w = workloads.make("tiny")
    per_step = bench.write_bytes(w.tokens_written, w.Hkv, w.D)
    # whole-job throughput counts every rank's bytes over the slowest time
    assert bench.aggregate_gbs(per_step, 10, world, 15.0) == per_step * 10 * 2 / 0.015 / 1e9


def test_reference_arm_on_a_non_zero_rank_exits_without_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"]) == 0
    assert capsys.readouterr().out == ""


def test_prefill_flops_counts_every_causal_pair():
    # brute force: query i of a chunk of L at context c sees positions 0 .. c - L + i
    import bench
    for ctx, chunk in (([1, 5, 40], 16), ([3000, 70, 2048], 2048), ([0, 9], 4)):
        pairs = 0
        for c in ctx:
            L = min(chunk, c)
            for i in range(L):
                pairs += sum(1 for pos in range(c) if pos <= c - L + i)
        assert bench.prefill_flops(ctx, chunk, Hq=3, D=8) == 4 * 8 * 3 * pairs


def test_source_digest_ignores_comments_only():
    import bench
    src = "int a; // one\n/* two\n three */ int b;\n\n  int c;  // four\n"
    assert bench.strip_comments(src) == "int a;\n int b;\n  int c;"
    assert bench.strip_comments(src) == bench.strip_comments(src.replace("one", "changed wording"))
    assert bench.strip_comments(src) != bench.strip_comments(src.replace("int b", "int bb"))


def test_reference_arm_prints_one_contract_line(monkeypatch, capsys):
    import json
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    assert bench.main(["--impl", "reference", "--config", "tiny", "--steps", "2", "--warmup", "1"]) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["value"] > 0 and d["steps"] == 2 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "tiny"


def test_bench_gpus_n_starts_n_ranks():
    """`python bench.py --gpus 2` with no torchrun starts two ranks itself;
    with --launch-check they count themselves over gloo on the CPU and rank 0
    prints the n_gpus the line would report."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--launch-check"],
                         capture_output=True, text=True, timeout=120, env=env, check=True).stdout
    lines = [json.loads(l) for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out
    assert lines[0]["n_gpus"] == 2 and lines[0]["ranks_seen"] == 2
