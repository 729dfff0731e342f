"""Host logic of the N-rank benchmark, on the CPU with two gloo ranks.

The FP4 path has no data-path collective (each rank runs an independent
replica of the step); what the multi-rank run adds is the rank setup, the
max-over-ranks step time and the whole-job token count.  These run here with
the gloo backend; the same functions take NCCL on the GPU machine."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    bench.init_ranks(world, torch.device("cpu"), backend="gloo")
    try:
        # rank r's step took (r + 1) * 10 ms: every rank must see the slowest
        ms = bench.max_over_ranks(10.0 * (rank + 1), torch.device("cpu"))
        rate = bench.whole_job_tokens_per_s(world, ms)
        results[rank] = (ms, rate)
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_ranks_take_the_slowest_step_and_count_all_tokens():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world,
                           start_method="spawn", join=True)
        got = dict(results)
    import bench
    for r in range(world):
        ms, rate = got[r]
        assert ms == 20.0
        assert rate == pytest.approx(world * bench.T / 0.020)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.whole_job_tokens_per_s(1, 1000.0) == bench.T
    bench.init_ranks(1, torch.device("cpu"))
    assert not torch.distributed.is_initialized()


@pytest.mark.timeout(120)
def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the oracle arm prints from rank 0; other ranks exit 0
    at once without work or output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=110)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""


def test_every_rank_draws_distinct_inputs():
    """Replicas must not all quantize the same tensors: the per-rank seeds of
    the benchmark's inputs never collide across ranks and layers."""
    import bench
    seeds = [s for rank in range(8) for i in range(len(bench.LAYERS))
             for s in bench.input_seeds(rank, i)]
    assert len(seeds) == len(set(seeds))


@pytest.mark.timeout(900)
def test_reference_arm_prints_the_contract_line():
    """The oracle arm on rank 0: one JSON line with the kernel arm's metric,
    unit and config, the oracle's cpu_baseline and an e2e with no copies."""
    import json
    import bench
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=880)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["config"] == bench.bench_config(1) and d["higher_is_better"] is True
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
