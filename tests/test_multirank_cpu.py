"""The N > 1 path of bench.py on CPU: two gloo ranks, each a replica with its
own time; the job time is the slowest rank's and the throughput counts the
units of every rank (weak scaling, no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 20.0][rank]
        worst = bench.max_over_ranks(local_ms, dist, "cpu")
        units = 1000.0   # per-rank work per step
        value = bench.job_throughput(units / (worst / 1e3), world, 1.0)
        results[rank] = (worst, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_replica_aggregation():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        worst, value = results[r]
        assert worst == 20.0
        assert value == pytest.approx(2 * 1000.0 / 0.020)


def test_single_rank_helpers():
    import bench
    assert bench.max_over_ranks(3.0) == 3.0
    assert bench.job_throughput(10.0, 1, 2.0) == 5.0


def test_reference_arm_non_zero_rank_exits_quietly():
    # under torchrun the reference arm runs on rank 0 only; the other ranks
    # exit 0 without work or output
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_line():
    # rank 0 times the oracle on a bounded sample and prints one JSON line
    # with the GPU arm's metric and unit, the reference marker, a cpu_baseline
    # describing this run and an e2e entry with no copies
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--workload", "square_mx", "--steps", "1", "--warmup", "0"], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    import bench
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s"
    assert d["steps"] == 1 and d["warmup"] == 0 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["config"]["workload"] == "MXFP4 quantize+GEMM M=N=K=4096"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["e2e"]["d2h_bytes_per_step"] == 0
