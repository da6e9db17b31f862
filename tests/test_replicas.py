"""The multi-GPU path of bench.py (independent replicas, no data-path
collective) exercised as world_size-2 gloo ranks on the CPU: the slowest
rank's time is what every rank reports, the job's throughput counts the
work of every replica, and the reference arm prints one line from rank 0
only."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    local_ms = [12.5, 20.0][rank]
    bench.barrier(world)
    m = bench.max_over_ranks(local_ms, world, device="cpu")
    v = bench.replica_throughput(1e12, 10, m, world)
    dist.destroy_process_group()
    out.put((rank, m, v))


def test_two_gloo_ranks_report_the_slowest_rank_and_the_whole_job():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, v in res:
        assert m == 20.0                                  # the slower rank's interval
        assert v == pytest.approx(2 * 1e12 * 10 / 0.020)  # both replicas' work in that time


def test_reference_arm_under_torchrun_prints_once():
    """`--impl reference` under a 2-rank launch: rank 0 times the oracle and
    prints one JSON line, the other rank exits 0 without work."""
    port = 30500 + os.getpid() % 1000
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "B1-H2-n256-d64-causal", "--reference-seconds", "2"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
