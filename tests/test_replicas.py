"""The multi-GPU path of bench.py (independent replicas, no data-path
collective) exercised as world_size-2 gloo ranks on the CPU: the slowest
rank's time is what every rank reports, the job's throughput counts the
work of every replica, and the reference arm prints one line from rank 0
only. One problem split across ranks by (batch, head) pairs (independent
attention problems, disjoint outputs, no exchange) gives the single-rank
result when the slices are gathered."""
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
    # the same config keys as the GPU arm's line, so the two lines compare
    cfg = line["config"]
    assert cfg["workload"] == "B1-H2-n256-d64-causal"
    assert cfg["global_batch"] == 2 and cfg["seq_len"] == 256 and cfg["parallelism"] == "replicas2"
    assert "l2" in cfg


def test_head_shards_cover_every_pair_once():
    sys.path.insert(0, ROOT)
    import bench
    for bh in (1, 2, 7, 8, 64):
        for world in (1, 2, 3, 8):
            spans = [bench.head_shard(bh, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == bh
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0                       # contiguous, no overlap
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1       # balanced


def _shard_main(rank, world, port, out):
    """One rank of a problem split by (batch, head): it computes its own
    slice of the heads with the oracle; the slices are gathered over gloo."""
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    from exact_softmax_attention_04_b200 import synth
    B, H, n, d = 2, 3, 77, 64
    q, k, v = synth.make_qkv(B, H, n, d, seed=11, q_std=2.0)
    a, b = bench.head_shard(B * H, world, rank)
    sl = lambda t: t.reshape(B * H, 1, n, d)[a:b].reshape(1, b - a, n, d)
    o, lse = oracle.attn_fwd(sl(q), sl(k), sl(v), 1.0 / 8.0, True, 20)
    # gather the variable-sized slices: pad to the largest, then trim
    most = -(-B * H // world)
    pad_o = torch.zeros((most, n, d), dtype=torch.float64)
    pad_l = torch.zeros((most, n), dtype=torch.float64)
    pad_o[: b - a] = torch.from_numpy(o.reshape(b - a, n, d))
    pad_l[: b - a] = torch.from_numpy(lse.reshape(b - a, n))
    go = [torch.empty_like(pad_o) for _ in range(world)]
    gl = [torch.empty_like(pad_l) for _ in range(world)]
    dist.all_gather(go, pad_o)
    dist.all_gather(gl, pad_l)
    dist.destroy_process_group()
    if rank == 0:
        spans = [bench.head_shard(B * H, world, r) for r in range(world)]
        o_all = torch.cat([g[: e - s] for g, (s, e) in zip(go, spans)]).numpy()
        l_all = torch.cat([g[: e - s] for g, (s, e) in zip(gl, spans)]).numpy()
        out.put((o_all, l_all))
    else:
        out.put(None)


def test_problem_split_by_heads_over_two_gloo_ranks_equals_one_rank():
    """The multi-GPU split of one problem: two gloo ranks each compute half of
    the (batch, head) pairs (the oracle stands in for the kernel on the CPU),
    and the gathered halves equal the single-process result bit for bit."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    from exact_softmax_attention_04_b200 import synth
    oracle.build()
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    port = 31500 + os.getpid() % 1000
    procs = [ctx.Process(target=_shard_main, args=(r, 2, port, q_)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q_.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    o_all, l_all = next(r for r in res if r is not None)
    q, k, v = synth.make_qkv(2, 3, 77, 64, seed=11, q_std=2.0)
    o_ref, l_ref = oracle.attn_fwd(q, k, v, 1.0 / 8.0, True, 20)
    assert np.array_equal(o_all, o_ref.reshape(6, 77, 64))
    assert np.array_equal(l_all, l_ref.reshape(6, 77))
