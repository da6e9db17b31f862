"""Benchmark: attention forward TFLOP/s (unmasked FLOPs) on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                [--workload NAME]

One step = one attention forward (the whole hot path: one kernel launch).
Default workload: B=1, H=8, n=131072, d=128, full causal mask, bf16 Q/K/V ~
N(0,1) from seed 0 -- the long-context stress case and the largest of the
target configurations that fits one GPU (the cost of long contexts is the
subject of "Quadratic cost and efficient attention", section "What long
context really costs"). Other workloads by name with --workload, e.g.
B8-H8-n8192-d64-none (the 8x8x8192 worked example of the same page, d_model
512 over 8 heads) or B1-H32-n32768-d128-window4096 (Mistral's w = 4096).
FLOPs counted: 4*d per attended (query, key) pair. Inputs and outputs of the
default workload (0.8 GB in, 0.27 GB out) exceed the 126 MB L2, so no
explicit flush is done between steps. Under torchrun every rank runs its own
replica (the work shards by (batch, head) with no exchange), so scaling is
weak and the value is the sum of all ranks' FLOPs over the slowest rank's
time.

--impl reference times the fp64 CPU oracle on a bounded row sample of the
same workload (rank 0 only): the deliberately slow reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOP/s (unmasked FLOPs) and % of B200 dense BF16 peak"
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
KERNEL_NAME = "attn_fwd_kernel"
# the largest target configuration that fits one GPU
DEFAULT_WORKLOAD = "B1-H8-n131072-d128-causal"


def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, FALLBACK_HBM_GBS, "fallback"


# Device code of the timed forward kernel: the traffic record goes stale when
# the code in either file changes (comments and blank lines do not count).
FWD_KERNEL_SOURCES = ("attn_fwd_kernel.cuh", "sm100.cuh")


def strip_comments(src: str) -> str:
    """C++ source without // and /* */ comments, trailing blanks and blank
    lines; string and character literals are kept as they are."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            while i < n and src[i] != "\n":
                i += 1
        elif src.startswith("/*", i):
            end = src.find("*/", i + 2)
            i = n if end < 0 else end + 2
        else:
            out.append(c)
            i += 1
    lines = [line.rstrip() for line in "".join(out).split("\n")]
    return "\n".join(line for line in lines if line)


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_softmax_attention_04_b200", "csrc")
    for f in FWD_KERNEL_SOURCES:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(f.encode() + b"\0" + strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary of this workload,
    if it was taken on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", f"{KERNEL_NAME}.{workload}.traffic.txt")
    try:
        vals = {}
        with open(path) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    vals[k.strip()] = v.strip()
        if vals.get("kernel_sources_sha256_16") != kernel_source_hash():
            return None
        return int(vals["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi samples during the timed region (SM clock, throttle reasons)."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        self.out = ""
        if self.gpu < 0:
            return self
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self, t0=None, t1=None):
        """Median SM clock and throttle reasons over the samples taken inside
        [t0, t1] (wall clock, seconds); all samples if none fall inside."""
        import datetime
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[1]), float(parts[2]),
                             {nm for nm, val in zip(names, parts[5:9]) if val.lower().startswith("active")}))
            except ValueError:
                continue
        inside = [r for r in rows if t0 is not None and t0 - 0.1 <= r[0] <= t1 + 0.1]
        use = inside or rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set().union(*(r[3] for r in use))
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": use[-1][2],
                "reasons": sorted(reasons), "samples": len(use),
                "window": "timed region" if inside else "whole run (no sample inside the timed region)"}


def dist_setup(n_gpus: int):
    world = _env_int("WORLD_SIZE", 1)
    rank = _env_int("RANK", 0)
    local = _env_int("LOCAL_RANK", 0)
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The largest x over all ranks (every rank gets it); the timed interval
    of a multi-GPU run is the slowest rank's."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(units_per_rank: float, steps: int, max_ms: float, world: int) -> float:
    """Whole-job throughput of independent replicas: every rank processes
    units_per_rank per step, the job takes the slowest rank's time."""
    return world * units_per_rank * steps / (max_ms / 1e3)


def head_shard(bh: int, world: int, rank: int):
    """Contiguous range [start, stop) of the flattened (batch, head) pairs that
    `rank` of `world` owns when one problem is split across ranks: every
    (batch, head) pair is an independent attention problem, so the ranks
    need no exchange and their outputs are disjoint slices. Earlier ranks
    take one extra pair when bh does not divide evenly."""
    base, extra = divmod(bh, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def workload_config(wl, world: int) -> dict:
    """The `config` object of a JSON line, identical for both arms: the
    workload, its size per replica and how L2 is handled between steps."""
    elems = wl.B * wl.H * wl.n * wl.d
    in_bytes = 2 * elems + 2 * 2 * wl.B * wl.kv_heads * wl.n * wl.d
    out_bytes = 2 * elems + 4 * wl.B * wl.H * wl.n
    return {**wl.describe(), "global_batch": wl.B * world, "seq_len": wl.n,
            "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": f"no flush: inputs {in_bytes / 1e6:.0f} MB + outputs {out_bytes / 1e6:.0f} MB per step "
                  + ("exceed" if in_bytes > 126e6 else "do NOT exceed") + " the 126 MB L2"}


def cpu_baseline_leg(wl, o_gpu=None, lse_gpu=None, target_s: float = 15.0):
    """Oracle timed on this host's cores over a bounded row sample of the
    workload; also compares those rows with the GPU outputs if given."""
    import numpy as np
    import oracle
    from exact_softmax_attention_04_b200 import synth
    oracle.build()
    q, k, v = synth.make_inputs(wl)
    pairs = synth.workload_pairs_per_head(wl)
    flops_per_row = 4.0 * wl.d * pairs / wl.n
    g = torch.Generator().manual_seed(2)
    total = wl.B * wl.H * wl.n
    # calibrate on a small sample, then size the sample to ~target_s seconds
    probe = torch.randint(0, total, (64,), generator=g).numpy()
    t0 = time.perf_counter()
    oracle.attn_rows_gqa(q, k, v, wl.scale, wl.causal, wl.window, probe, block=wl.block)
    dt = max(time.perf_counter() - t0, 1e-3)
    nrows = int(min(total, max(64, 64 * target_s / dt)))
    rows = np.sort(torch.randint(0, total, (nrows,), generator=g).numpy())
    t0 = time.perf_counter()
    o_ref, lse_ref = oracle.attn_rows_gqa(q, k, v, wl.scale, wl.causal, wl.window, rows, block=wl.block)
    dt = time.perf_counter() - t0
    out = {"value": nrows * flops_per_row / dt / 1e12, "unit": "TFLOP/s",
           "cores": oracle.num_threads(), "kind": "oracle",
           "sample": f"{nrows} random query rows (seed 2) of {wl.name}, fp64 two-pass softmax, "
                     f"{dt:.1f} s wall",
           "seconds": dt}
    if o_gpu is not None:
        idx = torch.as_tensor(rows, device=o_gpu.device)
        og = o_gpu.view(-1, wl.d)[idx].float().cpu().numpy()
        lg = lse_gpu.view(-1)[idx].cpu().numpy()
        diff = og - o_ref
        out["parity_vs_gpu"] = {
            "rows": int(nrows),
            "o_max_abs": float(np.abs(diff).max()),
            "o_rel_rms": float(np.sqrt((diff ** 2).sum() / (o_ref ** 2).sum())),
            "lse_max_abs": float(np.abs(lg - lse_ref).max()),
        }
    return out


def run_reference(args, wl, world, rank):
    if rank != 0:
        return 0
    import numpy as np
    import oracle
    from exact_softmax_attention_04_b200 import synth
    oracle.build()
    q, k, v = synth.make_inputs(wl)
    pairs = synth.workload_pairs_per_head(wl)
    flops_per_row = 4.0 * wl.d * pairs / wl.n
    total = wl.B * wl.H * wl.n
    g = torch.Generator().manual_seed(3)
    # each step: a bounded sample sized so warmup + steps stay within ~2 minutes
    probe = torch.randint(0, total, (32,), generator=g).numpy()
    t0 = time.perf_counter()
    oracle.attn_rows_gqa(q, k, v, wl.scale, wl.causal, wl.window, probe, block=wl.block)
    per_row = max((time.perf_counter() - t0) / 32, 1e-6)
    budget = args.reference_seconds / max(1, args.steps + args.warmup)
    nrows = int(max(8, min(total, budget / per_row)))
    samples = [np.sort(torch.randint(0, total, (nrows,), generator=g).numpy())
               for _ in range(args.steps + args.warmup)]
    for i in range(args.warmup):
        oracle.attn_rows_gqa(q, k, v, wl.scale, wl.causal, wl.window, samples[i], block=wl.block)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle.attn_rows_gqa(q, k, v, wl.scale, wl.causal, wl.window, samples[args.warmup + i], block=wl.block)
    dt = time.perf_counter() - t0
    value = args.steps * nrows * flops_per_row / dt / 1e12
    sample = f"{nrows} random query rows per step (seed 3) of {wl.name}, fp64 oracle"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, world),
        "note": "the fp64 oracle on the host cores; no GPU and no L2 involved",
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_e2e(args, wl, q, k, v, o, lse, flops, dev, stream, world):
    """The metric through the host-buffer C-ABI entry point: pinned host
    inputs copied in, kernel, O and LSE copied out, all inside the timed
    region, every step."""
    import exact_softmax_attention_04_b200 as attn
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
    lh = torch.empty((wl.B, wl.H, wl.n), dtype=torch.float32, pin_memory=True)
    e2e_steps = max(3, min(args.steps, 20))
    for _ in range(2):
        attn.attn_fwd_host(qh, kh, vh, wl.scale, wl.causal, wl.window, out=oh, lse=lh, stream=stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        attn.attn_fwd_host(qh, kh, vh, wl.scale, wl.causal, wl.window, out=oh, lse=lh, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    st = attn.sync_status(stream)
    if st != attn.ATTN_OK:
        raise RuntimeError(attn.strerror(st))
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e = {"value": world * flops * e2e_steps / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
           "h2d_bytes_per_step": 3 * q.numel() * 2, "d2h_bytes_per_step": o.numel() * 2 + lse.numel() * 4,
           "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps}
    attn.host_staging_release()

    return e2e


def run_ours(args, wl, world, rank, local):
    import exact_softmax_attention_04_b200 as attn
    from exact_softmax_attention_04_b200 import synth

    dev = torch.device("cuda", local)
    q, k, v = synth.make_inputs(wl)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o = torch.empty_like(qd)
    lse = torch.empty((wl.B, wl.H, wl.n), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flops = synth.unmasked_flops(wl)

    def step():
        attn.attn_fwd(qd, kd, vd, wl.scale, wl.causal, wl.window, out=o, lse=lse, stream=stream,
                      block=wl.block)

    for _ in range(args.warmup):
        step()
    st = attn.sync_status(stream)
    if st != attn.ATTN_OK:
        raise RuntimeError(attn.strerror(st))

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local if not args.profile else -1) as clocks:
        if not args.profile:
            time.sleep(0.5)  # let the sampler start before the timed region
        wall0 = time.time()
        start_all = torch.cuda.Event(enable_timing=True)
        end_all = torch.cuda.Event(enable_timing=True)
        start_all.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        end_all.record(stream)
        torch.cuda.synchronize(dev)
        wall1 = time.time()
    barrier(world)
    st = attn.sync_status(stream)
    if st != attn.ATTN_OK:
        raise RuntimeError(attn.strerror(st))
    total_ms = max_over_ranks(start_all.elapsed_time(end_all), world)
    per_launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    ms_per_step = total_ms / args.steps
    value = replica_throughput(flops, args.steps, total_ms, world) / 1e12

    bf16_peak, hbm_peak, peak_src = peaks()
    achieved = flops / (per_launch_ms / 1e3) / 1e12
    if args.profile:
        if rank == 0:
            print(json.dumps({"profile_run": wl.name, "steps": args.steps, "warmup": args.warmup,
                              "kernel_ms_per_launch": per_launch_ms, "tflops": achieved}), flush=True)
        return 0

    # end to end through the host-buffer entry point: H2D of q,k,v, kernel,
    # D2H of o and lse, every step (that entry point takes equal head counts)
    e2e = None
    if wl.kv_heads == wl.H and wl.block == 0:
        e2e = run_e2e(args, wl, q, k, v, o, lse, flops, dev, stream, world)
    elif wl.block > 0:
        e2e = {"value": None, "unit": "TFLOP/s",
               "note": "block-local workload: the host-buffer entry point takes causal / window masks"}
    else:
        e2e = {"value": None, "unit": "TFLOP/s",
               "note": "grouped-query workload: the host-buffer entry point takes equal head counts"}

    traffic = recorded_traffic(wl.name)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": bf16_peak, "unit": "TFLOP/s",
                "frac": achieved / bf16_peak, "traffic": traffic,
                "peak_source": f"{peak_src} bf16 dense (burst)",
                "algorithmic_flops_per_launch": flops,
                "min_hbm_bytes_per_launch": 2 * q.numel() * 2 + 2 * k.numel() * 2 + lse.numel() * 4,
                "kernel_ms_per_launch": per_launch_ms}
    if traffic is not None:
        roofline["traffic_gbs"] = traffic / (per_launch_ms / 1e3) / 1e9

    if rank != 0:
        return 0
    sustained = None
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            sustained = float(json.load(fh)["bf16_tflops_sustained"])
    except (OSError, KeyError, ValueError):
        pass
    if sustained:
        roofline["frac_of_sustained_peak"] = achieved / sustained
        roofline["sustained_peak"] = sustained
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(wl, world),
        "pct_of_peak": 100.0 * value / world / bf16_peak,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "fwd_schedule": {"setting": args.schedule,
                         "form": attn.fwd_schedule_for(wl.n, wl.causal, wl.window, wl.block)},
        "clocks": clocks.summary(wall0, wall1),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_leg(wl, o, lse, target_s=args.cpu_seconds)
    print(json.dumps(line), flush=True)
    return 0


BWD_METRIC = "attention bwd TFLOP/s (10*d FLOPs per attended pair: five matmuls)"


def run_bwd(args, wl, world, rank, local):
    """Backward pass of one workload: O and LSE from attn_fwd (untimed), then
    attn_bwd timed as one step (its three launches). FLOPs: five matmuls of
    2*d per attended pair (S, dP, dV, dK, dQ)."""
    import numpy as np
    import exact_softmax_attention_04_b200 as attn
    from exact_softmax_attention_04_b200 import synth

    dev = torch.device("cuda", local)
    q, k, v = synth.make_inputs(wl)
    do = synth.make_dout(wl.B, wl.H, wl.n, wl.d, seed=wl.seed)
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    stream = torch.cuda.current_stream(dev)
    o, lse = attn.attn_fwd(qd, kd, vd, wl.scale, wl.causal, wl.window, stream=stream, block=wl.block)
    ws = torch.empty(attn.bwd_workspace_bytes(wl.B, wl.H, wl.n, wl.d), dtype=torch.uint8, device=dev)
    pairs = synth.workload_pairs_per_head(wl) * wl.B * wl.H
    flops = 10 * wl.d * pairs
    grads = None

    def step():
        nonlocal grads
        grads = attn.attn_bwd(qd, kd, vd, o, lse, dod, wl.scale, wl.causal, wl.window, workspace=ws, block=wl.block,
                              stream=stream)

    for _ in range(args.warmup):
        step()
    st = attn.sync_status(stream)
    if st != attn.ATTN_OK:
        raise RuntimeError(attn.strerror(st))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local if not args.profile else -1) as clocks:
        if not args.profile:
            time.sleep(0.5)
        wall0 = time.time()
        start_all, end_all = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start_all.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        end_all.record(stream)
        torch.cuda.synchronize(dev)
        wall1 = time.time()
    barrier(world)
    st = attn.sync_status(stream)
    if st != attn.ATTN_OK:
        raise RuntimeError(attn.strerror(st))
    total_ms = max_over_ranks(start_all.elapsed_time(end_all), world)
    per_step_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    achieved = flops / (per_step_ms / 1e3) / 1e12
    if args.profile:
        if rank == 0:
            print(json.dumps({"profile_run": wl.name, "pass": "bwd", "steps": args.steps,
                              "ms_per_step": per_step_ms, "tflops": achieved}), flush=True)
        return 0
    if rank != 0:
        return 0
    bf16_peak, _, peak_src = peaks()
    line = {
        "metric": BWD_METRIC, "value": replica_throughput(flops, args.steps, total_ms, world) / 1e12,
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**wl.describe(), "pass": "backward", "dout": "N(0,1), seed + 1",
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "no flush: inputs Q, K, V, O, dO exceed the 126 MB L2"
                         if 5 * q.numel() * 2 > 126e6 else "no flush: inputs fit in L2"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": bf16_peak, "unit": "TFLOP/s",
                     "frac": achieved / bf16_peak, "traffic": None,
                     "peak_source": f"{peak_src} bf16 dense (burst)",
                     "algorithmic_flops_per_launch": flops,
                     "note": "achieved over the whole attn_bwd call (prep, main and dQ conversion "
                             "kernels)"},
        "e2e": {"value": None, "unit": "TFLOP/s",
                "note": "the backward pass has no host-buffer entry point"},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks.summary(wall0, wall1),
    }
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        g = torch.Generator().manual_seed(2)
        total = wl.B * wl.H * wl.n
        flops_per_row = flops / total
        probe = torch.randint(0, total, (16,), generator=g).numpy()
        t0 = time.perf_counter()
        oracle.attn_bwd_rows_gqa(q, k, v, do, wl.scale, wl.causal, wl.window, probe, [], block=wl.block)
        dt = max(time.perf_counter() - t0, 1e-3)
        nrows = int(min(total, max(16, 16 * args.cpu_seconds / dt)))
        rows = np.sort(torch.randint(0, total, (nrows,), generator=g).numpy())
        t0 = time.perf_counter()
        dq_ref, _, _ = oracle.attn_bwd_rows_gqa(q, k, v, do, wl.scale, wl.causal, wl.window, rows, [], block=wl.block)
        dt = time.perf_counter() - t0
        dq_gpu = grads[0].view(-1, wl.d)[torch.as_tensor(rows, device=dev)].float().cpu().numpy()
        diff = dq_gpu - dq_ref
        line["cpu_baseline"] = {
            "value": nrows * flops_per_row / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "seconds": dt,
            "sample": f"dQ of {nrows} random query rows (seed 2) of {wl.name}, fp64 oracle, counted at "
                      "the backward's per-row share of FLOPs",
            "parity_vs_gpu": {"rows": nrows, "dq_rel_rms": float(np.sqrt((diff ** 2).sum() / (dq_ref ** 2).sum())),
                              "dq_max_abs": float(np.abs(diff).max())}}
    print(json.dumps(line), flush=True)
    return 0


DECODE_METRIC = "decode GB/s (cached K and V read once, plus q, O, LSE)"


def run_decode(args, wl, world, rank, local):
    """One decode step against rolling caches (attn_decode, or
    attn_decode_multi for several new tokens per sequence: split kernel and
    merge) per step, timed like the forward; the roofline is HBM bandwidth on
    the algorithmic bytes: the cached keys and values, read once, plus q, O
    and LSE."""
    import numpy as np
    import exact_softmax_attention_04_b200 as attn
    from exact_softmax_attention_04_b200 import synth

    dev = torch.device("cuda", local)
    multi = wl.T > 1 or wl.w != wl.W - 1
    if multi:
        q, kc, vc = synth.make_decode_multi(wl.B, wl.H, wl.Hkv, wl.T, wl.W, wl.d, seed=wl.seed, q_std=wl.q_std)
    else:
        q, kc, vc = synth.make_decode(wl.B, wl.H, wl.Hkv, wl.W, wl.d, seed=wl.seed, q_std=wl.q_std)
    qd, kd, vd = q.to(dev), kc.to(dev), vc.to(dev)
    pos = torch.full((wl.B,), wl.pos, dtype=torch.int32, device=dev)
    o = torch.empty_like(qd)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=dev)
    ws = torch.empty(attn.decode_multi_workspace_bytes(wl.B, wl.H, wl.Hkv, wl.T, wl.W, wl.w, wl.d),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    nbytes = 2 * wl.B * wl.Hkv * wl.keys * wl.d * 2 + 2 * q.numel() * 2 + lse.numel() * 4
    flops = 4 * wl.d * wl.attended * wl.B * wl.H
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        if multi:
            attn.attn_decode_multi(qd, kd, vd, pos, wl.w, wl.scale, out=o, lse=lse, workspace=ws, stream=stream)
        else:
            attn.attn_decode(qd, kd, vd, pos, wl.scale, out=o, lse=lse, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    st = attn.sync_status(stream)
    if st != attn.ATTN_OK:
        raise RuntimeError(attn.strerror(st))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local if not args.profile else -1) as clocks:
        if not args.profile:
            time.sleep(0.5)
        wall0 = time.time()
        for i in range(args.steps):
            flush.zero_()  # the caches (1.07 GB) exceed L2 anyway; flush so q/O do not linger
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        wall1 = time.time()
    barrier(world)
    st = attn.sync_status(stream)
    if st != attn.ATTN_OK:
        raise RuntimeError(attn.strerror(st))
    times = [a.elapsed_time(b) for a, b in ev]
    ms = max_over_ranks(statistics.mean(times), world)
    gbs = nbytes / (ms / 1e3) / 1e9
    if args.profile:
        if rank == 0:
            print(json.dumps({"profile_run": wl.name, "pass": "decode", "ms_per_step": ms, "gbs": gbs}),
                  flush=True)
        return 0
    if rank != 0:
        return 0
    _, hbm_peak, peak_src = peaks()
    line = {
        "metric": DECODE_METRIC, "value": world * gbs, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**wl.describe(), "pass": "decode",
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "flushed (256 MB write) before each timed step; the caches exceed L2"},
        "tflops": flops / (ms / 1e3) / 1e12,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": gbs / hbm_peak, "traffic": None, "peak_source": f"{peak_src} HBM copy",
                     "algorithmic_bytes_per_launch": nbytes,
                     "note": "achieved over the decode call (split kernel and merge kernel)"},
        "e2e": {"value": None, "unit": "GB/s", "note": "decode has no host-buffer entry point"},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks.summary(wall0, wall1),
    }
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        g = torch.Generator().manual_seed(2)
        nseq = max(1, min(wl.B, 4))
        t0 = time.perf_counter()
        if multi:
            o_ref, lse_ref = oracle.attn_decode_multi(q[:nseq], kc[:nseq], vc[:nseq], [wl.pos] * nseq, wl.scale,
                                                      wl.w)
        else:
            o_ref, lse_ref = oracle.attn_decode(q[:nseq], kc[:nseq], vc[:nseq], [wl.pos] * nseq, wl.scale)
        dt = time.perf_counter() - t0
        og = o[:nseq].float().cpu().numpy()
        line["cpu_baseline"] = {
            "value": nbytes * nseq / wl.B / dt / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle", "seconds": dt,
            "sample": f"the first {nseq} sequences of {wl.name}, fp64 oracle",
            "parity_vs_gpu": {"o_max_abs": float(np.abs(og - o_ref).max()),
                              "lse_max_abs": float(np.abs(lse[:nseq].cpu().numpy() - lse_ref).max())}}
    print(json.dumps(line), flush=True)
    return 0


def run_sweep(args):
    """Kernel time of every target workload (one line each): TFLOP/s on
    unmasked FLOPs, % of the measured peak and HBM GB/s on the minimum bytes
    (Q, K, V read once, O and LSE written once). Informational table; the
    parity of each of these workloads is checked by the test suite."""
    import exact_softmax_attention_04_b200 as attn
    from exact_softmax_attention_04_b200 import synth
    torch.cuda.set_device(0)
    bf16_peak, hbm_peak, peak_src = peaks()
    wls = [synth.SMALL_CAUSAL, synth.FULL_N8192, synth.WINDOW_N32768, synth.CAUSAL_N131072,
           synth.GQA_N8192, synth.SYM_N16384, synth.BLOCK_N16384] + synth.sweep()
    for wl in wls:
        q, k, v = synth.make_inputs(wl)
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        o = torch.empty_like(qd)
        lse = torch.empty((wl.B, wl.H, wl.n), dtype=torch.float32, device="cuda")
        flops = synth.unmasked_flops(wl)
        min_bytes = 4 * q.numel() * 2 + lse.numel() * 4
        # L2 flush buffer (256 MB) between timed launches for small problems
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        f = lambda: attn.attn_fwd(qd, kd, vd, wl.scale, wl.causal, wl.window, out=o, lse=lse, block=wl.block)
        for _ in range(args.warmup):
            f()
        st = attn.sync_status()
        times = []
        for _ in range(max(3, args.steps)):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            f()
            b.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        ms = statistics.median(times)
        tf = flops / (ms / 1e3) / 1e12
        print(json.dumps({"workload": wl.name, "schedule": args.schedule, "ms": ms, "tflops": tf,
                          "pct_of_peak": 100 * tf / bf16_peak, "hbm_gbs": min_bytes / (ms / 1e3) / 1e9,
                          "pct_of_hbm": 100 * min_bytes / (ms / 1e3) / 1e9 / hbm_peak,
                          "status": st, "l2": "flushed (256 MB write) before each timed launch",
                          "peak_source": peak_src}), flush=True)
        del qd, kd, vd, o, lse, flush
        torch.cuda.empty_cache()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--reference-seconds", type=float, default=120.0,
                    help="oracle work budget of the --impl reference arm (warm-up and timed steps)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="time every target workload (kernel only, median of --steps, L2 flushed)")
    ap.add_argument("--decode", action="store_true",
                    help="time one decode step against rolling caches; --workload defaults to "
                         "decode-B64-H32-Hkv8-W4096-d128-pos32767 (one new token, attn_decode); "
                         "decode-B64-H32-Hkv8-T4-W4096-w4092-d128-pos32767 takes four new tokens per "
                         "sequence (attn_decode_multi)")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward pass (attn_bwd) of --workload instead of the forward")
    ap.add_argument("--schedule", choices=["auto", "per_item", "persistent"], default="auto",
                    help="forward work schedule (attn_fwd_schedule): automatic by mask and length, or forced")
    ap.add_argument("--profile", action="store_true",
                    help="timed kernel launches only (no e2e, CPU baseline or clock sampling): "
                         "the command profiled under ncu")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.schedule != "auto" and args.impl == "ours":
        import exact_softmax_attention_04_b200 as attn
        attn.set_fwd_schedule({"per_item": attn.SCHEDULE_PER_ITEM,
                               "persistent": attn.SCHEDULE_PERSISTENT}[args.schedule])
    if args.sweep:
        return run_sweep(args)
    from exact_softmax_attention_04_b200 import synth
    if args.decode:
        name = args.workload if args.workload.startswith("decode-") else synth.DECODE_W4096.name
        dwl = synth.decode_by_name(name)
        if dwl is None:
            raise SystemExit(f"unknown decode workload {name}")
        world, rank, local = dist_setup(args.gpus)
        try:
            return run_decode(args, dwl, world, rank, local)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
    wl = synth.by_name(args.workload)
    if wl is None:
        raise SystemExit(f"unknown workload {args.workload}")
    if args.impl == "reference":
        # CPU-only arm: no process group; under torchrun only rank 0 works.
        return run_reference(args, wl, _env_int("WORLD_SIZE", 1), _env_int("RANK", 0))
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.bwd:
            return run_bwd(args, wl, world, rank, local)
        return run_ours(args, wl, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
