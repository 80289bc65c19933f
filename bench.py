#!/usr/bin/env python3
"""Benchmark of the packed low-bit GEMV on B200.

Headline workload: the Q1_0_g128 GEMV with a 4096x4096 sign-bit matrix and
M=1 (fp16 scale per 128 weights, bf16 activations, fp32 output).  Metric:
packed-weight bytes (sign bits + scales) streamed per second, and that rate
as a fraction of the measured HBM bandwidth.

A launch multiplies one activation vector x by R distinct 4096x4096 weight
matrices (y_r = W_r x) in one grouped call -- the way the projections that
read one hidden state are applied in a decode step.  The R weight sets total
more than 3x the L2 cache, so every matrix streams from HBM (no L2 flush is
needed).  One step is --launches-per-step such launches (one CUDA graph
replay each), so that the timed region of --steps steps lasts about a second
and the sampled clocks cover it; exactly --steps steps are timed with CUDA
events after --warmup untimed ones.  The other workloads (layer-shape sweep,
64-layer stack, INT4_G64, 2-bit MLP, ternary format, reply loop) are measured
after the headline and reported in the same line under "workloads"
(--headline-only skips them).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload q1_4096|q1_sweep|q1_stack|int4|q2_mlp|ternary|z80_reply]

With N > 1 (under torchrun) every weight matrix is split by rows across the
ranks (each rank holds N/G rows of each of R*G matrices, so the bytes per GPU
stay those of R matrices: weak scaling), x is replicated, each rank computes
its rows, and one NCCL all-gather per launch gives every rank all of y.  The
time is the max over ranks and the value the sum of all ranks' bytes.
`--impl reference` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "packed-weight GB/s streamed & % of B200 HBM peak (Q1_0_g128 GEMV, M=1)"
FALLBACK_HBM_GBS = 6650.0
KERNEL_DTYPE = "u8xs8->s32 (tensor core), f32 epilogue"
DEFAULT_LAUNCHES_PER_STEP = 600


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured burst bf16_tflops (cuBLAS)"
    return 1590.0, "fallback burst bf16"


def q1_bytes(N, K):
    return N * K // 8 + 2 * N * (K // 128)


def int4_bytes(N, K):
    return N * K // 2 + 2 * N * (K // 64)


def q1_4096_sets(l2_bytes):
    """Weight sets of the headline launch: at least 3x L2 of distinct bytes."""
    return max(8, -(-3 * l2_bytes // q1_bytes(4096, 4096)))


def rotation(per_bytes, l2_bytes):
    """Distinct weight sets that total at least 3x L2."""
    return max(4, -(-3 * l2_bytes // per_bytes))


def sweep_sets(N, K, l2_bytes):
    return min(256, rotation(q1_bytes(N, K), l2_bytes))


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, pw, smax, reasons = [], [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [c.strip() for c in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            try:
                pw.append(float(f[3]))
            except ValueError:
                pass
            for name, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "samples_under_load": 0}
        loaded = [s for s in sm if smax and s > 0.5 * smax]
        return {"sm_mhz": statistics.median(loaded or sm), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm), "samples_under_load": len(loaded),
                "power_w_median": statistics.median(pw) if pw else None}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    if n_gpus != world and rank == 0:
        print(f"note: --gpus {n_gpus} but WORLD_SIZE={world}", file=sys.stderr)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    """The largest of every rank's v (a device time): one all-reduce of a
    scalar, on the GPU under NCCL, on the host under gloo."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# CPU baseline: the oracle as it stands, single-threaded, on one pinned core
# ---------------------------------------------------------------------------

def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class PinnedCore:
    """Run the enclosed host code on one core (the lowest this process may
    use), restoring the previous affinity afterwards."""

    def __enter__(self):
        self.prev = None
        self.core = None
        if hasattr(os, "sched_getaffinity"):
            try:
                self.prev = os.sched_getaffinity(0)
                self.core = min(self.prev)
                os.sched_setaffinity(0, {self.core})
            except OSError:
                self.prev = None
        return self

    def __exit__(self, *exc):
        if self.prev is not None:
            os.sched_setaffinity(0, self.prev)
        return False


def cpu_info(pin):
    n = os.cpu_count() or 1
    return {"cores": 1, "nproc": n, "cpu_model": cpu_model(),
            "pinned_core": pin.core, "note": f"1 of {n} cores used"}


def _timed_loop(fn, seconds, max_reps):
    fn(0)  # build + warm
    t0 = time.perf_counter()
    reps = 0
    while reps < max_reps:
        fn(reps)
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    return reps, time.perf_counter() - t0


def oracle_q1_rate(seconds=10.0, rows=1024, max_reps=1000, N=4096, K=4096, seed_index=None, tag=7):
    """The oracle's Q1 GEMV on row samples of an N x K M=1 workload until
    `seconds` have passed, on one pinned core.  Returns (cpu_baseline dict
    with value in GB/s of packed weights)."""
    import oracle
    import synth
    seed = synth.SEED_BASE + (synth.W_Q1_4096 if seed_index is None else seed_index)
    bits = synth.q1_packed_random(seed, N, K, tag=tag)
    scales = synth.q1_scales(seed, N, K, tag=tag)
    x = synth.bf16_normal(seed, (1, K))
    rows = min(rows, N)

    def one(i):
        r0 = (i * rows) % (N - rows + 1)
        oracle.q1_gemv(bits[r0:r0 + rows], scales[r0:r0 + rows], x)

    with PinnedCore() as pin:
        reps, dt = _timed_loop(one, seconds, max_reps)
    v = reps * q1_bytes(rows, K) / dt / 1e9
    return dict(value=round(v, 5), unit="GB/s", kind="oracle",
                sample=f"{reps} oracle GEMVs of {rows} rows x {K} of the {N}x{K} M=1 workload ({dt:.1f} s)",
                **cpu_info(pin))


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle timed on the host, rank 0 only."""
    if rank != 0:
        return 0
    import oracle
    import synth
    seed = synth.SEED_BASE + synth.W_Q1_4096
    N, K, rows = 4096, 4096, 512
    bits = synth.q1_packed_random(seed, N, K, tag=7)
    scales = synth.q1_scales(seed, N, K, tag=7)
    x = synth.bf16_normal(seed, (1, K))
    oracle.q1_gemv(bits[:8], scales[:8], x)

    def step(i):
        r0 = (i * rows) % N
        oracle.q1_gemv(bits[r0:r0 + rows], scales[r0:r0 + rows], x)

    with PinnedCore() as pin:
        for i in range(args.warmup):
            step(i)
        t0 = time.perf_counter()
        for i in range(args.steps):
            step(args.warmup + i)
        dt = time.perf_counter() - t0
    per_step = q1_bytes(rows, K)
    value = per_step * args.steps / dt / 1e9
    sample = f"each step: oracle GEMV over {rows} of the 4096 rows (K=4096, M=1), single thread"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "Q1_0_g128 GEMV 4096x4096, M=1", "N": 4096, "K": 4096, "M": 1,
                   "rows_per_step": rows},
        "cpu_baseline": dict(value=round(value, 4), unit="GB/s", kind="oracle", sample=sample, **cpu_info(pin)),
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------

def _capture(step, stream):
    import torch
    with torch.cuda.stream(stream):
        step()
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    return graph


def _graph_time(step, stream, steps, warmup, min_ms=20.0):
    """Capture step() in a CUDA graph on `stream`; return ms per replay.
    At least `steps` replays are timed, and more when those take under
    min_ms, so that the launch of the first replay is a small part of it."""
    import torch
    graph = _capture(step, stream)
    # replay() launches on torch's current stream: the warm-up goes to
    # `stream` too, so that it has finished before the first timed replay
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            graph.replay()
    stream.synchronize()

    def timed(n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(n):
                graph.replay()
            e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1)

    n = max(1, steps)
    total = timed(n)
    if total < min_ms:
        n = min(100000, int(math.ceil(n * min_ms / max(total, 1e-3))))
        total = timed(n)
    del graph
    return total / n


def load_traffic(kernel):
    """dram bytes per launch from the committed ncu summary, if it was taken
    on the current kernel code (comments and layout do not count), else null."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        from decode_packed_bit_b200 import build as lb_build
        ent = d.get(kernel)
        if ent and ent.get("kernel_sha1") == lb_build.kernel_digest(ent.get("sources")):
            return ent.get("dram_bytes_per_launch")
    except Exception:
        return None
    return None


# ---------------------------------------------------------------------------
# the GPU arm: Q1 4096x4096 M=1
# ---------------------------------------------------------------------------

def run_q1_4096(args, world, rank, local):
    import torch
    import synth
    from decode_packed_bit_b200 import build as lb_build
    lb_build.build()
    from decode_packed_bit_b200 import lowbit as lb
    from decode_packed_bit_b200.shard import RowShardedGroup, row_shard

    N = K = 4096
    M = 1
    dev = torch.device("cuda", local)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per = q1_bytes(N, K)
    R = q1_4096_sets(l2)
    L = max(1, args.launches_per_step)
    seed = synth.SEED_BASE + synth.W_Q1_4096
    x = torch.from_numpy(synth.bf16_normal(seed, (M, K)).view(np.int16)).to(dev)
    stream = torch.cuda.Stream(device=dev)

    if world == 1:
        bits, scales = [], []
        for r in range(R):
            b, s = synth.torch_q1_layer(seed, N, K, r, dev)
            bits.append(b)
            scales.append(s)
        y = torch.empty((R, M, N), dtype=torch.float32, device=dev)
        ys = [y[r] for r in range(R)]
        need = lb.lowbit_q1g128_group_workspace_bytes(R, M, N, K)
        ws = torch.zeros(need, dtype=torch.uint8, device=dev) if need else None

        def launch():
            lb.lowbit_q1g128_gemv_group(bits, scales, x, ys, workspace=ws, stream=stream)
        calls_per_launch = 1 if need == 0 else 2   # one launch from x, else prepare + product
        bytes_launch = R * per
        gather = None
        out_host_shape = (R, M, N)
        out_dev = y
    else:
        # row-sharded: R*world matrices, rows [n0, n1) of each on this rank
        n0, n1 = row_shard(N, world, rank)
        Rt = R * world
        bits, scales = [], []
        for r in range(Rt):
            b, s = synth.torch_q1_layer(seed + 7919 * rank, n1 - n0, K, r, dev)
            bits.append(b)
            scales.append(s)
        grp = RowShardedGroup("q1", bits, scales, N, K, M, device=dev, stream=stream)

        def launch():
            grp.compute(x)
        calls_per_launch = 1 if grp.workspace is None else 2
        bytes_launch = Rt * q1_bytes(n1 - n0, K)
        gather = grp.gather
        out_host_shape = (grp.gathered.numel(),)
        out_dev = grp.gathered

    # one launch per graph replay; a step is L replays (plus, with several
    # ranks, the all-gather of each launch's outputs)
    graph = _capture(launch, stream)

    def run_steps(n):
        with torch.cuda.stream(stream):
            for _ in range(n):
                for _ in range(L):
                    graph.replay()
                    if gather is not None:
                        gather()

    # context only: 20 launches right after the capture, before the board
    # has run long enough to reach its power limit
    burst = None
    if world == 1:
        with torch.cuda.stream(stream):
            for _ in range(3):
                graph.replay()
            b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            b0.record(stream)
            for _ in range(20):
                graph.replay()
            b1.record(stream)
        b1.synchronize()
        bus = b0.elapsed_time(b1) * 1e3 / 20
        burst = {"launches": 20, "us_per_launch": round(bus, 3),
                 "gbs": round(bytes_launch / (bus * 1e-6) / 1e9, 1),
                 "frac": round(bytes_launch / (bus * 1e-6) / 1e9 / measured_peaks()[0], 4),
                 "note": "not the bench value: timed before the sustained region, too short for clock samples"}
    run_steps(args.warmup)
    stream.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
        run_steps(args.steps)
        with torch.cuda.stream(stream):
            e1.record(stream)
        e1.synchronize()
    torch.cuda.synchronize(dev)
    barrier(world)
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, world)
    launches = L * args.steps

    bytes_step = bytes_launch * L
    value = bytes_step * args.steps * world / (ms_max * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    achieved = bytes_launch * launches / (ms * 1e-3) / 1e9   # this rank's stream rate per launch

    # end to end through the C ABI with host buffers: per call, x in from
    # pinned host memory and all outputs back to pinned host memory, inside
    # the timed region.  One GPU: two buffer sets, so that the outputs of
    # call i travel to the host on a second stream while call i+1 runs (each
    # call waits for the copy that last read its buffer set).  Several ranks:
    # one call at a time (the all-gather owns the output buffer).
    x_host = x.cpu().pin_memory()
    # as many calls as the timed region above, so that both run for about as
    # long (and at the clocks the power limit leaves)
    e2e_calls = max(200, L * args.steps)
    if world == 1:
        x2 = torch.empty_like(x)
        y2 = torch.empty_like(y)
        ys2 = [y2[r] for r in range(R)]

        def launch2():
            lb.lowbit_q1g128_gemv_group(bits, scales, x2, ys2, workspace=ws, stream=stream)
        graph2 = _capture(launch2, stream)
        sets = [(graph, x, y), (graph2, x2, y2)]
        hosts = [torch.empty(out_host_shape, dtype=torch.float32).pin_memory() for _ in range(2)]
        y_host = hosts[0]
        copy_stream = torch.cuda.Stream(device=dev)  # outputs to the host
        in_stream = torch.cuda.Stream(device=dev)    # inputs from the host
        done = [torch.cuda.Event() for _ in range(2)]
        copied = [torch.cuda.Event() for _ in range(2)]
        loaded = [torch.cuda.Event() for _ in range(2)]

        start = torch.cuda.Event()

        def e2e_run(n):
            # the copy streams start after what `stream` has enqueued so far
            # (the start of the timed region)
            start.record(stream)
            in_stream.wait_event(start)
            copy_stream.wait_event(start)
            for i in range(n):
                b = i % 2
                g_b, x_b, y_b = sets[b]
                # x of call i comes in while call i-1 runs (x_b was last read by call i-2)
                with torch.cuda.stream(in_stream):
                    if i >= 2:
                        in_stream.wait_event(done[b])
                    x_b.copy_(x_host, non_blocking=True)
                    loaded[b].record(in_stream)
                with torch.cuda.stream(stream):
                    stream.wait_event(loaded[b])
                    if i >= 2:
                        stream.wait_event(copied[b])  # y_b of call i-2 has reached the host
                    g_b.replay()
                    done[b].record(stream)
                with torch.cuda.stream(copy_stream):
                    copy_stream.wait_event(done[b])
                    hosts[b].copy_(y_b.view(out_host_shape), non_blocking=True)
                    copied[b].record(copy_stream)
            stream.wait_event(copied[(n - 1) % 2])
            if n >= 2:
                stream.wait_event(copied[(n - 2) % 2])
        e2e_note = ("x in from pinned host, all outputs out, every call; two buffer sets: the inputs of "
                    "one call copy in and the outputs of the one before copy out on two more streams "
                    "while a call runs")
    else:
        y_host = torch.empty(out_host_shape, dtype=torch.float32).pin_memory()

        def e2e_run(n):
            with torch.cuda.stream(stream):
                for _ in range(n):
                    x.copy_(x_host, non_blocking=True)
                    graph.replay()
                    gather()
                    y_host.copy_(out_dev.view(out_host_shape), non_blocking=True)
        e2e_note = "one grouped call per step: x in from pinned host, all outputs out"

    e2e_run(3)
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
    e2e_run(e2e_calls)
    with torch.cuda.stream(stream):
        t1.record(stream)
    t1.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), world)
    e2e_value = bytes_launch * e2e_calls * world / (e2e_ms * 1e-3) / 1e9

    # the single-matrix call (lowbit_q1g128_gemv), R separate calls in one graph
    single = None
    if world == 1:
        yone = torch.empty((M, N), dtype=torch.float32, device=dev)
        nws1 = lb.lowbit_q1g128_workspace_bytes(M, N, K)
        ws1 = torch.zeros(nws1, dtype=torch.uint8, device=dev) if nws1 else None

        def singles():
            for r in range(R):
                lb.lowbit_q1g128_gemv(bits[r], scales[r], x, yone, workspace=ws1, stream=stream)
        sms = _graph_time(singles, stream, 20, 3)
        single = {"call": "lowbit_q1g128_gemv, one 4096x4096 matrix per call", "calls_per_replay": R,
                  "us_per_call": round(sms * 1e3 / R, 3), "gbs": round(R * per / (sms * 1e-3) / 1e9, 1),
                  "frac_of_peak": round(R * per / (sms * 1e-3) / 1e9 / peak, 4)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_q1_rate(seconds=args.cpu_seconds)

    traffic = load_traffic("q1_gemv")
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": KERNEL_DTYPE, "data": "synthetic",
        "config": {"workload": "Q1_0_g128 GEMV 4096x4096, M=1", "N": N, "K": K, "M": M,
                   "weight_sets_per_launch": R * world, "bytes_per_gemv": per,
                   "launches_per_step": L,
                   "l2": f"inputs larger than L2: {R} distinct weight sets per GPU, "
                         f"{bytes_launch / 2**20:.0f} MiB per launch vs {l2 / 2**20:.0f} MiB L2",
                   "step": f"{L} grouped launches of R GEMVs from x (one CUDA graph replay each)"
                           + (", each followed by an NCCL all-gather of y" if world > 1 else ""),
                   "parallelism": (f"row-shard x{world}: each GPU holds N/{world} rows of every matrix, "
                                   "all-gather of y") if world > 1 else "single GPU"},
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "algorithmic_bytes_per_launch": bytes_launch,
                     "us_per_launch": round(ms * 1e3 / launches, 3),
                     "kernel": "k_q1_m1_lean<1, 4096>",
                     "peak_source": f"{peak_kind} hbm_gbs (copy bandwidth)"},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
                "d2h_bytes_per_step": int(y_host.numel() * y_host.element_size()),
                "note": e2e_note},
        "single_call": single,
        "burst": burst,
        "gpu_launches": calls_per_launch * launches,
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
    }
    del graph
    if world == 1 and not args.headline_only and args.workload == "q1_4096":
        del bits, scales
        torch.cuda.empty_cache()
        line["workloads"] = run_other_workloads(args, world, rank, local)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the other workloads
# ---------------------------------------------------------------------------

def _emit(rank, line):
    if rank == 0:
        print(json.dumps(line), flush=True)


def _lib():
    from decode_packed_bit_b200 import build as lb_build
    lb_build.build()
    from decode_packed_bit_b200 import lowbit as lb
    return lb


def sweep_results(args, world, rank, local, cpu=True):
    """Q1_0_g128 at the three layer shapes and M in {1, 4, 16}, grouped."""
    import torch
    import synth
    lb = _lib()
    dev = torch.device("cuda", local)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    peak = measured_peaks()[0]
    seed = synth.SEED_BASE + synth.W_Q1_SWEEP + 1000 * rank
    results = []
    for (N, K) in synth.Q1_SWEEP_SHAPES:
        per = q1_bytes(N, K)
        R = sweep_sets(N, K, l2)
        mats = [synth.torch_q1_layer(seed, N, K, r, dev) for r in range(R)]
        for M in (1, 4, 16):
            x = torch.from_numpy(synth.bf16_normal(seed, (M, K), tag=M).view(np.int16)).to(dev)
            ys = [torch.empty((M, N), dtype=torch.float32, device=dev) for _ in range(R)]
            stream = torch.cuda.Stream(device=dev)
            need = lb.lowbit_q1g128_group_workspace_bytes(R, M, N, K)
            ws = torch.zeros(need, dtype=torch.uint8, device=dev) if need else None

            def step():
                lb.lowbit_q1g128_gemv_group([b for b, _ in mats], [s for _, s in mats], x, ys, workspace=ws,
                                            stream=stream)
            ms = max_over_ranks(_graph_time(step, stream, max(20, args.steps), args.warmup), world)
            gbs = R * per / (ms * 1e-3) / 1e9
            results.append({"N": N, "K": K, "M": M, "weight_sets": R, "gbs": round(gbs, 1),
                            "frac_of_peak": round(gbs / peak, 4), "us_per_gemv": round(ms * 1e3 / R, 3)})
        del mats
        torch.cuda.empty_cache()
    out = {"metric": "packed-weight GB/s, Q1_0_g128 layer-shape sweep (grouped launches)", "unit": "GB/s",
           "config": {"workload": "Q1_0_g128 (5120,5120),(17408,5120),(5120,17408) x M in {1,4,16}",
                      "l2": "inputs larger than L2 (rotating weight sets)"},
           "results": results}
    if cpu and rank == 0 and not args.no_cpu_baseline:
        base = []
        for (N, K) in synth.Q1_SWEEP_SHAPES:
            b = oracle_q1_rate(seconds=args.cpu_seconds / 3, rows=256, N=N, K=K,
                               seed_index=synth.W_Q1_SWEEP, tag=N + K)
            base.append({"N": N, "K": K, "M": 1, "gbs": b["value"], "sample": b["sample"]})
        out["cpu_baseline"] = {"kind": "oracle", "unit": "GB/s", "per_shape": base,
                               **{k: v for k, v in b.items() if k in ("cores", "nproc", "cpu_model",
                                                                      "pinned_core", "note")}}
    return out


def int4_results(args, world, rank, local, cpu=True):
    """INT4_G64 11008 x 4096 at M in {1, 32, 256}."""
    import torch
    import synth
    lb = _lib()
    dev = torch.device("cuda", local)
    N, K = synth.INT4_N, synth.INT4_K
    per = int4_bytes(N, K)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    peak = measured_peaks()[0]
    tpeak, tkind = measured_bf16_peak()
    R = rotation(per, l2)
    g = torch.Generator(device=dev)
    g.manual_seed(synth.SEED_BASE + synth.W_INT4 + 1000 * rank)
    qs = [torch.randint(0, 256, (N, K // 2), generator=g, device=dev, dtype=torch.uint8) for _ in range(R)]
    ss = [(torch.randn((N, K // 64), generator=g, device=dev) * 0.01).abs().half() for _ in range(R)]
    results = []
    for M in (1, 32, 256):
        x = torch.randn((M, K), generator=g, device=dev).bfloat16()
        y = torch.empty((R, M, N), dtype=torch.float32, device=dev)
        stream = torch.cuda.Stream(device=dev)

        def step():
            for r in range(R):
                lb.lowbit_int4g64_gemm(qs[r], ss[r], x, y[r], stream=stream)
        ms = max_over_ranks(_graph_time(step, stream, max(20, args.steps), args.warmup), world)
        tf = 2.0 * M * N * K * R / (ms * 1e-3) / 1e12
        res = {"M": M, "us_per_call": round(ms * 1e3 / R, 3),
               "weight_gbs": round(R * per / (ms * 1e-3) / 1e9, 1),
               "frac_of_hbm_peak": round(R * per / (ms * 1e-3) / 1e9 / peak, 4),
               "tflops": round(tf, 2), "frac_of_bf16_peak": round(tf / tpeak, 4)}
        if M <= 32:
            ys = [y[r] for r in range(R)]

            def gstep():
                lb.lowbit_int4g64_gemm_group(qs, ss, x, ys, stream=stream)
            gms = max_over_ranks(_graph_time(gstep, stream, max(20, args.steps), args.warmup), world)
            res["group_us"] = round(gms * 1e3, 3)
            res["group_weight_gbs"] = round(R * per / (gms * 1e-3) / 1e9, 1)
            res["group_frac_of_hbm_peak"] = round(R * per / (gms * 1e-3) / 1e9 / peak, 4)
        results.append(res)
    assert lb.lowbit_fault_flags() == 0
    out = {"metric": "INT4_G64 11008x4096: packed-weight GB/s (M=1, 32) and TFLOP/s (M=256)",
           "unit": "GB/s",
           "config": {"workload": "INT4_G64 N=11008 K=4096 M in {1,32,256}", "weight_sets": R,
                      "l2": "inputs larger than L2 (rotating weight sets)", "tensor_peak_source": tkind},
           "results": results}
    if cpu and rank == 0 and not args.no_cpu_baseline:
        import oracle
        q = synth.rng(synth.SEED_BASE + synth.W_INT4, 0).integers(0, 256, size=(N, K // 2), dtype=np.uint8)
        s = synth.int4_scales(synth.SEED_BASE + synth.W_INT4, N, K)
        rows = 128
        base = []
        for M in (1, 32, 256):
            xm = synth.bf16_normal(synth.SEED_BASE + synth.W_INT4, (M, K), tag=M)

            def one(i):
                r0 = (i * rows) % (N - rows)
                oracle.int4_gemv(q[r0:r0 + rows], s[r0:r0 + rows], xm)
            with PinnedCore() as pin:
                reps, dt = _timed_loop(one, args.cpu_seconds / 3, 100000)
            base.append({"M": M, "weight_gbs": round(reps * int4_bytes(rows, K) / dt / 1e9, 6),
                         "gflops": round(reps * 2.0 * M * rows * K / dt / 1e9, 4),
                         "sample": f"{reps} oracle products of {rows} rows x {K} at M={M} ({dt:.1f} s)"})
        out["cpu_baseline"] = {"kind": "oracle", "per_m": base, **cpu_info(pin)}
    del qs, ss
    torch.cuda.empty_cache()
    return out


def q2_results(args, world, rank, local, cpu=True):
    """The 2-bit integer MLP (256->192->128->40) over 1024 and 1M vectors."""
    import torch
    import synth
    lb = _lib()
    dev = torch.device("cuda", local)
    seed = synth.SEED_BASE + synth.W_Q2_MLP + 1000 * rank
    dims = synth.Q2_DIMS
    w = []
    for c in synth.q2_codes(seed, dims):
        codes = torch.from_numpy(c).to(dev)
        packed = torch.empty((c.shape[0], c.shape[1] // 4), dtype=torch.uint8, device=dev)
        lb.lowbit_pack("q2", codes, packed)
        w.append(packed)
    macs = sum(dims[i] * dims[i + 1] for i in range(len(dims) - 1))
    results = []
    for batch in (1024, 1 << 20):
        xb = synth.q2_inputs(seed, 1024)
        x = torch.from_numpy(np.tile(xb, (batch // 1024, 1))).to(dev)
        logits = torch.empty((batch, dims[-1]), dtype=torch.int16, device=dev)
        am = torch.empty((batch,), dtype=torch.int32, device=dev)
        stream = torch.cuda.Stream(device=dev)
        ms = max_over_ranks(_graph_time(lambda: lb.lowbit_q2_mlp_forward(w, dims, x, logits, am, stream=stream),
                                        stream, args.steps, args.warmup), world)
        results.append({"batch": batch, "us": round(ms * 1e3, 3), "vectors_per_s": round(batch / (ms * 1e-3), 1),
                        "gmac_per_s": round(batch * macs / (ms * 1e-3) / 1e9, 2)})
    out = {"metric": "2-bit integer MLP vectors/s (256->192->128->40)", "unit": "vectors/s",
           "dtype": "int16 wrap / int32",
           "config": {"workload": "Z80-style 2-bit MLP, 1024 and 1048576 vectors", "macs_per_vector": macs},
           "results": results}
    if cpu and rank == 0 and not args.no_cpu_baseline:
        import oracle
        packed = [oracle.pack("q2", c) for c in synth.q2_codes(synth.SEED_BASE + synth.W_Q2_MLP, dims)]
        xb = synth.q2_inputs(synth.SEED_BASE + synth.W_Q2_MLP, 1024)
        with PinnedCore() as pin:
            reps, dt = _timed_loop(lambda i: oracle.q2_mlp_forward(packed, dims, xb), args.cpu_seconds / 3, 1000)
        vps = reps * 1024 / dt
        out["cpu_baseline"] = {"kind": "oracle", "value": round(vps, 1), "unit": "vectors/s",
                               "gmac_per_s": round(vps * macs / 1e9, 4),
                               "sample": f"{reps} oracle passes over the 1024 vectors ({dt:.1f} s)", **cpu_info(pin)}
    return out


def stack_results(args, world, rank, local, Ms=(1, 8), cpu=True):
    """64-layer Q1_0_g128 projection stack, one decode step per replay."""
    import torch
    import synth
    _lib()
    from decode_packed_bit_b200.stack import Q1Layer, Q1Stack
    dev = torch.device("cuda", local)
    seed = synth.SEED_BASE + synth.W_Q1_STACK + 1000 * rank
    layers = [Q1Layer({name: synth.torch_q1_layer(seed, n, k, li * 16 + pi, dev)
                       for pi, (name, n, k) in enumerate(synth.STACK_PROJ)})
              for li in range(synth.STACK_LAYERS)]
    peak = measured_peaks()[0]
    results = []
    for M in Ms:
        st = Q1Stack(layers, synth.STACK_HIDDEN, synth.STACK_FFN, M, dev)
        st.x.copy_(torch.from_numpy(synth.bf16_normal(seed, (M, synth.STACK_HIDDEN)).view(np.int16))
                   .view(torch.bfloat16).to(dev))
        stream = torch.cuda.Stream(device=dev)
        fused = st.fused_supported()
        ms = _graph_time(lambda: (st.step_fused if fused else st.step)(stream=stream), stream, max(5, args.steps),
                         args.warmup)
        ms = max_over_ranks(ms, world)
        gbs = st.bytes_per_step / (ms * 1e-3) / 1e9
        results.append({"M": M, "tokens_per_s": round(M * 1e3 / ms, 2), "ms_per_step": round(ms, 4),
                        "weight_gbs": round(gbs, 1), "frac_of_hbm_peak": round(gbs / peak, 4),
                        "launches_per_step": 1 if fused else st.launches_per_step(),
                        "step": "one launch (lowbit_q1g128_stack_step)" if fused else
                                "one launch per product and per normalisation"})
        del st
    out = {"metric": "decode tokens/s through the 64-layer Q1 stack", "unit": "tokens/s",
           "config": {"workload": "Q1_0_g128 64-layer stack, hidden 5120, ffn 17408",
                      "bytes_per_step": 3350200320, "l2": "inputs larger than L2 (3.35 GB)"},
           "results": results}
    if cpu and rank == 0 and not args.no_cpu_baseline:
        b = oracle_q1_rate(seconds=args.cpu_seconds / 3, rows=64, N=17408, K=5120,
                           seed_index=synth.W_Q1_STACK, tag=3)
        steps_per_s = b["value"] * 1e9 / 3350200320
        out["cpu_baseline"] = dict(b, value=round(steps_per_s, 8), unit="tokens/s (M=1)",
                                   weight_gbs=b["value"],
                                   sample=b["sample"] + "; tokens/s = that weight rate / 3.35 GB per step "
                                                        "(extrapolated, not a timed full step)")
    del layers
    torch.cuda.empty_cache()
    return out


def t3_bytes(N, K):
    return N * 26 * (K // 128) + 2 * N * (K // 128)


def t3_results(args, world, rank, local, cpu=True):
    """Ternary weights (FP16 scale per 128, base-3 bytes), 4096 x 4096, M = 1:
    grouped launches over weight sets larger than L2, and single calls."""
    import torch
    import synth
    lb = _lib()
    dev = torch.device("cuda", local)
    N = K = 4096
    per = t3_bytes(N, K)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    peak = measured_peaks()[0]
    R = min(256, rotation(per, l2))
    seed = synth.SEED_BASE + synth.W_T3 + 1000 * rank
    mats = [synth.torch_t3_layer(seed, N, K, r, dev) for r in range(R)]
    w = [m for m, _ in mats]
    sc = [s for _, s in mats]
    x = torch.from_numpy(synth.bf16_normal(seed, (1, K)).view(np.int16)).to(dev)
    ys = [torch.empty((1, N), dtype=torch.float32, device=dev) for _ in range(R)]
    stream = torch.cuda.Stream(device=dev)
    gms = max_over_ranks(_graph_time(lambda: lb.lowbit_t3g128_gemv_group(w, sc, x, ys, stream=stream), stream,
                                     max(20, args.steps), args.warmup), world)
    sms_ = max_over_ranks(_graph_time(lambda: [lb.lowbit_t3g128_gemv(w[r], sc[r], x, ys[r], stream=stream)
                                               for r in range(R)], stream, max(20, args.steps), args.warmup), world)
    g_gbs = R * per / (gms * 1e-3) / 1e9
    s_gbs = R * per / (sms_ * 1e-3) / 1e9
    out = {"metric": "packed-weight GB/s, ternary (FP16 scale per 128, 1.75 bits per weight) 4096x4096 M=1",
           "unit": "GB/s", "config": {"workload": "ternary 4096x4096, M=1", "weight_sets": R, "bytes_per_gemv": per,
                                      "l2": "inputs larger than L2 (rotating weight sets)"},
           "results": [{"call": "lowbit_t3g128_gemv_group (one launch)", "us": round(gms * 1e3, 3),
                        "gbs": round(g_gbs, 1), "frac_of_hbm_peak": round(g_gbs / peak, 4)},
                       {"call": "lowbit_t3g128_gemv, one call per matrix", "us_per_call": round(sms_ * 1e3 / R, 3),
                        "gbs": round(s_gbs, 1), "frac_of_hbm_peak": round(s_gbs / peak, 4)}]}
    if cpu and rank == 0 and not args.no_cpu_baseline:
        import oracle
        pk = mats[0][0][:1024].cpu().numpy()
        sk = mats[0][1][:1024].cpu().view(torch.int16).numpy().view(np.uint16)
        xh = synth.bf16_normal(seed, (1, K))
        rows = 256

        def one(i):
            r0 = (i * rows) % (1024 - rows + 1)
            oracle.t3_gemv(pk[r0:r0 + rows], sk[r0:r0 + rows], xh)
        with PinnedCore() as pin:
            reps, dt = _timed_loop(one, args.cpu_seconds / 3, 100000)
        out["cpu_baseline"] = {"kind": "oracle", "value": round(reps * t3_bytes(rows, K) / dt / 1e9, 6), "unit": "GB/s",
                               "sample": f"{reps} oracle products of {rows} rows x {K} ({dt:.1f} s)", **cpu_info(pin)}
    del mats, w, sc
    torch.cuda.empty_cache()
    return out


def z80_results(args, world, rank, local, cpu=True):
    """The Z80-uLM reply loop: 4096 conversations, up to 32 characters each,
    on the 256->192->128->40 network."""
    import torch
    import synth
    lb = _lib()
    dev = torch.device("cuda", local)
    seed = synth.SEED_BASE + synth.W_Q2_MLP + 1000 * rank
    dims = synth.Q2_DIMS
    w = []
    for c in synth.q2_codes(seed, dims):
        codes = torch.from_numpy(c).to(dev)
        packed = torch.empty((c.shape[0], c.shape[1] // 4), dtype=torch.uint8, device=dev)
        lb.lowbit_pack("q2", codes, packed)
        w.append(packed)
    batch, max_new, qlen = 4096, 32, 32
    q = torch.from_numpy(synth.chat_queries(seed, batch, qlen)).to(dev)
    reply = torch.empty((batch, max_new), dtype=torch.uint8, device=dev)
    lens = torch.empty((batch,), dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    ms = max_over_ranks(_graph_time(lambda: lb.lowbit_z80_generate(w, dims, q, synth.CHARSET, reply, lens,
                                                                   stream=stream), stream, args.steps, args.warmup),
                        world)
    chars = int(lens.sum().item())
    macs = sum(dims[i] * dims[i + 1] for i in range(len(dims) - 1))
    out = {"metric": "Z80-uLM reply loop: characters/s (4096 conversations, up to 32 characters)",
           "unit": "characters/s",
           "config": {"workload": "reply loop, 256->192->128->40 2-bit network, 4096 prompts of 1-5 words",
                      "max_new": max_new, "characters_generated": chars},
           "results": [{"us_per_batch": round(ms * 1e3, 3), "characters_per_s": round(chars / (ms * 1e-3), 1),
                        "conversations_per_s": round(batch / (ms * 1e-3), 1),
                        "gmac_per_s": round(chars * macs / (ms * 1e-3) / 1e9, 2)}]}
    if cpu and rank == 0 and not args.no_cpu_baseline:
        import oracle
        packed = [oracle.pack("q2", c) for c in synth.q2_codes(synth.SEED_BASE + synth.W_Q2_MLP, dims)]
        qh = synth.chat_queries(synth.SEED_BASE + synth.W_Q2_MLP, 64, qlen)
        with PinnedCore() as pin:
            t0 = time.perf_counter()
            n_done = 0
            total_chars = 0
            while n_done < 64:
                _, ln = oracle.z80_generate(packed, dims, qh[n_done:n_done + 8], np.frombuffer(synth.CHARSET, np.uint8),
                                            max_new)
                total_chars += int(ln.sum())
                n_done += 8
                if time.perf_counter() - t0 > args.cpu_seconds / 3:
                    break
            dt = time.perf_counter() - t0
        out["cpu_baseline"] = {"kind": "oracle", "value": round(total_chars / dt, 2), "unit": "characters/s",
                               "sample": f"{n_done} oracle replies ({total_chars} characters, {dt:.1f} s)",
                               **cpu_info(pin)}
    return out


def run_other_workloads(args, world, rank, local):
    out = {}
    for name, fn in (("q1_sweep", sweep_results), ("int4", int4_results), ("q2_mlp", q2_results),
                     ("q1_stack", stack_results), ("ternary", t3_results), ("z80_reply", z80_results)):
        try:
            out[name] = fn(args, world, rank, local)
        except Exception as e:  # a failing side workload must not hide the headline
            out[name] = {"error": f"{type(e).__name__}: {e}"}
    return out


def _single(fn, key):
    def run(args, world, rank, local):
        line = fn(args, world, rank, local)
        line.update({"n_gpus": world, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
                     "data": "synthetic", "scaling": "weak"})
        _emit(rank, line)
        return 0
    return run


OTHER_WORKLOADS = {"q1_stack": _single(lambda a, w, r, l: stack_results(a, w, r, l, Ms=(a.m,)), "q1_stack"),
                   "q1_sweep": _single(sweep_results, "q1_sweep"), "int4": _single(int4_results, "int4"),
                   "q2_mlp": _single(q2_results, "q2_mlp"), "ternary": _single(t3_results, "ternary"),
                   "z80_reply": _single(z80_results, "z80_reply")}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="q1_4096",
                    choices=["q1_4096", "q1_sweep", "q1_stack", "int4", "q2_mlp", "ternary", "z80_reply"])
    ap.add_argument("--launches-per-step", type=int, default=DEFAULT_LAUNCHES_PER_STEP,
                    help="grouped launches per headline step")
    ap.add_argument("--headline-only", action="store_true", help="skip the other workloads")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--m", type=int, default=1, help="batch rows for --workload q1_stack")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        return run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)

    world, rank, local = dist_setup(args.gpus)
    try:
        if args.workload == "q1_4096":
            return run_q1_4096(args, world, rank, local)
        return OTHER_WORKLOADS[args.workload](args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
