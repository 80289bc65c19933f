#!/usr/bin/env python3
"""Benchmark of the packed low-bit GEMV on B200.

Headline workload: the Q1_0_g128 GEMV with a 4096x4096 sign-bit matrix and
M=1 (fp16 scale per 128 weights, bf16 activations, fp32 output).  Metric:
packed-weight bytes (sign bits + scales) streamed per second, and that rate
as a fraction of the measured HBM bandwidth.

One step = one activation vector x prepared once, then multiplied by R
distinct 4096x4096 weight matrices (y_r = W_r x) in one grouped launch --
the way the projections that read one hidden state are applied in a decode
step.  The R weight sets total more than 3x the L2 cache, so every matrix
streams from HBM (no L2 flush is needed).  The step is one CUDA graph
replay on the launching stream; it is timed with CUDA events over exactly
--steps replays after --warmup untimed ones.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload q1_4096|q1_sweep|q1_stack|int4|q2_mlp]

With N > 1 (under torchrun) every rank runs the same workload on its own GPU
with its own weights (independent problems, no collective on the data path);
the time is the max over ranks and the value the sum of all ranks' bytes.
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


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def q1_bytes(N, K):
    return N * K // 8 + 2 * N * (K // 128)


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

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, smax, reasons = [], None, set()
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
            for name, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [s for s in sm if smax and s > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


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
# CPU baseline: the oracle as it stands, single-threaded, bounded sample
# ---------------------------------------------------------------------------

def oracle_q1_rate(seconds=10.0, rows=1024, max_reps=1000):
    """Time the oracle's Q1 GEMV on row samples of the 4096x4096 workload
    until `seconds` have passed.  Returns (GB/s of packed weights, sample)."""
    import oracle
    import synth
    seed = synth.SEED_BASE + synth.W_Q1_4096
    N, K = 4096, 4096
    bits = synth.q1_packed_random(seed, N, K, tag=7)
    scales = synth.q1_scales(seed, N, K, tag=7)
    x = synth.bf16_normal(seed, (1, K))
    oracle.q1_gemv(bits[:8], scales[:8], x)           # build + warm
    t0 = time.perf_counter()
    reps, done = 0, 0
    while reps < max_reps:
        r0 = (reps * rows) % N
        oracle.q1_gemv(bits[r0:r0 + rows], scales[r0:r0 + rows], x)
        reps += 1
        done += q1_bytes(rows, K)
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    sample = f"{reps} oracle GEMVs of {rows} rows x {K} of the 4096x4096 M=1 workload ({dt:.1f} s)"
    return done / dt / 1e9, sample


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
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the GPU arm: Q1 4096x4096 M=1
# ---------------------------------------------------------------------------

def run_q1_4096(args, world, rank, local):
    import torch
    import synth
    from decode_packed_bit_b200 import build as lb_build
    lb_build.build()
    from decode_packed_bit_b200 import lowbit as lb

    N = K = 4096
    M = 1
    dev = torch.device("cuda", local)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per = q1_bytes(N, K)
    R = max(8, -(-3 * l2 // per))                      # >= 3x L2 of distinct weights
    seed = synth.SEED_BASE + synth.W_Q1_4096 + 1000 * rank
    bits, scales = [], []
    for r in range(R):
        b, s = synth.torch_q1_layer(seed, N, K, r, dev)
        bits.append(b)
        scales.append(s)
    x = torch.from_numpy(synth.bf16_normal(seed, (M, K)).view(np.int16)).to(dev)
    y = torch.empty((R, M, N), dtype=torch.float32, device=dev)
    need = lb.lowbit_q1g128_group_workspace_bytes(R, M, N, K)
    ws = torch.zeros(need, dtype=torch.uint8, device=dev) if need else None
    stream = torch.cuda.Stream(device=dev)

    ys = [y[r] for r in range(R)]

    def step():
        lb.lowbit_q1g128_gemv_group(bits, scales, x, ys, workspace=ws, stream=stream)

    launches_per_step = 1 if need == 0 else 2  # one launch from x, else prepare + product
    # eager warm-up (also loads the module), then capture one step in a graph
    with torch.cuda.stream(stream):
        step()
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    for _ in range(args.warmup):
        graph.replay()
    stream.synchronize()

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
        e1.synchronize()
    torch.cuda.synchronize(dev)
    barrier(world)
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, world)

    bytes_step = R * per
    value = bytes_step * args.steps * world / (ms_max * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    achieved = bytes_step * args.steps / (ms * 1e-3) / 1e9   # this rank's stream rate

    # end to end through the C ABI with host buffers: x in from pinned host
    # memory, all R outputs back to pinned host memory, inside the timed region
    x_host = x.cpu().pin_memory()
    y_host = torch.empty((R, M, N), dtype=torch.float32).pin_memory()
    for _ in range(2):
        with torch.cuda.stream(stream):
            x.copy_(x_host, non_blocking=True)
            graph.replay()
            y_host.copy_(y, non_blocking=True)
        stream.synchronize()
    barrier(world)
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 50))
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(e2e_steps):
            x.copy_(x_host, non_blocking=True)
            graph.replay()
            y_host.copy_(y, non_blocking=True)
        t1.record(stream)
    t1.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), world)
    e2e_value = bytes_step * e2e_steps * world / (e2e_ms * 1e-3) / 1e9

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample = oracle_q1_rate(seconds=args.cpu_seconds)
        cpu = {"value": round(v, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample}

    traffic = load_traffic("q1_gemv")
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": KERNEL_DTYPE, "data": "synthetic",
        "config": {"workload": "Q1_0_g128 GEMV 4096x4096, M=1", "N": N, "K": K, "M": M,
                   "weight_sets_per_step": R, "bytes_per_gemv": per,
                   "l2": f"inputs larger than L2: {R} distinct weight sets, {R * per / 2**20:.0f} MiB "
                         f"per step vs {l2 / 2**20:.0f} MiB L2",
                   "step": ("1 grouped launch of R GEMVs from x" if launches_per_step == 1 else
                            "1 activation prepare + 1 grouped launch of R GEMVs") + ", one CUDA graph",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_source": f"{peak_kind} hbm_gbs (copy bandwidth)"},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
                "d2h_bytes_per_step": int(y_host.numel() * y_host.element_size())},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    return 0


# ---------------------------------------------------------------------------
# the other workloads (one JSON line each, with their own metric)
# ---------------------------------------------------------------------------

def _graph_time(step, stream, steps, warmup, min_ms=20.0):
    """Capture step() in a CUDA graph on `stream`; return ms per replay.
    At least `steps` replays are timed, and more when those take under
    min_ms, so that the launch of the first replay is a small part of it."""
    import torch
    with torch.cuda.stream(stream):
        step()
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
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


def _emit(rank, line):
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_q1_stack(args, world, rank, local):
    """64-layer Q1_0_g128 projection stack, one decode step per replay."""
    import torch
    import synth
    from decode_packed_bit_b200 import build as lb_build
    lb_build.build()
    from decode_packed_bit_b200.stack import Q1Layer, Q1Stack
    dev = torch.device("cuda", local)
    seed = synth.SEED_BASE + synth.W_Q1_STACK + 1000 * rank
    layers = [Q1Layer({name: synth.torch_q1_layer(seed, n, k, li * 16 + pi, dev)
                       for pi, (name, n, k) in enumerate(synth.STACK_PROJ)})
              for li in range(synth.STACK_LAYERS)]
    M = args.m
    st = Q1Stack(layers, synth.STACK_HIDDEN, synth.STACK_FFN, M, dev)
    st.x.copy_(torch.from_numpy(synth.bf16_normal(seed, (M, synth.STACK_HIDDEN)).view(np.int16))
               .view(torch.bfloat16).to(dev))
    stream = torch.cuda.Stream(device=dev)
    fused = st.fused_supported()  # M = 1: the whole step is one launch
    with ClockSampler(local) as clk:
        ms = _graph_time(lambda: (st.step_fused if fused else st.step)(stream=stream), stream, args.steps, args.warmup)
    ms = max_over_ranks(ms, world)
    gbs = st.bytes_per_step / (ms * 1e-3) / 1e9
    _emit(rank, {"metric": f"decode tokens/s through the 64-layer Q1 stack (M={M})",
                 "value": round(M * world * 1e3 / ms, 2), "unit": "tokens/s", "n_gpus": world,
                 "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
                 "higher_is_better": True, "scaling": "weak", "dtype": KERNEL_DTYPE if M == 1 else "bf16xsign->f32",
                 "data": "synthetic",
                 "config": {"workload": "Q1_0_g128 64-layer stack, hidden 5120, ffn 17408", "M": M,
                            "bytes_per_step": st.bytes_per_step, "l2": "inputs larger than L2 (3.35 GB)"},
                 "weight_gbs": round(gbs, 1), "pct_of_hbm_peak": round(100 * gbs / measured_peaks()[0], 2),
                 "gpu_launches": (1 if fused else st.launches_per_step()) * args.steps,
                 "step": "one cooperative launch (lowbit_q1g128_stack_step)" if fused else "one launch per product "
                         "and per normalisation", "clocks": clk.summary()})
    return 0


def _rotation(per_bytes, l2):
    return max(4, -(-3 * l2 // per_bytes))


def run_q1_sweep(args, world, rank, local):
    """Q1_0_g128 at the three layer shapes and M in {1, 4, 16}."""
    import torch
    import synth
    from decode_packed_bit_b200 import build as lb_build
    lb_build.build()
    from decode_packed_bit_b200 import lowbit as lb
    dev = torch.device("cuda", local)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    seed = synth.SEED_BASE + synth.W_Q1_SWEEP + 1000 * rank
    results = []
    for (N, K) in synth.Q1_SWEEP_SHAPES:
        per = q1_bytes(N, K)
        R = min(256, _rotation(per, l2))
        mats = [synth.torch_q1_layer(seed, N, K, r, dev) for r in range(R)]
        for M in (1, 4, 16):
            x = torch.from_numpy(synth.bf16_normal(seed, (M, K), tag=M).view(np.int16)).to(dev)
            ys = [torch.empty((M, N), dtype=torch.float32, device=dev) for _ in range(R)]
            stream = torch.cuda.Stream(device=dev)
            if M == 1:
                need = lb.lowbit_q1g128_group_workspace_bytes(R, 1, N, K)
                ws = torch.zeros(need, dtype=torch.uint8, device=dev) if need else None

                def step():
                    lb.lowbit_q1g128_gemv_group([b for b, _ in mats], [s for _, s in mats], x, ys, workspace=ws,
                                                stream=stream)
            else:
                need = lb.lowbit_q1g128_group_workspace_bytes(R, M, N, K)
                ws = torch.zeros(need, dtype=torch.uint8, device=dev) if need else None

                def step():
                    lb.lowbit_q1g128_gemv_group([b for b, _ in mats], [s for _, s in mats], x, ys, workspace=ws,
                                                stream=stream)
            ms = max_over_ranks(_graph_time(step, stream, max(20, args.steps), args.warmup), world)
            results.append({"N": N, "K": K, "M": M, "weight_sets": R,
                            "gbs": round(R * per / (ms * 1e-3) / 1e9, 1),
                            "us_per_gemv": round(ms * 1e3 / R, 3)})
        del mats
    _emit(rank, {"metric": "packed-weight GB/s, Q1_0_g128 layer-shape sweep", "unit": "GB/s",
                 "value": results[0]["gbs"], "n_gpus": world, "higher_is_better": True, "data": "synthetic",
                 "config": {"workload": "Q1_0_g128 (5120,5120),(17408,5120),(5120,17408) x M in {1,4,16}",
                            "l2": "inputs larger than L2 (rotating weight sets)"},
                 "results": results})
    return 0


def run_int4(args, world, rank, local):
    """INT4_G64 11008 x 4096 at M in {1, 32, 256}."""
    import torch
    import synth
    from decode_packed_bit_b200 import build as lb_build
    lb_build.build()
    from decode_packed_bit_b200 import lowbit as lb
    dev = torch.device("cuda", local)
    N, K = synth.INT4_N, synth.INT4_K
    per = N * K // 2 + 2 * N * (K // 64)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = _rotation(per, l2)
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
        res = {"M": M, "us_per_call": round(ms * 1e3 / R, 3),
               "weight_gbs": round(R * per / (ms * 1e-3) / 1e9, 1),
               "tflops": round(2.0 * M * N * K * R / (ms * 1e-3) / 1e12, 2)}
        if M <= 32:
            # the R weight sets read one x: one grouped launch
            ys = [y[r] for r in range(R)]

            def gstep():
                lb.lowbit_int4g64_gemm_group(qs, ss, x, ys, stream=stream)
            gms = max_over_ranks(_graph_time(gstep, stream, max(20, args.steps), args.warmup), world)
            res["group_us"] = round(gms * 1e3, 3)
            res["group_weight_gbs"] = round(R * per / (gms * 1e-3) / 1e9, 1)
        results.append(res)
    assert lb.lowbit_fault_flags() == 0
    _emit(rank, {"metric": "INT4_G64 11008x4096: packed-weight GB/s (M=1) and TFLOP/s (M=32, 256)",
                 "unit": "GB/s", "value": results[0]["weight_gbs"], "n_gpus": world, "higher_is_better": True,
                 "data": "synthetic",
                 "config": {"workload": "INT4_G64 N=11008 K=4096 M in {1,32,256}", "weight_sets": R,
                            "l2": "inputs larger than L2 (rotating weight sets)"},
                 "results": results})
    return 0


def run_q2_mlp(args, world, rank, local):
    """The 2-bit integer MLP (256->192->128->40) over 1024 and 1M vectors."""
    import torch
    import synth
    from decode_packed_bit_b200 import build as lb_build
    lb_build.build()
    from decode_packed_bit_b200 import lowbit as lb
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
    _emit(rank, {"metric": "2-bit integer MLP vectors/s (256->192->128->40)", "unit": "vectors/s",
                 "value": results[0]["vectors_per_s"], "n_gpus": world, "higher_is_better": True,
                 "dtype": "int16 wrap / int32", "data": "synthetic",
                 "config": {"workload": "Z80-style 2-bit MLP, 1024 and 1048576 vectors", "macs_per_vector": macs},
                 "results": results})
    return 0


OTHER_WORKLOADS = {"q1_stack": run_q1_stack, "q1_sweep": run_q1_sweep, "int4": run_int4, "q2_mlp": run_q2_mlp}


KERNEL_DTYPE = "u8xs8->s32 (tensor core), f32 epilogue"


def load_traffic(kernel):
    """dram bytes per launch from the committed ncu summary, if it matches
    the current kernel sources (else null)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        from decode_packed_bit_b200 import build as lb_build
        ent = d.get(kernel)
        if ent and ent.get("sources_sha1") == lb_build.digest():
            return ent.get("dram_bytes_per_launch")
    except Exception:
        return None
    return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="q1_4096",
                    choices=["q1_4096", "q1_sweep", "q1_stack", "int4", "q2_mlp"])
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
