"""Benchmark of the persistent op-queue runtime on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl reference]

A step is one pass of a whole op stream (default: the 20,000-op mixed fp32
elementwise DAG) through the persistent kernel. Each step's ops are published
before its kernel launches (GPUOS_START_DRAIN: the kernel exits when the
stream drained), and the next step's ops are written into the ring while the
current kernel runs. The timed region holds exactly K steps, bracketed by a
barrier and a device synchronisation, timed with CUDA events on the runtime's
stream; with N GPUs every rank runs its own replica (weak scaling) and the
slowest rank's time counts.

Rank 0 prints one JSON line. `--impl reference` times the CPU oracle instead
(single thread, bounded sample per step).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ops/sec and µs/op via persistent queue; aggregate HBM GB/s vs B200 peak"
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 256 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0

WORKLOAD_NAMES = {
    1: "dependent chain of 1,000 fused relu(a*x+b) ops on 4,096 fp32 (seed 0)",
    2: "20,000 mixed fp32 elementwise ops (add, mul, gelu, scale, relu-affine), n ~ logU[256, 65,536], "
       "random DAG with 0-2 deps per op (seed 1)",
    3: "bf16 decode non-GEMM stream: 32 layers x 16 ops (RMSNorm 2048, rotary 16x128, softmax 16x1024, "
       "SiLU*mul 5632, residual adds), layer-sequential deps; one step of 512 ops x 100 (seed 2)",
    4: "100,000 ops from 64 interleaved request chains: softmax [1-8, 128-4096], LayerNorm [1-8, 1024], "
       "adds (seed 3)",
    5: "256 large ops: fused relu(a*x+b) on 64 Mi fp32 (dependent ping-pong chain) and row sum/max of "
       "[8192, 8192] fp32 (seed 4)",
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "persistent_execution_b200", "csrc")
    for name in sorted(os.listdir(d)):
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(config: int):
    """DRAM bytes per launch of the persistent kernel from a committed ncu
    summary, if it was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", f"persistent_kernel_config{config}_traffic.json")
    try:
        with open(p) as f:
            j = json.load(f)
        if j.get("kernel_source_hash") == kernel_source_hash():
            return float(j["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class Clocks:
    """SM clock and throttle reasons sampled through NVML every 2 ms during the
    timed region (nvidia-smi cannot sample a region of tens of milliseconds)."""

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.max_mhz = None
        self._stop = None
        self._t = None

    def __enter__(self):
        import threading
        try:
            import pynvml as N
            N.nvmlInit()
            h = N.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM))
        except Exception:
            return self
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append((N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM),
                                         N.nvmlDeviceGetCurrentClocksEventReasons(h)))
                except Exception:
                    break
                self._stop.wait(0.002)

        self._t = threading.Thread(target=run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._t.join(timeout=2)

    def summary(self) -> dict:
        names = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
                 0x4: "sw_power_cap"}
        reasons = set()
        for _, r in self.samples:
            for bit, n in names.items():
                if r & bit:
                    reasons.add(n)
        sm = [c for c, _ in self.samples]
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvml, 2 ms"}


def setup_dist(args):
    from persistent_execution_b200 import replicas as R
    r = R.init("gloo" if args.impl == "reference" else "nccl")
    return r.rank, r.world, r.local


# ---------------------------------------------------------------- reference arm (CPU oracle)
def bench_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    from persistent_execution_b200 import workloads as W
    w = W.make(args.config)
    sample = args.ref_sample or {1: 1000, 2: 2000, 3: 512, 4: 2000, 5: 4}[args.config]
    idx = np.arange(min(sample, w.n_ops))
    orc = oracle.to_orc(w, idx)
    a32 = w.arena_f32.copy()
    a16 = w.arena_bf16.copy()
    for _ in range(args.warmup):
        oracle.run_ops(orc, a32, a16)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.run_ops(orc, a32, a16)
    dt = time.perf_counter() - t0
    v = args.steps * len(idx) / dt
    desc = f"first {len(idx)} ops of the stream per step, single thread"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "ops/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD_NAMES[args.config], "sample": desc},
        "cpu_baseline": {"value": v, "unit": "ops/s", "cores": 1, "kind": "oracle", "sample": desc},
        "e2e": {"value": v, "unit": "ops/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def cpu_baseline(w, config):
    import oracle
    budget = 15.0
    n = {1: 1000, 2: 20000, 3: 512 * 10, 4: 20000, 5: 4}[config]
    idx = np.arange(min(n, w.n_ops))
    orc = oracle.to_orc(w, idx)
    a32 = w.arena_f32.copy()
    a16 = w.arena_bf16.copy()
    t0 = time.perf_counter()
    done = 0
    for s in range(0, len(idx), 256):
        oracle.run_ops(orc[s:s + 256], a32, a16)
        done = min(s + 256, len(idx))
        if time.perf_counter() - t0 > budget:
            break
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": "ops/s", "cores": 1, "kind": "oracle",
            "sample": f"first {done} ops of one step of the same stream, single thread, {dt:.1f} s"}


# ---------------------------------------------------------------- persistent arm
def bench_gpu(args, rank, world, local):
    import torch

    from persistent_execution_b200 import build as B
    from persistent_execution_b200 import gpuos as G
    from persistent_execution_b200 import measure as Ms
    from persistent_execution_b200 import replicas as R
    from persistent_execution_b200 import streams
    from persistent_execution_b200 import workloads as W

    torch.cuda.set_device(local)
    B.build()
    w = W.make(args.config)
    n = w.n_ops
    alg_bytes = int(Ms.op_bytes(w).sum())
    stream = torch.cuda.Stream()
    dev = streams.DeviceArenas(w)
    torch.cuda.synchronize()
    descs = streams.descriptors(w, *dev.ptrs)
    cap = 1 << int(np.ceil(np.log2(2 * n + 2)))
    cap = max(cap, 4096)
    rt = G.Runtime(stream.cuda_stream, flags=G.CFG_NO_AUTOSTART, ring_capacity=cap,
                   timeout_ns=10_000_000_000, idle_exit_ns=30_000_000_000)

    if args.only_step:  # one drained step and nothing else (the command profiled with ncu)
        rt.submit_n(descs, dep_base=0)
        rt.flush()
        rt.start(drain=True)
        G.check(rt.wait(G.ALL, 120.0), "wait")
        G.check(rt.stop(120.0), "stop")
        rt.destroy()
        stream.synchronize()
        if rank == 0:
            print(json.dumps({"only_step": True, "config": args.config, "ops": n}))
        return

    # A working set that fits in L2 is flushed before every step (a write of a
    # buffer larger than L2, on the same stream, outside the step's events).
    flush_buf = None
    if dev.f32.numel() * 4 + dev.bf16.numel() * 2 < 2 * L2_BYTES:
        flush_buf = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    def step_loop(k, events=None):
        """k drained steps; the next step's ops are written while the kernel runs.
        events[i] = (start, end) brackets step i's kernel launches on the stream."""
        for i in range(k):
            if flush_buf is not None:
                with torch.cuda.stream(stream):
                    flush_buf.fill_(float(i))
            if events is not None:
                events[i][0].record(stream)
            rt.start(drain=True)
            if events is not None:
                events[i][1].record(stream)
            if i + 1 < k:
                rt.submit_n(descs, dep_base=0)
            st = rt.wait(first_of[i] + n - 1, 120.0)
            G.check(st, "wait")
            G.check(rt.stop(120.0), "stop")
            first_of.append(first_of[i] + n)
            rt.flush()

    # warm-up
    first_of = [rt.submit_n(descs, dep_base=0)]
    rt.flush()
    step_loop(args.warmup)
    first_of = [rt.submit_n(descs, dep_base=0)]
    rt.flush()
    torch.cuda.synchronize()
    ranks = R.from_env()
    R.barrier(ranks)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    st0 = rt.stats()
    t_wall = time.perf_counter()
    with Clocks(local) as clk:
        step_loop(args.steps, ev)
        torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    R.barrier(ranks)
    torch.cuda.synchronize()
    st1 = rt.stats()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    elapsed_ms = R.max_over_ranks(ranks, float(np.sum(step_ms)), device="cuda")
    launches = st1["kernel_launches"] - st0["kernel_launches"]
    span_ns = st1["gpu_span_ns"]
    ms_step = elapsed_ms / args.steps
    value = R.job_throughput(n * args.steps, ranks, elapsed_ms / 1e3)
    per_launch_s = float(np.mean(step_ms)) / 1e3  # one persistent kernel (and its reset kernel) per step
    peak, peak_kind = measured_peak()
    achieved = alg_bytes / per_launch_s / 1e9

    # host submission cost alone (C-level, no device involvement)
    rt2 = G.Runtime(stream.cuda_stream, flags=G.CFG_NO_AUTOSTART, ring_capacity=cap)
    t0 = time.perf_counter()
    rt2.submit_n(descs, dep_base=0)
    submit_us = (time.perf_counter() - t0) / n * 1e6
    rt2.destroy()

    # e2e: host buffers in, device run, results out, through the public API
    e2e = None
    if True:
        host_in32 = torch.from_numpy(w.arena_f32[:w.n_init_f32]).pin_memory()
        host_in16 = torch.from_numpy(w.arena_bf16[:w.n_init_bf16].view(np.int16)).pin_memory()
        out32 = torch.empty(w.arena_f32.size - w.n_init_f32, dtype=torch.float32).pin_memory()
        out16 = torch.empty(w.arena_bf16.size - w.n_init_bf16, dtype=torch.int16).pin_memory()
        h2d = host_in32.numel() * 4 + host_in16.numel() * 2
        d2h = out32.numel() * 4 + out16.numel() * 2
        e2e_steps = max(1, min(args.steps, 3))
        tms = []
        for rep in range(e2e_steps + 1):
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                dev.f32[:w.n_init_f32].copy_(host_in32, non_blocking=True)
                dev.bf16[:w.n_init_bf16].view(torch.int16).copy_(host_in16, non_blocking=True)
                f = rt.submit_n(descs, dep_base=0)
                rt.flush()
                rt.start(drain=True)
                out32.copy_(dev.f32[w.n_init_f32:], non_blocking=True)
                out16.copy_(dev.bf16[w.n_init_bf16:].view(torch.int16), non_blocking=True)
                e1.record(stream)
            e1.synchronize()
            G.check(rt.wait(f + n - 1, 120.0), "e2e wait")
            G.check(rt.stop(120.0), "e2e stop")
            if rep > 0:
                tms.append(e0.elapsed_time(e1))
        e2e_ms = R.max_over_ranks(ranks, float(np.median(tms)), device="cuda")
        e2e = {"value": R.job_throughput(n, ranks, e2e_ms / 1e3), "unit": "ops/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms}

    # Through the live API: a resident kernel (gpuos_create), the whole stream
    # submitted and flushed, wall time from the first submit to gpuos_wait(ALL).
    live = None
    try:
        rt3 = G.Runtime(stream.cuda_stream, ring_capacity=cap, timeout_ns=10_000_000_000,
                        idle_exit_ns=30_000_000_000)
        tl = []
        for rep in range(4):
            t0 = time.perf_counter()
            rt3.submit_n(descs, dep_base=0)
            rt3.flush()
            G.check(rt3.wait(G.ALL, 120.0), "live wait")
            if rep > 0:
                tl.append(time.perf_counter() - t0)
        rt3.destroy()
        stream.synchronize()
        live = {"us_per_op": float(np.median(tl)) / n * 1e6, "ms_per_stream": float(np.median(tl)) * 1e3,
                "what": "kernel resident (gpuos_create); wall time from the first gpuos_submit to gpuos_wait(ALL)"}
    except Exception as ex:  # reported, never fatal to the bench line
        live = {"error": str(ex)[:200]}

    baselines = None
    if args.baselines and rank == 0:
        baselines = run_baselines(args, G, torch, stream, descs, n, dev)

    rt.destroy()
    stream.synchronize()
    if rank != 0:
        return
    cpu = cpu_baseline(w, args.config) if world == 1 else None
    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "ops/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if args.config != 3 else "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_NAMES[args.config], "ops_per_step": n,
                   "algorithmic_bytes_per_step": alg_bytes,
                   "l2": ("L2 flushed before every step (write of a 256 MiB buffer)" if flush_buf is not None
                          else "inputs larger than L2 (no flush)"),
                   "timing": "CUDA events around each step's kernel launches on the runtime stream; "
                             "value and roofline use their sum",
                   "mode": "each step: ops published, then one persistent kernel (drain)"},
        "us_per_op": ms_step * 1e3 / n,
        "wall_ms_per_step": t_wall / args.steps * 1e3,
        "hbm_gbs": achieved,
        "hbm_frac_of_nominal_8000": achieved / NOMINAL_HBM_GBS,
        "host_submit_us_per_op": submit_us,
        "live_api": live,
        "gpu_span_ms_last_step": span_ns / 1e6,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": peak_kind, "traffic": profiled_traffic(args.config)},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks,
        "runtime_stats": {k: st1[k] - st0[k] for k in ("items_executed", "ops_claimed", "run_ops",
                                                       "idle_poll_cycles", "dep_wait_cycles", "fetch_descs")},
    }
    if baselines:
        line["baselines"] = baselines
    print(json.dumps(line), flush=True)


def run_baselines(args, G, torch, stream, descs, n, dev):
    """One kernel per op and CUDA Graph replay of the same launches, same stream."""
    import ctypes
    cfg = G.default_config()
    out = {}
    reps = 3
    # one launch per op: wall time from first launch to stream synchronisation
    G.check(G.gpuos_launch_ops(descs, n, cfg, stream.cuda_stream), "launch_ops")
    stream.synchronize()
    ts = []
    for _ in range(reps):
        t0 = time.perf_counter()
        G.check(G.gpuos_launch_ops(descs, n, cfg, stream.cuda_stream), "launch_ops")
        stream.synchronize()
        ts.append(time.perf_counter() - t0)
    out["per_op_launch_us_per_op"] = float(np.median(ts)) / n * 1e6
    for mode, name in ((0, "graph_chain"), (1, "graph_edges")):
        g = ctypes.c_void_p()
        bns = ctypes.c_uint64()
        st = G.gpuos_graph_create(descs, n, 0, cfg, stream.cuda_stream, mode, g, bns)
        if st != G.OK:
            out[name + "_error"] = G.STATUS[st]
            continue
        G.check(G.gpuos_graph_launch(g, stream.cuda_stream), "graph launch")
        stream.synchronize()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            G.check(G.gpuos_graph_launch(g, stream.cuda_stream), "graph launch")
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        G.gpuos_graph_destroy(g)
        out[name + "_us_per_op"] = float(np.median(ts)) * 1e3 / n
        out[name + "_build_s"] = bns.value / 1e9
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="persistent", choices=["persistent", "reference"])
    ap.add_argument("--baselines", type=int, default=1)
    ap.add_argument("--ref-sample", type=int, default=0)
    ap.add_argument("--only-step", action="store_true",
                    help="run one drained step of the stream and exit (for ncu captures)")
    args = ap.parse_args()
    rank, world, local = setup_dist(args)
    try:
        if args.impl == "reference":
            bench_reference(args, rank, world)
        else:
            bench_gpu(args, rank, world, local)
    finally:
        from persistent_execution_b200 import replicas as R
        R.finalize(R.from_env())


if __name__ == "__main__":
    main()
