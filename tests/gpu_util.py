"""Helpers that run a generated workload through the CUDA library (test infrastructure)."""

from __future__ import annotations

import numpy as np
import torch

from persistent_execution_b200 import gpuos as G
from persistent_execution_b200 import streams

TEST_CFG = dict(timeout_ns=3_000_000_000, idle_exit_ns=5_000_000_000, submit_timeout_ns=3_000_000_000,
                ring_capacity=4096)


def run_persistent(w, mode="drain", batch=256, trace=False, cfg=None, timeout_s=60.0):
    """Runs every op of w on the persistent kernel; returns (a32, a16, trace, stats).

    mode "drain": submit everything, flush, launch with GPUOS_START_DRAIN.
    mode "live": launch first, then submit in batches of `batch` with a flush each.
    """
    kw = dict(TEST_CFG)
    kw.update(cfg or {})
    kw["flags"] = kw.get("flags", 0) | G.CFG_NO_AUTOSTART | (G.CFG_TRACE if trace else 0)
    if w.n_ops >= kw["ring_capacity"]:
        kw["ring_capacity"] = 1 << int(np.ceil(np.log2(w.n_ops + 1)))
    stream = torch.cuda.Stream()
    dev = streams.DeviceArenas(w, fill_outputs=float("nan"))
    torch.cuda.synchronize()
    descs = streams.descriptors(w, *dev.ptrs)
    rt = G.Runtime(stream.cuda_stream, **kw)
    try:
        if mode == "drain":
            first = rt.submit_n(descs, dep_base=0)
            rt.flush()
            rt.start(drain=True)
        else:
            rt.start(drain=False)
            first = streams.submit_stream(rt, descs, batch=batch)
        st = rt.wait(G.ALL, timeout_s)
        assert st == G.OK, f"wait: {G.STATUS[st]} stats={rt.stats()}"
        st = rt.stop(timeout_s)
        assert st == G.OK, f"stop: {G.STATUS[st]}"
        tr = rt.trace(first, w.n_ops) if trace else None
        stats = rt.stats()
    finally:
        rt.destroy()
    stream.synchronize()
    a32, a16 = dev.download()
    return a32, a16, tr, stats


def run_launches(w, graph_mode=None, cfg=None):
    """The same ops, one kernel per op (graph_mode None) or as a CUDA Graph (0 or 1)."""
    c = G.default_config(**(cfg or {}))
    stream = torch.cuda.Stream()
    dev = streams.DeviceArenas(w, fill_outputs=float("nan"))
    torch.cuda.synchronize()
    descs = streams.descriptors(w, *dev.ptrs)
    if graph_mode is None:
        G.check(G.gpuos_launch_ops(descs, len(descs), c, stream.cuda_stream), "gpuos_launch_ops")
    else:
        g = __import__("ctypes").c_void_p()
        ns = __import__("ctypes").c_uint64()
        G.check(G.gpuos_graph_create(descs, len(descs), 0, c, stream.cuda_stream, graph_mode, g, ns),
                "gpuos_graph_create")
        G.check(G.gpuos_graph_launch(g, stream.cuda_stream), "gpuos_graph_launch")
        stream.synchronize()
        G.gpuos_graph_destroy(g)
    stream.synchronize()
    return dev.download()
