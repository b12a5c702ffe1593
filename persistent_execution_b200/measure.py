"""Algorithmic byte counts and roofline arithmetic.

The algorithmic bytes of an op are the bytes it must move: each operand read
once and the output written once ("Launch Overhead and Fusion", section
"Fusion": a fused relu(a*x+b) moves 8 bytes per fp32 element, the three
unfused kernels 24). A broadcast operand counts its distinct elements,
min(in_n, n). Row ops read their row tensor once and their per-column
weights once.
"""

from __future__ import annotations

import numpy as np

from . import workloads as W

ESIZE = (4, 2)  # fp32, bf16


def _chain_operands(prog_row) -> tuple:
    names = {W.MICRO[p] for p in prog_row if p >= 0}
    return ("add1" in names or "mul1" in names), ("add2" in names or "mul2" in names)


def op_bytes(w: W.Workload) -> np.ndarray:
    """Algorithmic bytes of every op of a workload (int64 array)."""
    o = w.ops
    n = o["rows"] * o["cols"]
    es = np.where(o["dtype"] == 0, 4, 2).astype(np.int64)
    in0 = np.minimum(o["in_n"][:, 0], n)
    in1 = np.minimum(o["in_n"][:, 1], n)
    out = np.zeros(w.n_ops, dtype=np.int64)
    for i in range(w.n_ops):
        k = W.KINDS[o["kind"][i]]
        if k in ("add", "mul", "silu_mul"):
            e = in0[i] + in1[i] + n[i]
        elif k in ("scale", "gelu", "relu_affine"):
            e = in0[i] + n[i]
        elif k == "ew_chain":
            u1, u2 = _chain_operands(o["prog"][i])
            e = in0[i] + (in1[i] if u1 else 0) + (n[i] if u2 else 0) + n[i]
        elif k in ("rowsum", "rowmax"):
            e = n[i] + o["rows"][i]
        elif k in ("softmax", "rotary"):
            e = 2 * n[i]
        elif k == "rmsnorm":
            e = 2 * n[i] + o["cols"][i]
        elif k == "layernorm":
            e = 2 * n[i] + 2 * o["cols"][i]
        else:
            raise ValueError(k)
        out[i] = e * es[i]
    return out


def launch_overhead_share(launches: int, per_launch_s: float, compute_s: float) -> float:
    """Fraction of a step spent launching when launches do not overlap compute."""
    t = launches * per_launch_s
    return t / (t + compute_s)


def roofline(bytes_per_launch: float, seconds: float, peak_gbs: float) -> dict:
    achieved = bytes_per_launch / seconds / 1e9
    return {"achieved": achieved, "peak": peak_gbs, "frac": achieved / peak_gbs}
