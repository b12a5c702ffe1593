"""Turns a generated workload into gpuos descriptors on device arenas, and runs it.

The device copy of a workload is two torch tensors (fp32 and bf16 arenas);
each op's operands are pointers into them. Dependencies are written as
indices into the workload (submitted with dep_base = 0), so the same
descriptor array can be submitted again in every step.
"""

from __future__ import annotations

import numpy as np
import torch

from . import gpuos as G
from . import workloads as W

_OPC = np.array([G.OP[k] for k in W.KINDS], dtype=np.uint16)
_MIC = np.array([G.MICRO[m] for m in W.MICRO], dtype=np.uint8)


class DeviceArenas:
    """fp32 and bf16 arenas of a workload in device memory."""

    def __init__(self, w: W.Workload, device="cuda", upload=True, fill_outputs=None):
        self.f32 = torch.empty(w.arena_f32.size, dtype=torch.float32, device=device)
        self.bf16 = torch.empty(w.arena_bf16.size, dtype=torch.bfloat16, device=device)
        self.w = w
        if upload:
            self.upload(fill_outputs)

    def upload(self, fill_outputs=None):
        """Copies the input region; the output region starts as zeros, or as
        `fill_outputs` (NaN makes an op that never ran visible)."""
        w = self.w
        self.f32[:w.n_init_f32].copy_(torch.from_numpy(w.arena_f32[:w.n_init_f32]))
        self.bf16[:w.n_init_bf16].copy_(
            torch.from_numpy(w.arena_bf16[:w.n_init_bf16].view(np.int16)).view(torch.bfloat16))
        fill = 0.0 if fill_outputs is None else fill_outputs
        self.f32[w.n_init_f32:].fill_(fill)
        self.bf16[w.n_init_bf16:].fill_(fill)

    def download(self):
        a32 = self.f32.cpu().numpy()
        a16 = self.bf16.cpu().view(torch.int16).numpy().view(np.uint16)
        return a32, a16

    @property
    def ptrs(self):
        return self.f32.data_ptr(), self.bf16.data_ptr()


def descriptors(w: W.Workload, ptr_f32: int, ptr_bf16: int) -> np.ndarray:
    """gpuos_desc array of every op of w; deps are workload indices (dep_base 0)."""
    o = w.ops
    n = w.n_ops
    d = np.zeros(n, dtype=G.DESC)
    d["opcode"] = _OPC[o["kind"]]
    d["dtype"] = o["dtype"]
    base = np.where(o["dtype"] == 0, ptr_f32, ptr_bf16).astype(np.uint64)
    es = np.where(o["dtype"] == 0, 4, 2).astype(np.uint64)
    ins = np.zeros((n, 3), dtype=np.uint64)
    for k in range(3):
        off = o["in_off"][:, k]
        ok = off >= 0
        ins[ok, k] = base[ok] + off[ok].astype(np.uint64) * es[ok]
    d["in_"] = ins
    d["out"] = base + o["out_off"].astype(np.uint64) * es
    d["rows"] = o["rows"]
    d["cols"] = o["cols"]
    kind = np.asarray(W.KINDS)[o["kind"]]
    ew = np.isin(kind, ["add", "mul", "scale", "gelu", "relu_affine", "silu_mul", "ew_chain"])
    d["in_n"] = np.where(ew[:, None], o["in_n"], 0)
    d["s"] = o["s"]
    d["pos"] = o["pos"]
    prog = o["prog"]
    nm = (prog >= 0).sum(axis=1)
    d["nmicro"] = np.where(kind == "ew_chain", nm, 0)
    micro = np.where(prog >= 0, _MIC[np.clip(prog, 0, None)], 0).astype(np.uint8)
    d["micro"] = micro
    dep = o["dep"]
    d["dep"] = np.where(dep >= 0, dep.astype(np.uint64), np.uint64(G.NO_DEP))
    return d


def submit_stream(rt: G.Runtime, descs: np.ndarray, batch: int = 0) -> int:
    """Submits a whole descriptor array; flushes every `batch` ops (0 = once at the end)."""
    n = len(descs)
    first = None
    if batch <= 0:
        batch = n
    for s in range(0, n, batch):
        f = rt.submit_n(descs[s:s + batch], dep_base=s)
        if first is None:
            first = f
        rt.flush()
    return first if first is not None else rt.query()
