"""Ordering audit of a device event log against the dependency DAG.

The persistent kernel may run ops in any order that respects every declared
dependency (GPUOS, arXiv 2604.17861: a persistent worker claims tasks from a
host-managed work queue; CUDA streams run FIFO, which is the ordering a
dependency edge stands in for, LithOS summary section 2.1). The audit checks a
recorded schedule: every op starts only after each of its dependencies ended.
"""

from __future__ import annotations

import numpy as np


def violations(dep: np.ndarray, t_start: np.ndarray, t_end: np.ndarray) -> list:
    """Edges (d, c) with end(d) > start(c); `dep` is (n, 2) of earlier-op indices or -1."""
    dep = np.asarray(dep, dtype=np.int64)
    bad = []
    for k in range(dep.shape[1]):
        c = np.nonzero(dep[:, k] >= 0)[0]
        d = dep[c, k]
        viol = t_end[d] > t_start[c]
        bad.extend(zip(d[viol].tolist(), c[viol].tolist()))
    return bad


def is_valid_order(dep, order) -> bool:
    """True if the sequence `order` (op indices, each once) places every op after its dependencies."""
    order = list(order)
    n = len(dep)
    if sorted(order) != list(range(n)):
        return False
    pos = np.empty(n, dtype=np.int64)
    pos[np.asarray(order, dtype=np.int64)] = np.arange(n)
    return not violations(dep, pos, pos)


def order_from_times(t_start: np.ndarray) -> np.ndarray:
    return np.argsort(np.asarray(t_start), kind="stable")
