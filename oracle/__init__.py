"""CPU oracle for op streams: ctypes adapter over ``liboracle.so``.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The GPU runtime never
imports it, and it imports nothing from the GPU runtime: it shares only the
seeded generator module ``persistent_execution_b200.workloads``, which holds
no op arithmetic.

Parity status of each op definition (every op is pinned by tests in
``tests/test_oracle_pins.py``): relu-affine, add, mul, scale, gelu, silu_mul,
fused chains, row sum, row max, softmax, RMSNorm, LayerNorm, rotary, bf16
rounding.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from persistent_execution_b200 import workloads as W

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_HDR = os.path.join(_HERE, "oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")

KIND_CODE = {
    "add": 101, "mul": 102, "scale": 103, "gelu": 104, "relu_affine": 105, "silu_mul": 106,
    "ew_chain": 107, "rowsum": 108, "rowmax": 109, "softmax": 110, "rmsnorm": 111,
    "layernorm": 112, "rotary": 113,
}
MICRO_CODE = {
    "affine": 1, "scale": 2, "adds": 3, "relu": 4, "gelu": 5, "silu": 6,
    "add1": 7, "mul1": 8, "add2": 9, "mul2": 10,
}

ORC_OP = np.dtype([
    ("kind", "<i4"), ("dtype", "<i4"), ("in_off", "<i8", (3,)), ("out_off", "<i8"),
    ("rows", "<i8"), ("cols", "<i8"), ("in_n", "<i8", (2,)), ("s", "<f4", (4,)),
    ("pos", "<i4"), ("nprog", "<i4"), ("prog", "i1", (8,)),
])
assert ORC_OP.itemsize == 104

_lib = None


def build(force: bool = False) -> str:
    """Compiles liboracle.so with plain gcc (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
            os.path.getmtime(_SRC), os.path.getmtime(_HDR)):
        tmp = _LIB + ".tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        vp, i64 = ctypes.c_void_p, ctypes.c_int64
        L.orc_run.argtypes = [vp, i64, vp, i64, vp, i64, ctypes.POINTER(i64)]
        L.orc_run.restype = ctypes.c_int
        L.orc_apply.argtypes = [vp, vp, i64, vp, i64, vp]
        L.orc_apply.restype = ctypes.c_int
        L.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        L.orc_f32_to_bf16.restype = ctypes.c_uint16
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_gelu.argtypes = [ctypes.c_double]
        L.orc_gelu.restype = ctypes.c_double
        _lib = L
    return _lib


def to_orc(w: W.Workload, idx=None) -> np.ndarray:
    """Converts the generator's op columns (all, or the indices `idx`) to orc_op records."""
    ops = w.ops
    sel = np.arange(w.n_ops) if idx is None else np.asarray(idx, dtype=np.int64)
    out = np.zeros(len(sel), dtype=ORC_OP)
    kinds = ops["kind"][sel]
    out["kind"] = np.array([KIND_CODE[W.KINDS[k]] for k in kinds], dtype=np.int32)
    out["dtype"] = ops["dtype"][sel]
    out["in_off"] = ops["in_off"][sel]
    out["out_off"] = ops["out_off"][sel]
    out["rows"] = ops["rows"][sel]
    out["cols"] = ops["cols"][sel]
    out["in_n"] = ops["in_n"][sel]
    out["s"] = ops["s"][sel]
    out["pos"] = ops["pos"][sel]
    prog = ops["prog"][sel]
    nprog = (prog >= 0).sum(axis=1)
    out["nprog"] = nprog
    codes = np.zeros_like(prog)
    for j, name in enumerate(W.MICRO):
        codes[prog == j] = MICRO_CODE[name]
    out["prog"] = codes
    return out


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def run_ops(orc: np.ndarray, a32: np.ndarray, a16: np.ndarray) -> None:
    """Executes orc_op records in order on the given arenas (modified in place)."""
    orc = np.ascontiguousarray(orc, dtype=ORC_OP)
    assert a32.dtype == np.float32 and a16.dtype == np.uint16
    assert a32.flags.c_contiguous and a16.flags.c_contiguous
    bad = ctypes.c_int64(-1)
    rc = lib().orc_run(_ptr(orc), len(orc), _ptr(a32), a32.size, _ptr(a16), a16.size,
                       ctypes.byref(bad))
    if rc != 0:
        raise RuntimeError(f"oracle rejected op {bad.value}: status {rc}")


def run(w: W.Workload):
    """Runs a whole workload from its initial arenas; returns (arena_f32, arena_bf16)."""
    a32 = w.arena_f32.copy()
    a16 = w.arena_bf16.copy()
    run_ops(to_orc(w), a32, a16)
    return a32, a16


def apply(w: W.Workload, i: int, a32: np.ndarray, a16: np.ndarray) -> np.ndarray:
    """Op i of w applied to operands read from the given arenas; returns its output."""
    rec = to_orc(w, [i])
    n = W.output_extent(w, i)
    dt = int(w.ops["dtype"][i])
    out = np.empty(n, dtype=np.float32 if dt == 0 else np.uint16)
    a32 = np.ascontiguousarray(a32, dtype=np.float32)
    a16 = np.ascontiguousarray(a16, dtype=np.uint16)
    rc = lib().orc_apply(_ptr(rec), _ptr(a32), a32.size, _ptr(a16), a16.size, _ptr(out))
    if rc != 0:
        raise RuntimeError(f"oracle rejected op {i}: status {rc}")
    return out


def f32_to_bf16(x: float) -> int:
    return int(lib().orc_f32_to_bf16(x))


def bf16_to_f32(h: int) -> float:
    return float(lib().orc_bf16_to_f32(h))


def gelu(x: float) -> float:
    return float(lib().orc_gelu(x))
