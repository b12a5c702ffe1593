"""ctypes binding of the C ABI in include/gpuos.h (argument marshalling only).

Every function below has the name and argument order of its C counterpart and
returns the integer gpuos_status. ``Runtime`` wraps the same calls and raises
``GpuosError`` on a non-zero status. There is no fallback: if libgpuos.so was
not built, ``lib()`` raises.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("GPUOS_LIB", os.path.join(HERE, "libgpuos.so"))  # override: an alternative build

OK, EINVAL, EAGAIN, ETIMEDOUT, EBADOP, EDEVICE, ESTOPPED, ENOMEM = range(8)
STATUS = ("OK", "EINVAL", "EAGAIN", "ETIMEDOUT", "EBADOP", "EDEVICE", "ESTOPPED", "ENOMEM")
F32, BF16 = 0, 1
OP = {
    "nop": 0, "add": 1, "mul": 2, "scale": 3, "gelu": 4, "relu_affine": 5, "silu_mul": 6,
    "ew_chain": 7, "rowsum": 16, "rowmax": 17, "softmax": 18, "rmsnorm": 19, "layernorm": 20,
    "rotary": 21, "stall": 250,
}
MICRO = {"affine": 1, "scale": 2, "adds": 3, "relu": 4, "gelu": 5, "silu": 6,
         "add1": 7, "mul1": 8, "add2": 9, "mul2": 10}
NO_DEP = (1 << 64) - 1
ALL = NO_DEP
NO_BASE = NO_DEP
CFG_NO_AUTOSTART = 1
CFG_TRACE = 2
CFG_NO_BULK = 4
CFG_NO_HANDOFF = 8
CFG_NO_FUSION = 16
START_DRAIN = 1

# numpy view of gpuos_desc (128 bytes), for building many descriptors at once
DESC = np.dtype([
    ("opcode", "<u2"), ("dtype", "u1"), ("nmicro", "u1"), ("flags", "<u4"),
    ("dep", "<u8", (2,)), ("in_", "<u8", (3,)), ("out", "<u8"),
    ("rows", "<i8"), ("cols", "<i8"), ("in_n", "<i8", (2,)), ("s", "<f4", (4,)),
    ("pos", "<i4"), ("micro", "u1", (8,)), ("reserved0", "<u4"), ("reserved1", "<u8"),
])
assert DESC.itemsize == 128


class Config(ctypes.Structure):
    _fields_ = [
        ("ring_capacity", ctypes.c_uint32), ("grid", ctypes.c_uint32),
        ("timeout_ns", ctypes.c_uint64), ("submit_timeout_ns", ctypes.c_uint64),
        ("idle_exit_ns", ctypes.c_uint64), ("elem_chunk", ctypes.c_uint32),
        ("row_chunk", ctypes.c_uint32), ("backoff_ns", ctypes.c_uint32), ("flags", ctypes.c_uint32),
    ]


class Stats(ctypes.Structure):
    _fields_ = [
        ("ops_submitted", ctypes.c_uint64), ("ops_completed", ctypes.c_uint64),
        ("items_executed", ctypes.c_uint64), ("ops_claimed", ctypes.c_uint64),
        ("run_ops", ctypes.c_uint64), ("idle_poll_cycles", ctypes.c_uint64),
        ("dep_wait_cycles", ctypes.c_uint64), ("fetch_descs", ctypes.c_uint64),
        ("max_ring_occupancy", ctypes.c_uint64), ("gpu_span_ns", ctypes.c_uint64),
        ("kernel_launches", ctypes.c_uint64), ("num_ctas", ctypes.c_uint32),
        ("last_error", ctypes.c_int32), ("error_op", ctypes.c_uint64),
    ]

    def as_dict(self) -> dict:
        return {k: getattr(self, k) for k, _ in self._fields_}


TRACE = np.dtype([("id", "<u8"), ("t_start", "<u8"), ("t_end", "<u8"), ("cta", "<u4"),
                  ("smid", "<u4"), ("items", "<u4"), ("claim", "<u4")])
assert TRACE.itemsize == 40

_lib = None
_vp = ctypes.c_void_p
_u64 = ctypes.c_uint64
_u32 = ctypes.c_uint32

_SIGS = {
    "gpuos_default_config": [ctypes.POINTER(Config)],
    "gpuos_create": [_vp, ctypes.POINTER(_vp)],
    "gpuos_create_ex": [_vp, ctypes.POINTER(Config), ctypes.POINTER(_vp)],
    "gpuos_start": [_vp, _u32],
    "gpuos_stop": [_vp, _u64],
    "gpuos_destroy": [_vp],
    "gpuos_submit": [_vp, _vp, ctypes.POINTER(_u64)],
    "gpuos_submit_n": [_vp, _vp, _u64, _u64, ctypes.POINTER(_u64)],
    "gpuos_flush": [_vp],
    "gpuos_wait": [_vp, _u64, _u64],
    "gpuos_query": [_vp, ctypes.POINTER(_u64)],
    "gpuos_get_stats": [_vp, ctypes.POINTER(Stats)],
    "gpuos_trace_read": [_vp, _u64, _u64, _vp],
    "gpuos_launch_ops": [_vp, _u64, ctypes.POINTER(Config), _vp],
    "gpuos_graph_create": [_vp, _u64, _u64, ctypes.POINTER(Config), _vp, _u32, ctypes.POINTER(_vp),
                           ctypes.POINTER(_u64)],
    "gpuos_graph_launch": [_vp, _vp],
    "gpuos_graph_destroy": [_vp],
    "gpuos_validate": [_vp],
    "gpuos_debug_submit_raw": [_vp, _vp, ctypes.POINTER(_u64)],
    "gpuos_debug_release_stall": [_vp],
    "gpuos_run_static": [_vp, _u64, ctypes.POINTER(Config), _vp],
}


def lib():
    """Loads libgpuos.so (raises if it was not built: there is no CPU path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with `python -m persistent_execution_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.gpuos_work_items.argtypes = [_vp, ctypes.POINTER(Config)]
        L.gpuos_work_items.restype = _u64
        L.gpuos_status_string.argtypes = [ctypes.c_int]
        L.gpuos_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _ptr(a) -> int:
    if isinstance(a, np.ndarray):
        return a.ctypes.data
    return a


# ---------------------------------------------------------------- C-named calls
def gpuos_default_config(cfg: Config) -> int:
    return lib().gpuos_default_config(ctypes.byref(cfg))


def gpuos_create(stream: int, out: ctypes.c_void_p) -> int:
    return lib().gpuos_create(_vp(stream), ctypes.byref(out))


def gpuos_create_ex(stream: int, cfg: Config, out: ctypes.c_void_p) -> int:
    return lib().gpuos_create_ex(_vp(stream), ctypes.byref(cfg) if cfg is not None else None, ctypes.byref(out))


def gpuos_start(rt, flags: int) -> int:
    return lib().gpuos_start(rt, flags)


def gpuos_stop(rt, timeout_ns: int) -> int:
    return lib().gpuos_stop(rt, timeout_ns)


def gpuos_destroy(rt) -> int:
    return lib().gpuos_destroy(rt)


def gpuos_submit(rt, desc: np.ndarray, id_out: ctypes.c_uint64 = None) -> int:
    return lib().gpuos_submit(rt, _ptr(desc), ctypes.byref(id_out) if id_out is not None else None)


def gpuos_submit_n(rt, descs: np.ndarray, n: int, dep_base: int, first_id_out: ctypes.c_uint64 = None) -> int:
    return lib().gpuos_submit_n(rt, _ptr(descs), n, dep_base,
                                ctypes.byref(first_id_out) if first_id_out is not None else None)


def gpuos_flush(rt) -> int:
    return lib().gpuos_flush(rt)


def gpuos_wait(rt, id_: int, timeout_ns: int) -> int:
    return lib().gpuos_wait(rt, id_, timeout_ns)


def gpuos_query(rt, completed: ctypes.c_uint64) -> int:
    return lib().gpuos_query(rt, ctypes.byref(completed))


def gpuos_get_stats(rt, out: Stats) -> int:
    return lib().gpuos_get_stats(rt, ctypes.byref(out))


def gpuos_trace_read(rt, first_id: int, n: int, out: np.ndarray) -> int:
    return lib().gpuos_trace_read(rt, first_id, n, _ptr(out))


def gpuos_launch_ops(descs: np.ndarray, n: int, cfg: Config, stream: int) -> int:
    return lib().gpuos_launch_ops(_ptr(descs), n, ctypes.byref(cfg) if cfg is not None else None, _vp(stream))


def gpuos_graph_create(descs, n, dep_base, cfg, stream, mode, out: ctypes.c_void_p, build_ns: ctypes.c_uint64) -> int:
    return lib().gpuos_graph_create(_ptr(descs), n, dep_base, ctypes.byref(cfg) if cfg is not None else None,
                                    _vp(stream), mode, ctypes.byref(out), ctypes.byref(build_ns))


def gpuos_graph_launch(g, stream: int) -> int:
    return lib().gpuos_graph_launch(g, _vp(stream))


def gpuos_graph_destroy(g) -> int:
    return lib().gpuos_graph_destroy(g)


def gpuos_validate(desc: np.ndarray) -> int:
    return lib().gpuos_validate(_ptr(desc))


def gpuos_work_items(desc: np.ndarray, cfg: Config = None) -> int:
    return lib().gpuos_work_items(_ptr(desc), ctypes.byref(cfg) if cfg is not None else None)


def gpuos_status_string(s: int) -> str:
    return lib().gpuos_status_string(s).decode()


def gpuos_debug_submit_raw(rt, desc: np.ndarray, id_out: ctypes.c_uint64 = None) -> int:
    return lib().gpuos_debug_submit_raw(rt, _ptr(desc), ctypes.byref(id_out) if id_out is not None else None)


def gpuos_debug_release_stall(rt) -> int:
    return lib().gpuos_debug_release_stall(rt)


def gpuos_run_static(descs: np.ndarray, n: int, cfg: Config, stream: int) -> int:
    return lib().gpuos_run_static(_ptr(descs), n, ctypes.byref(cfg) if cfg is not None else None, _vp(stream))


# ---------------------------------------------------------------- convenience wrapper
class GpuosError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS[status] if 0 <= status < len(STATUS) else status}")


def check(status: int, what: str) -> None:
    if status != OK:
        raise GpuosError(status, what)


def default_config(**kw) -> Config:
    c = Config()
    check(gpuos_default_config(c), "gpuos_default_config")
    for k, v in kw.items():
        setattr(c, k, v)
    return c


class Runtime:
    """One persistent runtime on one CUDA stream (a cudaStream_t as int)."""

    def __init__(self, stream: int, cfg: Config = None, **kw):
        if cfg is None:
            cfg = default_config(**kw)
        self.cfg = cfg
        self.stream = stream
        self.h = ctypes.c_void_p()
        check(gpuos_create_ex(stream, cfg, self.h), "gpuos_create_ex")

    def start(self, drain: bool = False) -> None:
        check(gpuos_start(self.h, START_DRAIN if drain else 0), "gpuos_start")

    def stop(self, timeout_s: float = 10.0) -> int:
        return gpuos_stop(self.h, int(timeout_s * 1e9))

    def submit(self, desc: np.ndarray) -> int:
        i = ctypes.c_uint64()
        check(gpuos_submit(self.h, desc, i), "gpuos_submit")
        return i.value

    def submit_n(self, descs: np.ndarray, dep_base: int = 0) -> int:
        descs = np.ascontiguousarray(descs, dtype=DESC)
        first = ctypes.c_uint64()
        check(gpuos_submit_n(self.h, descs, len(descs), dep_base, first), "gpuos_submit_n")
        return first.value

    def flush(self) -> None:
        check(gpuos_flush(self.h), "gpuos_flush")

    def wait(self, id_: int = ALL, timeout_s: float = 30.0) -> int:
        return gpuos_wait(self.h, id_, int(timeout_s * 1e9))

    def query(self) -> int:
        c = ctypes.c_uint64()
        gpuos_query(self.h, c)
        return c.value

    def stats(self) -> dict:
        s = Stats()
        check(gpuos_get_stats(self.h, s), "gpuos_get_stats")
        return s.as_dict()

    def trace(self, first_id: int, n: int) -> np.ndarray:
        out = np.zeros(n, dtype=TRACE)
        check(gpuos_trace_read(self.h, first_id, n, out), "gpuos_trace_read")
        return out

    def destroy(self) -> int:
        if self.h:
            s = gpuos_destroy(self.h)
            self.h = ctypes.c_void_p()
            return s
        return OK

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.destroy()
