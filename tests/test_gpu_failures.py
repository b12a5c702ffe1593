"""Failure detection without faulting the GPU: every failure is made on the host
(an op that waits for a host flag nobody sets, a raw ring entry with an unknown
opcode, a flood of submits) and every device wait is bounded, so the kernel
reports a status and leaves while the CUDA context stays usable."""

import ctypes
import time

import numpy as np
import pytest
import torch

from persistent_execution_b200 import build as B
from persistent_execution_b200 import gpuos as G
from persistent_execution_b200 import streams
from persistent_execution_b200 import workloads as W

from . import gpu_util as U
from . import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()


def _desc(op, dep=(G.NO_DEP, G.NO_DEP)):
    d = np.zeros(1, dtype=G.DESC)
    d["opcode"] = G.OP[op] if isinstance(op, str) else op
    d["dep"] = [list(dep)]
    return d


def _rt(**kw):
    s = torch.cuda.Stream()
    cfg = dict(U.TEST_CFG)
    cfg.update(kw)
    return G.Runtime(s.cuda_stream, **cfg), s


def test_device_wait_times_out_and_reports():
    rt, s = _rt(timeout_ns=300_000_000, ring_capacity=1024)
    a = rt.submit(_desc("stall"))
    rt.submit(_desc("nop", (a, G.NO_DEP)))
    t0 = time.time()
    st = rt.wait(G.ALL, 10.0)
    assert st == G.ETIMEDOUT
    assert time.time() - t0 < 5.0
    assert rt.stats()["last_error"] == G.ETIMEDOUT
    with pytest.raises(G.GpuosError):
        rt.submit(_desc("nop"))  # sticky
    rt.destroy()
    s.synchronize()
    # the context is still usable
    w = W.make(1, small=True, n_ops=20)
    a32, a16, _, _ = U.run_persistent(w)
    assert not P.check_ops(w, a32, a16)


def test_host_wait_timeout_is_not_sticky():
    rt, s = _rt(timeout_ns=5_000_000_000, ring_capacity=1024)
    a = rt.submit(_desc("stall"))
    b = rt.submit(_desc("nop", (a, G.NO_DEP)))
    assert rt.wait(b, 0.05) == G.ETIMEDOUT
    G.check(G.gpuos_debug_release_stall(rt.h), "release")
    assert rt.wait(G.ALL, 5.0) == G.OK
    assert rt.stop() == G.OK
    rt.destroy()


def test_unknown_opcode_is_rejected_on_device():
    rt, s = _rt(ring_capacity=1024)
    assert G.gpuos_validate(_desc(99)) == G.EINVAL
    with pytest.raises(G.GpuosError):
        rt.submit(_desc(99))
    i = ctypes.c_uint64()
    G.check(G.gpuos_debug_submit_raw(rt.h, _desc(99), i), "raw")
    assert rt.wait(G.ALL, 5.0) == G.EBADOP
    st = rt.stats()
    assert st["last_error"] == G.EBADOP and st["error_op"] == i.value
    rt.destroy()
    s.synchronize()


def test_ring_full_returns_eagain_then_drains():
    rt, s = _rt(ring_capacity=1024, submit_timeout_ns=200_000_000, timeout_ns=10_000_000_000)
    prev = rt.submit(_desc("stall"))
    for _ in range(1023):
        prev = rt.submit(_desc("nop", (prev, G.NO_DEP)))
    t0 = time.time()
    with pytest.raises(G.GpuosError) as e:
        rt.submit(_desc("nop", (prev, G.NO_DEP)))
    assert e.value.status == G.EAGAIN and time.time() - t0 >= 0.15
    G.check(G.gpuos_debug_release_stall(rt.h), "release")
    rt.submit(_desc("nop", (prev, G.NO_DEP)))
    assert rt.wait(G.ALL, 10.0) == G.OK
    assert rt.stats()["max_ring_occupancy"] == 1024
    assert rt.stop() == G.OK
    rt.destroy()


def test_idle_exit_then_flush_relaunches():
    rt, s = _rt(idle_exit_ns=100_000_000, ring_capacity=1024)
    for _ in range(3):
        rt.submit(_desc("nop"))
    assert rt.wait(G.ALL, 5.0) == G.OK
    time.sleep(0.6)  # the kernel leaves after 0.1 s without work
    launches = rt.stats()["kernel_launches"]
    for _ in range(3):
        rt.submit(_desc("nop"))
    rt.flush()
    assert rt.wait(G.ALL, 5.0) == G.OK
    assert rt.stats()["kernel_launches"] == launches + 2
    assert rt.stop() == G.OK
    rt.destroy()


def test_sessions_with_dependencies_across_restarts():
    w = W.make(5, n_groups=2, vec=300_000, mat=512)
    stream = torch.cuda.Stream()
    dev = streams.DeviceArenas(w, fill_outputs=float("nan"))
    torch.cuda.synchronize()
    d = streams.descriptors(w, *dev.ptrs)
    rt = G.Runtime(stream.cuda_stream, flags=G.CFG_NO_AUTOSTART, elem_chunk=16384, row_chunk=8192,
                   **{k: v for k, v in U.TEST_CFG.items() if k != "ring_capacity"}, ring_capacity=1024)
    half = w.n_ops // 2
    rt.submit_n(d[:half], dep_base=0)
    rt.flush()
    rt.start(drain=True)
    assert rt.wait(G.ALL, 10.0) == G.OK
    assert rt.stop() == G.OK
    rt.start(drain=False)                  # live session; ops depend on the first session's ops
    rt.submit_n(d[half:], dep_base=half)
    assert rt.wait(G.ALL, 10.0) == G.OK
    assert rt.stop() == G.OK
    rt.destroy()
    stream.synchronize()
    a32, a16 = dev.download()
    import oracle
    r32, r16 = oracle.run(w)
    assert P.bit_exact(w, a32, a16, r32, r16) == []
    assert not P.check_ops(w, a32, a16, idx=P.teacher_forcible(w))
