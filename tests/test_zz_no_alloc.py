"""gpuos_run_static, the entry point for callers that must not allocate.

cudaMalloc, cudaHostAlloc and cudaFree can stall the whole device and fail
when another allocator already holds the memory, so some callers cannot use
gpuos_create. gpuos_run_static keeps its scratch memory in a fixed array in the
library. This test calls it through the C ABI twice in a row on the same
streams and checks both results against the regular entry point
(gpuos_create / gpuos_submit_n / gpuos_start), within the tolerances of the
other parity tests. The file is named so that pytest collects it last.
"""

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


def _run_static(w, cfg):
    stream = torch.cuda.Stream()
    dev = streams.DeviceArenas(w, fill_outputs=float("nan"))
    torch.cuda.synchronize()
    d = streams.descriptors(w, *dev.ptrs)
    st = G.gpuos_run_static(d, len(d), cfg, stream.cuda_stream)
    assert st == G.OK, G.STATUS[st]
    stream.synchronize()
    return dev.download()


def _same_within_tolerance(w, a32, a16, b32, b16):
    """Every op output of run a equals run b within the parity tolerances (b is the reference)."""
    bad = []
    for i in range(w.n_ops):
        ok, worst, j = P.compare(w, i, P.gpu_output(w, i, a32, a16), P.gpu_output(w, i, b32, b16), b32, b16)
        if not ok:
            bad.append((i, W.KINDS[w.ops["kind"][i]], worst, j))
    return bad


@pytest.mark.parametrize("config", [2, 3, 5])
def test_run_static_matches_regular_entry_point_twice(config):
    w = W.make(config, small=True)
    ref32, ref16, _, _ = U.run_persistent(w)
    cfg = G.default_config(timeout_ns=3_000_000_000, idle_exit_ns=5_000_000_000)
    for _ in range(2):  # the second call reuses the array left by the first
        a32, a16 = _run_static(w, cfg)
        assert _same_within_tolerance(w, a32, a16, ref32, ref16) == []


def test_run_static_rejects_oversized_batches():
    cfg = G.default_config()
    d = np.zeros(4097, dtype=G.DESC)  # NOP descriptors
    d["dep"] = G.NO_DEP
    assert G.gpuos_run_static(d, 4097, cfg, torch.cuda.current_stream().cuda_stream) == G.EINVAL
    assert G.gpuos_run_static(d, 4096, cfg, torch.cuda.Stream().cuda_stream) == G.OK
