"""The C-ABI library: loads, exports every declared entry point, validates
descriptors and splits work items on the host (no GPU needed)."""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

from persistent_execution_b200 import build as B
from persistent_execution_b200 import gpuos as G
from persistent_execution_b200 import streams
from persistent_execution_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "gpuos.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gpuos_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    L = G.lib()
    names = declared_symbols()
    assert len(names) >= 20
    for n in names:
        assert hasattr(L, n), n


def test_struct_sizes():
    assert G.DESC.itemsize == 128
    assert ctypes.sizeof(G.Config) == 48
    assert ctypes.sizeof(G.Stats) == 104
    assert G.TRACE.itemsize == 40


def desc(op="add", dtype=G.F32, rows=1, cols=16, **kw):
    d = np.zeros(1, dtype=G.DESC)
    d["opcode"] = G.OP[op]
    d["dtype"] = dtype
    d["rows"] = rows
    d["cols"] = cols
    d["in_"] = [[0x10000, 0x20000, 0x30000]]
    d["out"] = 0x40000
    d["dep"] = [[G.NO_DEP, G.NO_DEP]]
    for k, v in kw.items():
        d[k] = v
    return d


def test_validate_accepts_and_rejects():
    v = G.gpuos_validate
    assert v(desc()) == G.OK
    assert v(desc("nop", rows=0, cols=0)) == G.OK
    assert v(desc(opcode=99)) == G.EINVAL
    assert v(desc(dtype=2)) == G.EINVAL
    assert v(desc(rows=0)) == G.EINVAL
    assert v(desc(flags=1)) == G.EINVAL
    assert v(desc(reserved1=5)) == G.EINVAL
    assert v(desc(out=0)) == G.EINVAL
    assert v(desc(out=0x40002)) == G.EINVAL              # fp32 output not 4-byte aligned
    assert v(desc(dtype=G.BF16, out=0x40002)) == G.OK     # bf16 needs 2-byte alignment
    d = desc(); d["in_"][0, 1] = 0
    assert v(d) == G.EINVAL                               # add reads operand 1
    d = desc("scale"); d["in_"][0, 1] = 0
    assert v(d) == G.OK                                   # scale does not
    assert v(desc("rotary", rows=16, cols=127)) == G.EINVAL
    assert v(desc("rotary", rows=16, cols=128)) == G.OK
    ch = desc("ew_chain", nmicro=2)
    ch["micro"][0, :2] = [G.MICRO["affine"], G.MICRO["relu"]]
    assert v(ch) == G.OK
    ch["micro"][0, 1] = 42
    assert v(ch) == G.EINVAL
    ch = desc("ew_chain", nmicro=3)
    ch["micro"][0, :3] = [G.MICRO["affine"], G.MICRO["affine"], G.MICRO["scale"]]  # 5 scalars
    assert v(ch) == G.EINVAL
    assert v(desc("ew_chain", nmicro=0)) == G.EINVAL
    d = desc("layernorm", rows=4, cols=1024); d["in_"][0, 2] = 0
    assert v(d) == G.EINVAL


def test_work_items():
    wi = G.gpuos_work_items
    assert wi(desc(cols=262144)) == 1
    assert wi(desc(cols=262145)) == 2
    assert wi(desc(cols=64 << 20)) == 256
    assert wi(desc("rowsum", rows=8192, cols=8192)) == 128    # 64 rows per item
    assert wi(desc("softmax", rows=8, cols=4096)) == 1
    assert wi(desc("layernorm", rows=3000, cols=64)) == 3       # at most 1024 rows per item
    assert wi(desc("rowmax", rows=5, cols=200000)) == 3         # two rows per item
    assert wi(desc("rowmax", rows=5, cols=600000)) == 5         # one row per item at least
    cfg = G.default_config(elem_chunk=4096)
    assert wi(desc(cols=4097), cfg) == 2
    assert wi(desc(opcode=99)) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_create_without_gpu_reports_edevice():
    h = ctypes.c_void_p()
    assert G.gpuos_create(0, h) == G.EDEVICE
    assert G.gpuos_launch_ops(desc(), 1, None, 0) == G.EDEVICE


def test_descriptor_builder_fields():
    w = W.make(3, small=True)
    d = streams.descriptors(w, 0x7f0000000000, 0x7e0000000000)
    assert len(d) == w.n_ops
    assert set(np.unique(d["opcode"])) == {G.OP[k] for k in ("rmsnorm", "rotary", "softmax", "add", "silu_mul")}
    assert (d["dtype"] == G.BF16).all()
    i = 1  # rotary(q)
    assert d["opcode"][i] == G.OP["rotary"] and d["rows"][i] == 16 and d["cols"][i] == 128
    assert d["in_"][i, 0] == 0x7e0000000000 + 2 * w.ops["in_off"][i, 0]
    assert d["dep"][i, 0] == 0 and d["dep"][i, 1] == G.NO_DEP
    for x in d:
        assert G.gpuos_validate(np.array([x], dtype=G.DESC)) == G.OK
    w1 = W.make(1, small=True)
    d1 = streams.descriptors(w1, 0x10000, 0x20000)
    assert (d1["nmicro"] == 2).all()
    assert (d1["micro"][:, 0] == G.MICRO["affine"]).all() and (d1["micro"][:, 1] == G.MICRO["relu"]).all()
