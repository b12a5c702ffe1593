"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle.

Every test compares element by element on seeded inputs with the tolerances
in tests/parity.py. Sizes span several work items and ragged tails.
"""

import numpy as np
import pytest
import torch

import oracle
from persistent_execution_b200 import build as B
from persistent_execution_b200 import gpuos as G
from persistent_execution_b200 import streams
from persistent_execution_b200 import trace as T
from persistent_execution_b200 import workloads as W

from . import gpu_util as U
from . import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()


# ------------------------------------------------------------------ single ops, edge sizes
EW_SIZES = [1, 3, 8, 4095, 4097, 65536, 3 * 65536 + 37, 3 * 262144 + 37]
EW_CASES = [("add", {}), ("mul", {}), ("scale", dict(scalars=(-1.75, 0, 0, 0))),
            ("gelu", {}), ("relu_affine", dict(scalars=(1.3, -0.2, 0, 0))), ("silu_mul", {}),
            ("ew_chain", dict(scalars=(0.7, 0.1, 2.0, 0), prog=("affine", "relu", "add1", "scale", "mul2"))),
            ("ew_chain", dict(scalars=(0.5, 0, 0, 0), prog=("gelu", "silu", "scale")))]


def _run_both(w):
    a32, a16, _, _ = U.run_persistent(w)
    fails = P.check_ops(w, a32, a16)
    b32, b16 = U.run_launches(w)
    fails_b = P.check_ops(w, b32, b16)
    return a32, a16, b32, b16, fails, fails_b


@pytest.mark.parametrize("dtype", [0, 1])
@pytest.mark.parametrize("kind,kw", EW_CASES, ids=[c[0] + str(i) for i, c in enumerate(EW_CASES)])
def test_elementwise_edge_sizes(kind, kw, dtype):
    for n in EW_SIZES:
        w = W.single_op(kind, dtype, 1, n, seed=n, **kw)
        _, _, _, _, f, fb = _run_both(w)
        assert not f, (n, f)
        assert not fb, (n, fb)


@pytest.mark.parametrize("dtype", [0, 1])
def test_elementwise_broadcast(dtype):
    for n, n0, n1 in [(1000, 7, 1000), (4097, 4097, 13), (65536 * 2 + 5, 65536 * 2 + 5, 3000), (96, 8, 16),
                      (600000, 600000, 3000)]:
        for kind in ("add", "mul", "silu_mul"):
            w = W.single_op(kind, dtype, 1, n, bcast=(n0, n1), seed=n + n1)
            _, _, _, _, f, fb = _run_both(w)
            assert not f and not fb, (kind, n, n0, n1, f, fb)


@pytest.mark.parametrize("sd", [1.0, 4.0, 12.0])
def test_gelu_fp32_wide_range(sd):
    # the fp32 gelu path over the bulk (|x| <= 10) and the double-precision
    # tails, within 1e-6 relative of the oracle element by element
    w = W.single_op("gelu", 0, 1, 1 << 20, seed=int(sd * 10), sd=sd)
    _, _, _, _, f, fb = _run_both(w)
    assert not f and not fb, (f, fb)


ROW_SHAPES = [(1, 1), (3, 5), (7, 1000), (16, 1024), (1, 2048), (8, 4096), (5, 4100), (2000, 64),
              (3, 8192), (9, 65536 + 8)]


@pytest.mark.parametrize("dtype", [0, 1])
@pytest.mark.parametrize("kind", ["rowsum", "rowmax", "softmax", "rmsnorm", "layernorm"])
def test_row_ops(kind, dtype):
    for rows, cols in ROW_SHAPES:
        sc = (1e-6 if kind == "rmsnorm" else 1e-5, 0, 0, 0)
        w = W.single_op(kind, dtype, rows, cols, seed=rows * 7 + cols, scalars=sc, sd=2.0)
        _, _, _, _, f, fb = _run_both(w)
        assert not f and not fb, (kind, rows, cols, f, fb)


@pytest.mark.parametrize("dtype", [0, 1])
def test_rotary(dtype):
    for rows, cols, pos in [(16, 128, 1023), (1, 128, 0), (3, 6, 7), (40, 64, 517), (2048, 128, 924)]:
        w = W.single_op("rotary", dtype, rows, cols, pos=pos, scalars=(10000.0, 0, 0, 0), seed=pos + rows)
        a32, a16, _, _, f, fb = _run_both(w)
        assert not f and not fb, (rows, cols, pos, f, fb)
        if pos == 0:  # identity, bit for bit
            x = P.gpu_output(w, 0, a32, a16)
            src = (a32 if dtype == 0 else a16)[w.ops["in_off"][0, 0]:][:x.size]
            assert np.array_equal(x, src)


# ------------------------------------------------------------------ streams (reduced sizes)
@pytest.mark.parametrize("config", [1, 2, 3, 4, 5])
def test_config_small_drain(config):
    w = W.make(config, small=True)
    a32, a16, tr, st = U.run_persistent(w, trace=True)
    fails = P.check_ops(w, a32, a16, idx=P.teacher_forcible(w) if config == 5 else None)
    assert not fails, fails
    # ordering audit and item coverage from the device event log
    assert (tr["id"] == np.arange(1, w.n_ops + 1) + (tr["id"][0] - 1)).all()
    assert T.violations(w.ops["dep"], tr["t_start"], tr["t_end"]) == []
    # each work item ran exactly once: items per op equal the host's split
    d = streams.descriptors(w, 1 << 20, 1 << 21)
    items = np.array([G.gpuos_work_items(d[i:i + 1]) for i in range(w.n_ops)])
    assert (tr["items"] == items).all()
    if config in (1, 5):  # chains of bit-exact ops: free-running equality with the oracle
        r32, r16 = oracle.run(w)
        assert P.bit_exact(w, a32, a16, r32, r16) == []


def test_config_small_live_mode():
    for config in (2, 3, 4):
        w = W.make(config, small=True)
        a32, a16, _, st = U.run_persistent(w, mode="live", batch=97)
        assert not P.check_ops(w, a32, a16)


def test_chain_affinity_keeps_chains_on_one_cta():
    w = W.make(1, small=True)
    a32, a16, tr, st = U.run_persistent(w, trace=True)
    assert not P.check_ops(w, a32, a16)
    # all but the first op of the chain are taken as runs by the CTA that ran the predecessor
    assert (tr["claim"][1:] == 1).mean() > 0.9, st
    assert len(np.unique(tr["cta"])) <= 3


@pytest.mark.parametrize("dtype", [0, 1])
@pytest.mark.parametrize("n", [4096, 2048, 8192, 256 * 16 * 12, 4100, 300])
def test_dependent_elementwise_chains_bit_exact(dtype, n):
    # Chains of fused relu-affine ops and adds, each reading the previous
    # output as its first or second operand, at sizes of whole tiles, partial
    # warps and ragged tails. Every output must equal the oracle's, bit for bit.
    b = W._Builder("forwarding", 5)
    rng = b.rng

    def data():
        v = rng.standard_normal(n, dtype=np.float32)
        return v if dtype == 0 else W.bf16_bits_trunc(v)

    src = b.alloc_input(dtype, data())
    other = b.alloc_input(dtype, data())
    prev = -1
    for i in range(60):
        out = b.alloc_output(dtype, n)
        if i % 5 == 4:  # the previous output as second operand
            prev = b.add_op("add", dtype, [other, src], out, 1, n, in_n=(n, n), deps=[prev])
        elif i % 3 == 2:
            prev = b.add_op("add", dtype, [src, other], out, 1, n, in_n=(n, n), deps=[prev])
        else:
            a, c = rng.uniform(-1.5, 1.5, 2)
            prev = b.add_op("ew_chain", dtype, [src], out, 1, n, in_n=(n, 0), s=(a, c, 0, 0),
                            prog=("affine", "relu"), deps=[prev])
        src = out
    w = b.finish({})
    a32, a16, _, _ = U.run_persistent(w)
    assert not P.check_ops(w, a32, a16)
    r32, r16 = oracle.run(w)
    assert P.bit_exact(w, a32, a16, r32, r16) == []


@pytest.mark.parametrize("config", [1, 2, 5])
def test_fused_pairs_match_unfused(config):
    # consecutive dependent scalar elementwise ops are fused into pairs at
    # submit; outputs must be bit-identical with fusion off, and match the oracle
    w = W.make(config, small=True)
    a32, a16, _, _ = U.run_persistent(w)
    assert not P.check_ops(w, a32, a16, idx=P.teacher_forcible(w) if config == 5 else None)
    b32, b16, _, _ = U.run_persistent(w, cfg=dict(flags=G.CFG_NO_FUSION))
    assert np.array_equal(a32.view(np.uint32), b32.view(np.uint32)) and np.array_equal(a16, b16)
    if config == 1:
        r32, r16 = oracle.run(w)
        assert P.bit_exact(w, a32, a16, r32, r16) == []


@pytest.mark.parametrize("mode", ["drain", "live"])
def test_chain_handoff_interleaved_streams(mode):
    # config 4's request chains are interleaved, so a claimed op's predecessor
    # usually runs on another CTA: the claimer posts it to that CTA's mailbox.
    w = W.make(4, small=True)
    a32, a16, tr, st = U.run_persistent(w, mode=mode, trace=True, batch=101)
    assert not P.check_ops(w, a32, a16)
    assert T.violations(w.ops["dep"], tr["t_start"], tr["t_end"]) == []
    handed = tr["claim"] == 3
    assert handed.any(), np.bincount(tr["claim"])
    # a handed-off op runs on the CTA that ran its predecessor
    dep = w.ops["dep"][:, 0]
    idx = np.nonzero(handed & (dep >= 0))[0]
    assert (tr["cta"][idx] == tr["cta"][dep[idx]]).mean() > 0.99
    # the same stream without hand-off gives bit-identical outputs
    b32, b16, _, _ = U.run_persistent(w, mode=mode, cfg=dict(flags=G.CFG_NO_HANDOFF), batch=101)
    assert P.bit_exact(w, a32, a16, b32, b16) == []


@pytest.mark.parametrize("config", [2, 4])
def test_baselines_match_persistent(config):
    w = W.make(config, small=True)
    a32, a16, _, _ = U.run_persistent(w)
    for mode in (None, 0, 1):
        b32, b16 = U.run_launches(w, graph_mode=mode)
        assert P.bit_exact(w, a32, a16, b32, b16) == [], mode


@pytest.mark.parametrize("mode", ["drain", "live"])
def test_long_dag_with_multi_item_ops(mode):
    # a long DAG stream with 1024-element items: most ops are multi-item
    # (opened in submission order, joined by many CTAs) between single-item ones
    w = W.make(2, n_ops=6000)
    a32, a16, tr, st = U.run_persistent(w, mode=mode, trace=True, batch=1500,
                                        cfg={"elem_chunk": 1024, "ring_capacity": 8192})
    assert not P.check_ops(w, a32, a16)
    assert T.violations(w.ops["dep"], tr["t_start"], tr["t_end"]) == []
    d = streams.descriptors(w, 1 << 20, 1 << 21)
    c = G.default_config(elem_chunk=1024)
    items = np.array([G.gpuos_work_items(d[i:i + 1], c) for i in range(w.n_ops)])
    assert (tr["items"] == items).all()
    assert (items > 1).mean() > 0.3


def test_large_multi_item_ops_and_chunk_sizes():
    # elementwise op of 5 items followed by dependants, with small chunks so many CTAs join
    for cfg in ({"elem_chunk": 4096, "row_chunk": 4096}, {}):
        w = W.make(5, n_groups=3, vec=(1 << 20) + 37, mat=1024)
        a32, a16, tr, st = U.run_persistent(w, trace=True, cfg=cfg)
        assert not P.check_ops(w, a32, a16, idx=P.teacher_forcible(w))
        r32, r16 = oracle.run(w)
        assert P.bit_exact(w, a32, a16, r32, r16) == []
