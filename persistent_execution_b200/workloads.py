"""Seeded synthetic op streams: the only module shared by the CUDA path and the oracle.

This module draws random numbers and lays out buffers. It holds none of the
method's arithmetic: it never evaluates an op. Each side (the CUDA runtime's
descriptor builder and the CPU oracle's adapter) maps the op-kind names below to
its own codes.

Workloads follow the five stream shapes of the persistent-kernel task (GPUOS,
arXiv 2604.17861, abstract: "many small tensor operations ... micro-batched
inference and attention patterns"; "Launch Overhead and Fusion", section
"Fusion", for y = relu(a*x+b)). Sizes and distributions not fixed by the pages
are readings, listed in the design doc.

Representation
--------------
All fp32 tensors of a workload live in one host array ``arena_f32`` and all
bf16 tensors in ``arena_bf16`` (uint16 bit patterns). An op names its operands
by element offsets into the arena of its dtype. Offsets are multiples of
``ALIGN`` elements so that every operand starts on a 256-byte boundary.
Inputs occupy the front of each arena ([0, n_init_*)); outputs follow and
start as zeros.

``ops`` is a dict of equal-length numpy columns:

kind      int16  index into KINDS
dtype     int8   0 = fp32, 1 = bf16
in_off    (n,3) int64  element offsets of operands 0..2, -1 = unused
out_off   int64  element offset of the output
rows,cols int64  shape; elementwise ops use rows=1, cols=n
in_n      (n,2) int64  element counts of operands 0 and 1 (modulo broadcast)
s         (n,4) float32 scalars; meaning per kind (SCALAR_USE)
pos       int32  rotary position
prog      (n,8) int8   fused-chain program as indices into MICRO, -1 = end
dep       (n,2) int64  indices of earlier ops in this workload, -1 = none
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

KINDS = (
    "add",          # y = x0 + x1
    "mul",          # y = x0 * x1
    "scale",        # y = s0 * x0
    "gelu",         # erf form
    "relu_affine",  # y = relu(s0 * x0 + s1)
    "silu_mul",     # y = silu(x0) * x1
    "ew_chain",     # fused elementwise micro-op program over x0 (and x1, x2)
    "rowsum",       # [rows, cols] -> [rows]
    "rowmax",       # [rows, cols] -> [rows]
    "softmax",      # per row
    "rmsnorm",      # per row, weight = operand 1, eps = s0
    "layernorm",    # per row, gamma = operand 1, beta = operand 2, eps = s0
    "rotary",       # [heads, 128] half-split pairs, base = s0, position = pos
)
K = {name: i for i, name in enumerate(KINDS)}

# Micro-ops of a fused elementwise chain. The accumulator starts as x0.
# Scalar-consuming micro-ops take the op's scalars s0, s1, ... in program order.
MICRO = (
    "affine",   # acc = fma(s[k], acc, s[k+1]); k += 2
    "scale",    # acc = acc * s[k]; k += 1
    "adds",     # acc = acc + s[k]; k += 1
    "relu",     # acc = max(acc, +0)
    "gelu",     # erf-form gelu of acc
    "silu",     # acc * sigmoid(acc)
    "add1",     # acc = acc + x1
    "mul1",     # acc = acc * x1
    "add2",     # acc = acc + x2
    "mul2",     # acc = acc * x2
)
M = {name: i for i, name in enumerate(MICRO)}

SCALAR_USE = {
    "scale": ("s",),
    "relu_affine": ("a", "b"),
    "rmsnorm": ("eps",),
    "layernorm": ("eps",),
    "rotary": ("base",),
}

DTYPES = ("f32", "bf16")
ALIGN = 64  # elements; 256 B for fp32, 128 B for bf16

RMSNORM_EPS = 1e-6
LAYERNORM_EPS = 1e-5
ROTARY_BASE = 10000.0
HEAD_DIM = 128


@dataclass
class Workload:
    name: str
    seed: int
    arena_f32: np.ndarray
    arena_bf16: np.ndarray
    n_init_f32: int
    n_init_bf16: int
    ops: dict
    meta: dict = field(default_factory=dict)

    @property
    def n_ops(self) -> int:
        return int(self.ops["kind"].shape[0])

    def op(self, i: int) -> dict:
        return {k: v[i] for k, v in self.ops.items()}


def _round_up(x: int, a: int = ALIGN) -> int:
    return (x + a - 1) // a * a


def bf16_bits_trunc(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns by truncating fp32 toward zero (input preparation only)."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


class _Builder:
    """Accumulates arena allocations and op rows."""

    def __init__(self, name: str, seed: int):
        self.name = name
        self.seed = seed
        self.rng = np.random.default_rng(seed)
        self.size = [0, 0]          # allocated elements per dtype
        self.init_chunks = [[], []]  # (offset, array) for input data
        self.init_end = [0, 0]
        self.rows = []

    def alloc_input(self, dt: int, data: np.ndarray) -> int:
        assert self.size[dt] == self.init_end[dt], "inputs must be allocated before outputs"
        off = self.size[dt]
        n = int(data.shape[0])
        self.init_chunks[dt].append((off, data))
        self.size[dt] = _round_up(off + n)
        self.init_end[dt] = self.size[dt]
        return off

    def alloc_output(self, dt: int, n: int) -> int:
        off = self.size[dt]
        self.size[dt] = _round_up(off + n)
        return off

    def add_op(self, kind, dtype, ins, out_off, rows, cols, in_n=(0, 0), s=(0, 0, 0, 0),
               pos=0, prog=(), deps=()):
        ins = list(ins) + [-1] * (3 - len(ins))
        deps = [d for d in deps if d is not None and d >= 0]
        assert len(deps) <= 2
        deps = deps + [-1] * (2 - len(deps))
        prog = list(prog)
        assert len(prog) <= 8
        self.rows.append((K[kind], dtype, ins, out_off, rows, cols, list(in_n), list(s), pos,
                          [M[p] for p in prog] + [-1] * (8 - len(prog)), deps))
        return len(self.rows) - 1

    def finish(self, meta=None) -> Workload:
        n = len(self.rows)
        ops = {
            "kind": np.array([r[0] for r in self.rows], dtype=np.int16),
            "dtype": np.array([r[1] for r in self.rows], dtype=np.int8),
            "in_off": np.array([r[2] for r in self.rows], dtype=np.int64).reshape(n, 3),
            "out_off": np.array([r[3] for r in self.rows], dtype=np.int64),
            "rows": np.array([r[4] for r in self.rows], dtype=np.int64),
            "cols": np.array([r[5] for r in self.rows], dtype=np.int64),
            "in_n": np.array([r[6] for r in self.rows], dtype=np.int64).reshape(n, 2),
            "s": np.array([r[7] for r in self.rows], dtype=np.float32).reshape(n, 4),
            "pos": np.array([r[8] for r in self.rows], dtype=np.int32),
            "prog": np.array([r[9] for r in self.rows], dtype=np.int8).reshape(n, 8),
            "dep": np.array([r[10] for r in self.rows], dtype=np.int64).reshape(n, 2),
        }
        arenas = []
        for dt in (0, 1):
            total = max(self.size[dt], ALIGN)
            a = np.zeros(total, dtype=np.float32 if dt == 0 else np.uint16)
            for off, data in self.init_chunks[dt]:
                a[off:off + data.shape[0]] = data
            arenas.append(a)
        return Workload(self.name, self.seed, arenas[0], arenas[1],
                        self.init_end[0], self.init_end[1], ops, meta or {})


# --------------------------------------------------------------------------
# Config 1: dependent chain of fused relu(a*x+b) ops
# --------------------------------------------------------------------------
def config1(n_ops: int = 1000, n: int = 4096, seed: int = 0) -> Workload:
    """Chain y_i = relu(a_i * y_{i-1} + b_i) on an fp32 vector; x ~ N(0,1), a,b ~ U(-2,2).

    Each op is a fused micro-op chain [affine, relu] and writes its own output
    buffer so that every intermediate can be checked.
    """
    b = _Builder("config1", seed)
    x = b.rng.standard_normal(n, dtype=np.float32)
    ab = b.rng.uniform(-2.0, 2.0, size=(n_ops, 2)).astype(np.float32)
    src = b.alloc_input(0, x)
    prev = -1
    for i in range(n_ops):
        out = b.alloc_output(0, n)
        prev = b.add_op("ew_chain", 0, [src], out, 1, n, in_n=(n, 0),
                        s=(ab[i, 0], ab[i, 1], 0, 0), prog=("affine", "relu"),
                        deps=[prev])
        src = out
    return b.finish({"config": 1, "n": n})


# --------------------------------------------------------------------------
# Config 2: random DAG of mixed fp32 elementwise ops
# --------------------------------------------------------------------------
_C2_KINDS = ("add", "mul", "gelu", "scale", "relu_affine")
_BINARY = {"add", "mul"}


def config2(n_ops: int = 20000, nmin: int = 256, nmax: int = 65536, seed: int = 1) -> Workload:
    """Random DAG; kind ~ U{add,mul,gelu,scale,relu_affine}; n ~ logU[nmin,nmax];
    each op depends on 0..2 uniformly chosen earlier ops; fresh inputs ~ N(0,1).

    Operand slot k reads the output of dep[k] when present (modulo broadcast to
    this op's size), else a fresh N(0,1) tensor of this op's size. Unary ops
    read slot 0 only; their second dependency orders without data flow.
    """
    b = _Builder("config2", seed)
    rng = b.rng
    kinds = rng.integers(0, len(_C2_KINDS), size=n_ops)
    ns = np.floor(np.exp(rng.uniform(math.log(nmin), math.log(nmax + 1), size=n_ops))).astype(np.int64)
    ns = np.clip(ns, nmin, nmax)
    ndeps = rng.integers(0, 3, size=n_ops)
    scal = rng.uniform(-2.0, 2.0, size=(n_ops, 2)).astype(np.float32)
    deps = []
    for i in range(n_ops):
        k = min(int(ndeps[i]), i)
        if k == 0:
            deps.append([])
        elif k == 1:
            deps.append([int(rng.integers(0, i))])
        else:  # two distinct earlier ops, uniformly
            d0 = int(rng.integers(0, i))
            d1 = int(rng.integers(0, i - 1))
            d1 = d1 + 1 if d1 >= d0 else d1
            deps.append(sorted([d0, d1]))
    # fresh inputs first (arena inputs precede outputs)
    fresh = {}
    for i in range(n_ops):
        kind = _C2_KINDS[kinds[i]]
        nslots = 2 if kind in _BINARY else 1
        for slot in range(nslots):
            if slot >= len(deps[i]):
                fresh[(i, slot)] = b.alloc_input(0, rng.standard_normal(int(ns[i]), dtype=np.float32))
    out_off = [b.alloc_output(0, int(ns[i])) for i in range(n_ops)]
    for i in range(n_ops):
        kind = _C2_KINDS[kinds[i]]
        nslots = 2 if kind in _BINARY else 1
        ins, in_n = [], []
        for slot in range(nslots):
            if slot < len(deps[i]):
                d = deps[i][slot]
                ins.append(out_off[d])
                in_n.append(int(ns[d]))
            else:
                ins.append(fresh[(i, slot)])
                in_n.append(int(ns[i]))
        in_n += [0] * (2 - len(in_n))
        if kind == "scale":
            s = (scal[i, 0], 0, 0, 0)
        elif kind == "relu_affine":
            s = (scal[i, 0], scal[i, 1], 0, 0)
        else:
            s = (0, 0, 0, 0)
        b.add_op(kind, 0, ins, out_off[i], 1, int(ns[i]), in_n=in_n, s=s, deps=deps[i])
    return b.finish({"config": 2})


# --------------------------------------------------------------------------
# Config 3: non-GEMM op stream of a batch-1 bf16 decode step
# --------------------------------------------------------------------------
def config3(steps: int = 100, layers: int = 32, hidden: int = 2048, heads: int = 16,
            ctx: int = 1024, inter: int = 5632, pos0: int = 924, seed: int = 2) -> Workload:
    """steps x layers x 2 blocks x 8 ops, all bf16, one dependent chain.

    Block: RMSNorm(h), rotary(q), rotary(k), softmax(scores), h=add(h,o),
    RMSNorm(h), silu_mul(g,u), h=add(h,d). GEMM outputs are seeded stand-in
    tensors reused across steps; q,k,o,d,g,u ~ N(0,1), scores ~ N(0,3),
    RMSNorm weights ~ U(0.5,1.5); h0 ~ N(0,1) per step; position 924+step.
    Each op depends on its predecessor; residual adds also depend on the op
    that last wrote h. Every op writes its own output tensor.
    """
    b = _Builder("config3", seed)
    rng = b.rng
    hd = HEAD_DIM
    assert heads * hd == hidden
    nblk = layers * 2

    def nrm(n, sd=1.0):
        return bf16_bits_trunc(rng.standard_normal(n, dtype=np.float32) * np.float32(sd))

    blk = []
    for _ in range(nblk):
        blk.append({
            "q": b.alloc_input(1, nrm(heads * hd)),
            "k": b.alloc_input(1, nrm(heads * hd)),
            "scores": b.alloc_input(1, nrm(heads * ctx, 3.0)),
            "o": b.alloc_input(1, nrm(hidden)),
            "d": b.alloc_input(1, nrm(hidden)),
            "g": b.alloc_input(1, nrm(inter)),
            "u": b.alloc_input(1, nrm(inter)),
            "w1": b.alloc_input(1, bf16_bits_trunc(rng.uniform(0.5, 1.5, hidden).astype(np.float32))),
            "w2": b.alloc_input(1, bf16_bits_trunc(rng.uniform(0.5, 1.5, hidden).astype(np.float32))),
        })
    h0 = [b.alloc_input(1, nrm(hidden)) for _ in range(steps)]
    prev = -1
    for st in range(steps):
        h_off, h_writer = h0[st], -1
        pos = pos0 + st
        for j in range(nblk):
            t = blk[j]
            out = b.alloc_output(1, hidden)
            prev = b.add_op("rmsnorm", 1, [h_off, t["w1"]], out, 1, hidden,
                            in_n=(hidden, hidden), s=(RMSNORM_EPS, 0, 0, 0), deps=[prev])
            out = b.alloc_output(1, heads * hd)
            prev = b.add_op("rotary", 1, [t["q"]], out, heads, hd, in_n=(heads * hd, 0),
                            s=(ROTARY_BASE, 0, 0, 0), pos=pos, deps=[prev])
            out = b.alloc_output(1, heads * hd)
            prev = b.add_op("rotary", 1, [t["k"]], out, heads, hd, in_n=(heads * hd, 0),
                            s=(ROTARY_BASE, 0, 0, 0), pos=pos, deps=[prev])
            out = b.alloc_output(1, heads * ctx)
            prev = b.add_op("softmax", 1, [t["scores"]], out, heads, ctx,
                            in_n=(heads * ctx, 0), deps=[prev])
            out = b.alloc_output(1, hidden)
            prev = b.add_op("add", 1, [h_off, t["o"]], out, 1, hidden, in_n=(hidden, hidden),
                            deps=[prev, h_writer] if h_writer >= 0 and h_writer != prev else [prev])
            h_off, h_writer = out, prev
            out = b.alloc_output(1, hidden)
            prev = b.add_op("rmsnorm", 1, [h_off, t["w2"]], out, 1, hidden,
                            in_n=(hidden, hidden), s=(RMSNORM_EPS, 0, 0, 0), deps=[prev])
            out = b.alloc_output(1, inter)
            prev = b.add_op("silu_mul", 1, [t["g"], t["u"]], out, 1, inter,
                            in_n=(inter, inter), deps=[prev])
            out = b.alloc_output(1, hidden)
            prev = b.add_op("add", 1, [h_off, t["d"]], out, 1, hidden, in_n=(hidden, hidden),
                            deps=[prev, h_writer])
            h_off, h_writer = out, prev
    return b.finish({"config": 3, "steps": steps, "layers": layers})


# --------------------------------------------------------------------------
# Config 4: dynamic-shape micro-batched serving stream
# --------------------------------------------------------------------------
def config4(n_ops: int = 100000, streams: int = 64, pool_elems: int = 16 << 20,
            hidden: int = 1024, lmin: int = 128, lmax: int = 4096, bmax: int = 8,
            seed: int = 3) -> Workload:
    """Round-robin interleaving of `streams` request chains; op i belongs to
    stream i % streams and depends on that stream's previous op.

    Kinds uniform over {softmax, layernorm, add}; batch B ~ U{1..bmax};
    softmax rows of length L ~ U{lmin..lmax} drawn from an N(0,2) pool;
    LayerNorm [B, hidden] from an N(0,1) pool with gamma ~ U(0.5,1.5) and
    beta ~ N(0,0.1) pools; add(prev_out, fresh N(0,1)) of shape [B, hidden]
    with modulo broadcast from the predecessor's output. Fresh operands are
    windows at seeded offsets into the pools.
    """
    b = _Builder("config4", seed)
    rng = b.rng
    pools = {
        "sm": b.alloc_input(0, rng.standard_normal(pool_elems, dtype=np.float32) * np.float32(2.0)),
        "n01": b.alloc_input(0, rng.standard_normal(pool_elems, dtype=np.float32)),
        "gamma": b.alloc_input(0, rng.uniform(0.5, 1.5, pool_elems).astype(np.float32)),
        "beta": b.alloc_input(0, rng.standard_normal(pool_elems, dtype=np.float32) * np.float32(0.1)),
    }

    def window(pool: str, n: int) -> int:
        hi = (pool_elems - n) // ALIGN
        return pools[pool] + int(rng.integers(0, hi + 1)) * ALIGN

    kinds = rng.integers(0, 3, size=n_ops)
    bs = rng.integers(1, bmax + 1, size=n_ops)
    ls = rng.integers(lmin, lmax + 1, size=n_ops)
    last = [-1] * streams
    out_n = []
    for i in range(n_ops):
        sidx = i % streams
        prev = last[sidx]
        kind = ("softmax", "layernorm", "add")[kinds[i]]
        B = int(bs[i])
        if kind == "softmax":
            L = int(ls[i])
            n = B * L
            out = b.alloc_output(0, n)
            b.add_op("softmax", 0, [window("sm", n)], out, B, L, in_n=(n, 0), deps=[prev])
        elif kind == "layernorm":
            n = B * hidden
            out = b.alloc_output(0, n)
            b.add_op("layernorm", 0, [window("n01", n), window("gamma", hidden), window("beta", hidden)],
                     out, B, hidden, in_n=(n, hidden), s=(LAYERNORM_EPS, 0, 0, 0), deps=[prev])
        else:
            n = B * hidden
            out = b.alloc_output(0, n)
            if prev >= 0:
                src, src_n = b.rows[prev][3], out_n[prev]
            else:
                src, src_n = window("n01", n), n
            b.add_op("add", 0, [src, window("n01", n)], out, 1, n, in_n=(src_n, n), deps=[prev])
        out_n.append(n)
        last[sidx] = i
    return b.finish({"config": 4, "streams": streams})


# --------------------------------------------------------------------------
# Config 5: large-op stress against the HBM roofline
# --------------------------------------------------------------------------
def config5(n_groups: int = 64, vec: int = 64 << 20, mat: int = 8192, seed: int = 4) -> Workload:
    """Groups of four ops C,S,C,M: C is a fused [affine, relu] op on a `vec`-element
    fp32 vector in one dependent ping-pong chain x -> A -> B -> A ...; S and M
    are row sum and row max of a fixed [mat, mat] N(0,1) matrix, independent.
    """
    b = _Builder("config5", seed)
    rng = b.rng
    x = b.alloc_input(0, rng.standard_normal(vec, dtype=np.float32))
    mtx = b.alloc_input(0, rng.standard_normal(mat * mat, dtype=np.float32))
    ab = rng.uniform(-2.0, 2.0, size=(2 * n_groups, 2)).astype(np.float32)
    pp = [b.alloc_output(0, vec), b.alloc_output(0, vec)]
    src, prev, c = x, -1, 0
    for g in range(n_groups):
        for kind in ("C", "S", "C", "M"):
            if kind == "C":
                dst = pp[c % 2]
                prev = b.add_op("ew_chain", 0, [src], dst, 1, vec, in_n=(vec, 0),
                                s=(ab[c, 0], ab[c, 1], 0, 0), prog=("affine", "relu"), deps=[prev])
                src = dst
                c += 1
            else:
                out = b.alloc_output(0, mat)
                b.add_op("rowsum" if kind == "S" else "rowmax", 0, [mtx], out, mat, mat,
                         in_n=(mat * mat, 0))
    return b.finish({"config": 5, "vec": vec, "mat": mat})


CONFIGS = {1: config1, 2: config2, 3: config3, 4: config4, 5: config5}

# Reduced sizes with the same structure, for tests whose oracle runs in seconds.
SMALL = {
    1: dict(n_ops=200, n=4096),
    2: dict(n_ops=600, nmin=256, nmax=65536),
    3: dict(steps=2, layers=4),
    4: dict(n_ops=2000, streams=64, pool_elems=1 << 20),
    5: dict(n_groups=2, vec=(1 << 20) + 37, mat=1024),
}


def make(config: int, small: bool = False, **kw) -> Workload:
    args = dict(SMALL[config]) if small else {}
    args.update(kw)
    return CONFIGS[config](**args)


def single_op(kind: str, dtype: int, rows: int, cols: int, seed: int = 11,
              bcast=(None, None), scalars=(0.0, 0.0, 0.0, 0.0), pos: int = 0,
              prog=(), sd: float = 1.0) -> Workload:
    """One op on fresh N(0, sd) operands, for edge-size tests.

    bcast[k] gives operand k's element count when it differs from the op's
    size (modulo broadcast); weights of norms are U(0.5,1.5).
    """
    b = _Builder(f"{kind}_{rows}x{cols}", seed)
    rng = b.rng
    n = rows * cols

    def data(m, lo=None, hi=None):
        v = (rng.uniform(lo, hi, m).astype(np.float32) if lo is not None
             else rng.standard_normal(m, dtype=np.float32) * np.float32(sd))
        return v if dtype == 0 else bf16_bits_trunc(v)

    ins, in_n = [], [0, 0]
    if kind in ("rmsnorm",):
        ins = [b.alloc_input(dtype, data(n)), b.alloc_input(dtype, data(cols, 0.5, 1.5))]
        in_n = [n, cols]
    elif kind == "layernorm":
        ins = [b.alloc_input(dtype, data(n)), b.alloc_input(dtype, data(cols, 0.5, 1.5)),
               b.alloc_input(dtype, data(cols))]
        in_n = [n, cols]
    elif kind in ("add", "mul", "silu_mul") or (kind == "ew_chain" and any(
            p in ("add1", "mul1", "add2", "mul2") for p in prog)):
        n0 = bcast[0] or n
        n1 = bcast[1] or n
        ins = [b.alloc_input(dtype, data(n0)), b.alloc_input(dtype, data(n1))]
        if kind == "ew_chain":
            ins.append(b.alloc_input(dtype, data(n)))
        in_n = [n0, n1]
    else:
        n0 = bcast[0] or n
        ins = [b.alloc_input(dtype, data(n0))]
        in_n = [n0, 0]
    out_n = rows if kind in ("rowsum", "rowmax") else n
    out = b.alloc_output(dtype, out_n)
    b.add_op(kind, dtype, ins, out, rows, cols, in_n=in_n, s=scalars, pos=pos, prog=prog)
    return b.finish({"single": kind})


def output_extent(w: Workload, i: int) -> int:
    """Element count of op i's output."""
    kind = KINDS[w.ops["kind"][i]]
    if kind in ("rowsum", "rowmax"):
        return int(w.ops["rows"][i])
    return int(w.ops["rows"][i] * w.ops["cols"][i])
