"""Element-by-element comparison of GPU results with the oracle (test infrastructure).

Tolerances (per element, applied per op on the GPU's own inputs):
  - fp32 elementwise ops (add, mul, scale, gelu, relu_affine, silu_mul,
    fused chains, rotary): |g - o| <= 1e-6 |o|; o == 0 requires g == 0.
  - fp32 softmax, RMSNorm, row max: |g - o| <= 1e-4 |o|.
  - LayerNorm: the relative bound (1e-4 for fp32, 2 bf16 ulp for bf16) is taken
    at the magnitude of the terms the output is computed from,
    (|x| + |mean|) inv_std |gamma| + |beta|: where x - mean and the final + beta
    cancel, no fp32 evaluation can meet a bound relative to the tiny result.
  - fp32 row sum: |g - o| <= 1e-4 sum|x| over the row.
  - bf16 outputs: |g - o| <= 2 ulp_bf16(o).
  - NaN must meet NaN; infinities must match exactly.
"""

from __future__ import annotations

import numpy as np

import oracle
from persistent_execution_b200 import workloads as W

EW = {"add", "mul", "scale", "gelu", "relu_affine", "silu_mul", "ew_chain", "rotary"}


def bf16_to_f64(h: np.ndarray) -> np.ndarray:
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def ulp_bf16(x: np.ndarray) -> np.ndarray:
    a = np.abs(x)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 7)


def _row_view(w, i, a32, a16):
    o = w.ops
    dt = int(o["dtype"][i])
    off = int(o["in_off"][i, 0])
    n = int(o["rows"][i] * o["cols"][i])
    x = a32[off:off + n].astype(np.float64) if dt == 0 else bf16_to_f64(a16[off:off + n])
    return x.reshape(int(o["rows"][i]), int(o["cols"][i]))


def _vec(w, i, k, a32, a16, n):
    off = int(w.ops["in_off"][i, k])
    return a32[off:off + n].astype(np.float64) if int(w.ops["dtype"][i]) == 0 else bf16_to_f64(a16[off:off + n])


def tolerance(w, i, a32, a16, ref: np.ndarray) -> np.ndarray:
    kind = W.KINDS[w.ops["kind"][i]]
    dt = int(w.ops["dtype"][i])
    if kind == "layernorm":
        x = _row_view(w, i, a32, a16)
        cols = x.shape[1]
        g = _vec(w, i, 1, a32, a16, cols)
        b = _vec(w, i, 2, a32, a16, cols)
        mu = x.mean(axis=1, keepdims=True)
        inv = 1.0 / np.sqrt(((x - mu) ** 2).mean(axis=1, keepdims=True) + float(w.ops["s"][i, 0]))
        scale = ((np.abs(x) + np.abs(mu)) * inv * np.abs(g) + np.abs(b)).ravel()
        return 2.0 * ulp_bf16(scale) if dt == 1 else 1e-4 * scale
    if dt == 1:
        return 2.0 * ulp_bf16(ref)
    if kind in EW:
        return 1e-6 * np.abs(ref)
    if kind == "rowsum":
        return 1e-4 * np.abs(_row_view(w, i, a32, a16)).sum(axis=1)
    return 1e-4 * np.abs(ref)


def gpu_output(w, i, a32, a16) -> np.ndarray:
    n = W.output_extent(w, i)
    off = int(w.ops["out_off"][i])
    return a32[off:off + n] if int(w.ops["dtype"][i]) == 0 else a16[off:off + n]


def compare(w, i, got_raw, ref_raw, a32, a16):
    """Returns (ok, worst ratio |g-o|/tol, index of the worst element)."""
    dt = int(w.ops["dtype"][i])
    g = got_raw.astype(np.float64) if dt == 0 else bf16_to_f64(got_raw)
    o = ref_raw.astype(np.float64) if dt == 0 else bf16_to_f64(ref_raw)
    nan_g, nan_o = np.isnan(g), np.isnan(o)
    if not np.array_equal(nan_g, nan_o):
        return False, np.inf, int(np.argmax(nan_g != nan_o))
    fin = ~nan_o
    inf_o = np.isinf(o) & fin
    if not np.array_equal(g[inf_o], o[inf_o]):
        return False, np.inf, int(np.nonzero(inf_o)[0][0])
    m = fin & ~inf_o
    tol = tolerance(w, i, a32, a16, o)
    err = np.abs(g - o)
    bad = m & (err > tol)
    if bad.any():
        j = int(np.argmax(np.where(bad, err / np.maximum(tol, 1e-300), 0)))
        return False, float(err[j] / max(tol[j], 1e-300)), j
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(m & (tol > 0), err / np.where(tol > 0, tol, 1), 0)
    return True, float(r.max()) if r.size else 0.0, -1


def check_ops(w, a32, a16, idx=None, limit_fail=5):
    """Teacher-forced check of ops `idx` (default all): each GPU output against
    the oracle applied to the GPU's own inputs. Returns a list of failures."""
    fails = []
    idx = range(w.n_ops) if idx is None else idx
    for i in idx:
        ref = oracle.apply(w, i, a32, a16)
        got = gpu_output(w, i, a32, a16)
        ok, worst, j = compare(w, i, got, ref, a32, a16)
        if not ok:
            fails.append((i, W.KINDS[w.ops["kind"][i]], worst, j))
            if len(fails) >= limit_fail:
                break
    return fails


EXACT = {"add", "mul", "scale", "relu_affine", "rowmax"}


def exact_ops(w) -> list:
    """Ops whose result is fixed bit for bit (single IEEE operations, fma chains, max)."""
    out = []
    for i in range(w.n_ops):
        k = W.KINDS[w.ops["kind"][i]]
        if k in EXACT or (k == "ew_chain" and int(w.ops["dtype"][i]) == 0 and
                          not ({W.M["gelu"], W.M["silu"]} & set(w.ops["prog"][i].tolist()))):
            out.append(i)
    return out


def bit_exact(w, a32, a16, r32, r16, idx=None) -> list:
    """Free-running comparison of the outputs of exact ops (default: all of
    them, see exact_ops) with an oracle run from the initial arenas; returns
    the ops whose outputs differ in any bit."""
    bad = []
    for i in (exact_ops(w) if idx is None else idx):
        g = gpu_output(w, i, a32, a16)
        r = gpu_output(w, i, r32, r16)
        if g.dtype == np.float32:
            g, r = g.view(np.uint32), r.view(np.uint32)
        if not np.array_equal(g, r):
            bad.append(i)
    return bad


def teacher_forcible(w) -> list:
    """Ops whose operands and output no later op overwrites (both survive in
    the final arenas, so the op can be checked on the GPU's own inputs)."""
    o = w.ops
    n = w.n_ops
    out0 = o["out_off"].astype(np.int64)
    out1 = out0 + np.array([W.output_extent(w, i) for i in range(n)], dtype=np.int64)
    dt = o["dtype"]
    keep = []
    idx = np.arange(n)
    for i in range(n):
        ok = not ((idx > i) & (dt == dt[i]) & (out0 < out1[i]) & (out1 > out0[i])).any()
        for k in range(3):
            if not ok:
                break
            a = int(o["in_off"][i, k])
            if a < 0:
                continue
            m = int(o["in_n"][i, k]) if k < 2 and o["in_n"][i, k] > 0 else int(o["rows"][i] * o["cols"][i])
            later = (np.arange(n) > i) & (dt == dt[i]) & (out0 < a + m) & (out1 > a)
            if later.any():
                ok = False
                break
        if ok:
            keep.append(i)
    return keep
