"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test names the fact that pins it: a worked example printed on the pages,
a closed form, an identity, a library routine, or brute force. A plausible
mistake in an op (a dropped term, a wrong sign or index, a transposed
operand, a wrong rounding) fails at least one of these.
"""

import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.special as sps
import torch

import oracle
from persistent_execution_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def one(kind, dtype, rows, cols, ins, s=(0, 0, 0, 0), pos=0, prog=(), in_n=None):
    """Runs a single op on explicit operand arrays; returns the output array."""
    b = W._Builder("pin", 0)
    offs = []
    for a in ins:
        a = np.asarray(a, dtype=np.float32) if dtype == 0 else np.asarray(a, dtype=np.uint16)
        offs.append(b.alloc_input(dtype, a))
    n_out = rows if kind in ("rowsum", "rowmax") else rows * cols
    out = b.alloc_output(dtype, n_out)
    if in_n is None:
        in_n = [len(ins[0]), len(ins[1]) if len(ins) > 1 else 0]
    b.add_op(kind, dtype, offs, out, rows, cols, in_n=in_n, s=s, pos=pos, prog=prog)
    w = b.finish()
    a32, a16 = oracle.run(w)
    return (a32 if dtype == 0 else a16)[out:out + n_out]


def f32(x):
    return np.float32(x)


# --------------------------------------------------------------------------
# relu(a*x+b): "Launch Overhead and Fusion", section "Code" (fusion.go) uses
# x_i = (i mod 100) - 50, a = 1.5, b = 0.5. Every result is a multiple of 0.5
# with |y| <= 74.5, so the exact rational value is the fp32 result.
# --------------------------------------------------------------------------
def test_relu_affine_fusion_demo_values():
    fx = open(__file__.replace("test_oracle_pins.py", "golden/fusion_demo.txt")).read()
    consts = dict(l.split("=", 1) for l in fx.splitlines() if "=" in l and not l.startswith("#"))
    a, b = float(consts["a"]), float(consts["b"])
    n = 1000
    x = np.array([(i % 100) - 50 for i in range(n)], dtype=np.float32)
    y = one("relu_affine", 0, 1, n, [x], s=(a, b, 0, 0))
    exact = [max(Fraction(a) * Fraction(int(v)) + Fraction(b), Fraction(0)) for v in x]
    assert all(float(e) == float(g) for e, g in zip(exact, y))
    assert y.max() == 74.0 and y.min() == 0.0
    # the same chain written as fused micro-ops gives the same bits
    y2 = one("ew_chain", 0, 1, n, [x], s=(a, b, 0, 0), prog=("affine", "relu"))
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32))


def test_relu_affine_is_single_rounding_fma():
    # a*x+b with one rounding differs from round(round(a*x)+b) on these inputs;
    # the exact rational value decides which is right.
    rng = np.random.default_rng(5)
    x = rng.standard_normal(20000).astype(np.float32)
    a, b = f32(1.1), f32(-0.3)
    y = one("relu_affine", 0, 1, x.size, [x], s=(a, b, 0, 0))
    exact = np.array([float(max(Fraction(float(a)) * Fraction(float(v)) + Fraction(float(b)), 0))
                      for v in x], dtype=np.float64).astype(np.float32)
    assert np.array_equal(y, exact)
    two_step = np.maximum((a * x) + b, 0).astype(np.float32)
    assert (two_step != y).any()


def test_relu_sign_cases():
    x = np.array([-1.0, 0.0, -0.0, 1.0, np.nan, -np.inf, np.inf], dtype=np.float32)
    y = one("relu_affine", 0, 1, x.size, [x], s=(1.0, 0.0, 0, 0))
    assert np.signbit(y[:3]).sum() == 0 and (y[:3] == 0).all()
    assert y[3] == 1.0 and np.isnan(y[4]) and y[5] == 0 and y[6] == np.inf


# --------------------------------------------------------------------------
# add / mul / scale: IEEE fp32 round-to-nearest, as numpy float32 arithmetic.
# --------------------------------------------------------------------------
def test_binary_ops_match_ieee_fp32():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal(5000) * np.exp(rng.uniform(-30, 30, 5000))).astype(np.float32)
    z = (rng.standard_normal(5000) * np.exp(rng.uniform(-30, 30, 5000))).astype(np.float32)
    assert np.array_equal(one("add", 0, 1, 5000, [x, z]), x + z)
    assert np.array_equal(one("mul", 0, 1, 5000, [x, z]), x * z)
    assert np.array_equal(one("scale", 0, 1, 5000, [x], s=(f32(-1.75), 0, 0, 0)), f32(-1.75) * x)
    # operand order matters for nothing here, but slot 1 must be read
    assert not np.array_equal(one("add", 0, 1, 5000, [x, z]), x + x)


def test_modulo_broadcast_closed_form():
    x = np.arange(1, 7, dtype=np.float32)        # 1..6
    z = np.array([10, 20, 30], dtype=np.float32)  # broadcast by modulo
    assert one("add", 0, 1, 6, [x, z]).tolist() == [11, 22, 33, 14, 25, 36]
    # operand 0 shorter than the op: repeats too
    assert one("mul", 0, 1, 6, [z, x], in_n=[3, 6]).tolist() == [10, 40, 90, 40, 100, 180]


# --------------------------------------------------------------------------
# GELU (erf form): gelu(x) = x * Phi(x), Phi the standard normal CDF.
# --------------------------------------------------------------------------
def test_gelu_table_and_identities():
    # standard normal CDF table values
    table = {1.0: 0.8413447460685429, 2.0: 0.9772498680518208,
             -1.0: 0.15865525393145707, 0.5: 0.6914624612740131}
    for x, phi in table.items():
        assert abs(oracle.gelu(x) - x * phi) <= 1e-15
    assert oracle.gelu(0.0) == 0.0
    for x in np.linspace(-7, 7, 141):
        assert abs((oracle.gelu(x) - oracle.gelu(-x)) - x) <= 4e-15 * max(1, abs(x))


def test_gelu_matches_scipy_ndtr():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.uniform(-9, 9, 20000), rng.standard_normal(20000)]).astype(np.float32)
    y = one("gelu", 0, 1, x.size, [x])
    ref = (x.astype(np.float64) * sps.ndtr(x.astype(np.float64))).astype(np.float32)
    ulp = np.spacing(np.abs(ref)).astype(np.float64)
    assert (np.abs(y.astype(np.float64) - ref) <= ulp).all()


# --------------------------------------------------------------------------
# SiLU * mul: y = g * sigmoid(g) * u.
# --------------------------------------------------------------------------
def test_silu_mul_closed_forms():
    g = np.array([0.0, math.log(3.0), -math.log(3.0)], dtype=np.float32)
    u = np.array([5.0, 1.0, 2.0], dtype=np.float32)
    y = one("silu_mul", 0, 1, 3, [g, u])
    gd = g.astype(np.float64)
    assert y[0] == 0.0
    # sigmoid(ln 3) = 3/4, sigmoid(-ln 3) = 1/4
    assert abs(y[1] - 0.75 * gd[1]) <= 1e-7 * abs(gd[1])
    assert abs(y[2] - 2 * 0.25 * gd[2]) <= 1e-7 * abs(gd[2])
    rng = np.random.default_rng(8)
    g = rng.standard_normal(5000).astype(np.float32) * 4
    u = rng.standard_normal(5000).astype(np.float32)
    y = one("silu_mul", 0, 1, 5000, [g, u])
    ref = (g.astype(np.float64) * sps.expit(g.astype(np.float64)) * u).astype(np.float32)
    assert (np.abs(y - ref) <= np.spacing(np.abs(ref))).all()
    # operands are not interchangeable
    assert not np.allclose(one("silu_mul", 0, 1, 5000, [u, g]), y)


# --------------------------------------------------------------------------
# Row reductions.
# --------------------------------------------------------------------------
def test_rowsum_arange_and_fsum():
    for n in (1, 7, 100, 4096, 5792):
        y = one("rowsum", 0, 1, n, [np.arange(n, dtype=np.float32)])
        assert y[0] == n * (n - 1) // 2
    alt = np.array([1, -1] * 50 + [1], dtype=np.float32)
    assert one("rowsum", 0, 1, alt.size, [alt])[0] == 1.0
    rng = np.random.default_rng(9)
    m = rng.standard_normal((16, 3000)).astype(np.float32)
    y = one("rowsum", 0, 16, 3000, [m.ravel()])
    ref = np.array([math.fsum(r.astype(np.float64)) for r in m]).astype(np.float32)
    assert np.array_equal(y, ref)  # double accumulation of 3000 terms rounds like the exact sum here


def test_rowmax():
    for n in (1, 5, 8192):
        assert one("rowmax", 0, 1, n, [np.arange(n, dtype=np.float32)])[0] == n - 1
    rng = np.random.default_rng(10)
    m = rng.standard_normal((32, 777)).astype(np.float32)
    assert np.array_equal(one("rowmax", 0, 32, 777, [m.ravel()]), m.max(axis=1))
    # rows are not mixed up
    m[3, 5] = 100.0
    y = one("rowmax", 0, 32, 777, [m.ravel()])
    assert y[3] == 100.0 and (np.delete(y, 3) < 100).all()


# --------------------------------------------------------------------------
# Softmax.
# --------------------------------------------------------------------------
def test_softmax_closed_forms_and_scipy():
    y = one("softmax", 0, 1, 3, [np.array([0.0, math.log(2), math.log(3)], dtype=np.float32)])
    assert np.allclose(y, [1 / 6, 2 / 6, 3 / 6], rtol=2e-7, atol=0)
    for L in (1, 128, 1024, 4096):
        yc = one("softmax", 0, 1, L, [np.full(L, 0.37, dtype=np.float32)])
        assert (yc == np.float32(1.0 / L)).all()
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((8, 1500)) * 3).astype(np.float32)
    y = one("softmax", 0, 8, 1500, [x.ravel()]).reshape(8, 1500)
    assert np.allclose(y.astype(np.float64).sum(axis=1), 1.0, atol=1e-5)
    ref = sps.softmax(x.astype(np.float64), axis=1).astype(np.float32)
    assert np.allclose(y, ref, rtol=1e-6, atol=0)
    # shift invariance
    y2 = one("softmax", 0, 8, 1500, [(x + 5.0).ravel().astype(np.float32)]).reshape(8, 1500)
    assert np.allclose(y2, y, rtol=1e-5, atol=1e-30)
    # two elements: sigmoid of the difference
    y3 = one("softmax", 0, 1, 2, [np.array([1.5, -0.5], dtype=np.float32)])
    assert abs(y3[0] - sps.expit(2.0)) <= 1e-7


# --------------------------------------------------------------------------
# RMSNorm and LayerNorm.
# --------------------------------------------------------------------------
def test_rmsnorm_closed_forms():
    eps = np.float32(1e-6)
    L = 2048
    w = np.linspace(0.5, 1.5, L).astype(np.float32)
    for c in (0.25, 1.0, 3.0):
        y = one("rmsnorm", 0, 1, L, [np.full(L, c, dtype=np.float32), w], s=(eps, 0, 0, 0))
        ref = (w.astype(np.float64) * c / math.sqrt(c * c + float(eps))).astype(np.float32)
        assert np.array_equal(y, ref)
        alt = np.array([c, -c] * (L // 2), dtype=np.float32)
        y = one("rmsnorm", 0, 1, L, [alt, w], s=(eps, 0, 0, 0))
        assert np.array_equal(y, (np.sign(alt) * ref).astype(np.float32))
    # one nonzero element v: mean square v^2/L
    x = np.zeros(L, dtype=np.float32)
    x[7] = 2.0
    y = one("rmsnorm", 0, 1, L, [x, w], s=(eps, 0, 0, 0))
    assert abs(y[7] - 2.0 / math.sqrt(4.0 / L + 1e-6) * w[7]) <= 1e-6 * abs(y[7])
    assert (np.delete(y, 7) == 0).all()


def test_layernorm_closed_forms_and_torch():
    eps = np.float32(1e-5)
    L = 1024
    rng = np.random.default_rng(12)
    gam = rng.uniform(0.5, 1.5, L).astype(np.float32)
    bet = (rng.standard_normal(L) * 0.1).astype(np.float32)
    y = one("layernorm", 0, 1, L, [np.full(L, 2.5, np.float32), gam, bet], s=(eps, 0, 0, 0))
    assert np.array_equal(y, bet)
    alt = np.array([1.0, -1.0] * (L // 2), dtype=np.float32)
    y = one("layernorm", 0, 1, L, [alt, gam, bet], s=(eps, 0, 0, 0))
    ref = (alt * gam.astype(np.float64) / math.sqrt(1 + float(eps)) + bet).astype(np.float32)
    assert np.allclose(y, ref, rtol=1e-7, atol=1e-8)
    x = (rng.standard_normal((6, L)) + 3.0).astype(np.float32)
    y = one("layernorm", 0, 6, L, [x.ravel(), gam, bet], s=(eps, 0, 0, 0)).reshape(6, L)
    t = torch.nn.functional.layer_norm(torch.from_numpy(x).double(), (L,), torch.from_numpy(gam).double(),
                                       torch.from_numpy(bet).double(), eps=float(eps)).numpy()
    assert np.allclose(y, t.astype(np.float32), rtol=1e-6, atol=1e-7)
    # gamma and beta are not swapped
    y_sw = one("layernorm", 0, 6, L, [x.ravel(), bet, gam], s=(eps, 0, 0, 0)).reshape(6, L)
    assert not np.allclose(y_sw, y, atol=1e-3)


# --------------------------------------------------------------------------
# Rotary embedding, half-split pairs (i, i + D/2), theta_i = base^(-2i/D).
# --------------------------------------------------------------------------
def test_rotary_identities():
    rng = np.random.default_rng(13)
    H, D = 16, 128
    x = rng.standard_normal(H * D).astype(np.float32)
    # position 0 is the identity
    assert np.array_equal(one("rotary", 0, H, D, [x], s=(10000.0, 0, 0, 0), pos=0), x)
    pos = 517
    y = one("rotary", 0, H, D, [x], s=(10000.0, 0, 0, 0), pos=pos).reshape(H, D)
    xr = x.reshape(H, D).astype(np.float64)
    # complex-number formulation: (x_i + j x_{i+64}) * exp(j pos theta_i)
    theta = 10000.0 ** (-2.0 * np.arange(D // 2) / D)
    zc = (xr[:, :D // 2] + 1j * xr[:, D // 2:]) * np.exp(1j * pos * theta)
    ref = np.concatenate([zc.real, zc.imag], axis=1).astype(np.float32)
    assert np.allclose(y, ref, rtol=0, atol=1e-6)
    # pair norms preserved
    n0 = np.hypot(xr[:, :D // 2], xr[:, D // 2:])
    n1 = np.hypot(y[:, :D // 2].astype(np.float64), y[:, D // 2:].astype(np.float64))
    assert np.allclose(n0, n1, rtol=1e-6)
    # pair 0 turns by exactly pos radians (theta_0 = 1); pair 32 by pos/100
    x2 = np.zeros(D, dtype=np.float32)
    x2[0] = 1.0
    x2[32] = 1.0
    y2 = one("rotary", 0, 1, D, [x2], s=(10000.0, 0, 0, 0), pos=100)
    assert abs(y2[0] - math.cos(100)) < 1e-7 and abs(y2[64] - math.sin(100)) < 1e-7
    assert abs(y2[32] - math.cos(1.0)) < 1e-7 and abs(y2[96] - math.sin(1.0)) < 1e-7


# --------------------------------------------------------------------------
# bf16 rounding: round to nearest, ties to even, checked against a second
# formulation (nearest of the two neighbouring bf16 values by distance).
# --------------------------------------------------------------------------
def _bf16_nearest(bits: np.ndarray) -> np.ndarray:
    f = bits.view(np.float32).astype(np.float64)
    lo = (bits >> 16).astype(np.uint32)
    hi = lo + 1
    vlo = (lo << 16).view(np.float32).astype(np.float64)
    hi_bits = (hi << 16).astype(np.uint32)
    vhi = hi_bits.view(np.float32).astype(np.float64)
    # the pattern after the largest finite value is infinity; for rounding it
    # stands for 2^128
    over = (hi & 0x7FFF) == 0x7F80
    vhi = np.where(over, np.copysign(2.0 ** 128, f), vhi)
    dlo, dhi = np.abs(f - vlo), np.abs(vhi - f)
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((lo & 1) == 1))
    return np.where(pick_hi, hi, lo).astype(np.uint16)


def test_bf16_rne_against_second_formulation():
    L = oracle.lib()
    hi16 = np.arange(1 << 16, dtype=np.uint32)
    # all ties and near-ties for every upper half, plus random patterns
    lows = np.array([0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF], dtype=np.uint32)
    bits = ((hi16[:, None] << 16) | lows[None, :]).ravel()
    rng = np.random.default_rng(14)
    bits = np.concatenate([bits, rng.integers(0, 1 << 32, 200000, dtype=np.uint64).astype(np.uint32)])
    fin = (bits & 0x7F800000) != 0x7F800000
    bits = bits[fin]
    # the oracle rounds through the same helper it uses for every bf16 store
    x = bits.view(np.float32)
    w = one("scale", 1, 1, 1, [np.array([0x3F80], dtype=np.uint16)], s=(1.0, 0, 0, 0))  # warm-up load
    assert w[0] == 0x3F80
    got = np.fromiter((L.orc_f32_to_bf16(float(v)) for v in x[:60000]), dtype=np.uint16, count=60000)
    assert np.array_equal(got, _bf16_nearest(bits[:60000]))
    got = np.fromiter((L.orc_f32_to_bf16(float(v)) for v in x[-60000:]), dtype=np.uint16, count=60000)
    assert np.array_equal(got, _bf16_nearest(bits[-60000:]))
    # NaN stays NaN, infinities stay
    assert (L.orc_f32_to_bf16(float("nan")) & 0x7FC0) == 0x7FC0
    assert L.orc_f32_to_bf16(float("inf")) == 0x7F80


def test_bf16_ops_round_once():
    # bf16 add: exact sum rounded once (fp32 intermediate is exact for bf16 operands here)
    rng = np.random.default_rng(15)
    x = W.bf16_bits_trunc(rng.standard_normal(4000).astype(np.float32))
    z = W.bf16_bits_trunc(rng.standard_normal(4000).astype(np.float32))
    y = one("add", 1, 1, 4000, [x, z])
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    zf = (z.astype(np.uint32) << 16).view(np.float32)
    ref = _bf16_nearest((xf + zf).view(np.uint32))
    assert np.array_equal(y, ref)


# --------------------------------------------------------------------------
# Stream semantics: submission order, chains, bounds.
# --------------------------------------------------------------------------
def test_chain_runs_in_submission_order():
    b = W._Builder("chain", 0)
    x = b.alloc_input(0, np.array([1.0, -2.0, 3.0, -4.0], dtype=np.float32))
    o1 = b.alloc_output(0, 4)
    o2 = b.alloc_output(0, 4)
    o3 = b.alloc_output(0, 4)
    i1 = b.add_op("relu_affine", 0, [x], o1, 1, 4, in_n=(4, 0), s=(2.0, 1.0, 0, 0))
    i2 = b.add_op("scale", 0, [o1], o2, 1, 4, in_n=(4, 0), s=(-0.5, 0, 0, 0), deps=[i1])
    b.add_op("add", 0, [o2, o1], o3, 1, 4, in_n=(4, 4), deps=[i2, i1])
    a32, _ = oracle.run(b.finish())
    # relu(2x+1) = [3, 0, 7, 0]; scale -> [-1.5, 0, -3.5, 0]; add -> [1.5, 0, 3.5, 0]
    assert a32[o1:o1 + 4].tolist() == [3, 0, 7, 0]
    assert a32[o2:o2 + 4].tolist() == [-1.5, 0, -3.5, 0]
    assert a32[o3:o3 + 4].tolist() == [1.5, 0, 3.5, 0]


def test_chain_micro_ops():
    x = np.array([-2.0, -0.5, 0.5, 2.0], dtype=np.float32)
    z = np.array([10.0, 20.0, 30.0, 40.0], dtype=np.float32)
    q = np.array([1.0, 2.0, 3.0, 4.0], dtype=np.float32)
    # ((x*3 + 1) relu) + z, then * q
    y = one("ew_chain", 0, 1, 4, [x, z, q], s=(3.0, 1.0, 0, 0), prog=("affine", "relu", "add1", "mul2"))
    assert y.tolist() == [10.0, 40.0, 3 * (2.5 + 30), 4 * (7 + 40)]
    y = one("ew_chain", 0, 1, 4, [x], s=(2.0, 0.5, 0, 0), prog=("scale", "adds"))
    assert y.tolist() == [-3.5, -0.5, 1.5, 4.5]


def test_oracle_rejects_out_of_bounds():
    b = W._Builder("bad", 0)
    x = b.alloc_input(0, np.ones(8, dtype=np.float32))
    out = b.alloc_output(0, 8)
    b.add_op("add", 0, [x, x], out, 1, 16, in_n=(1000, 8))  # operand 0 runs past the arena
    w = b.finish()
    with pytest.raises(RuntimeError):
        oracle.run(w)


def test_small_configs_run():
    for c in (1, 3, 5):
        w = W.make(c, small=True)
        a32, a16 = oracle.run(w)
        assert np.isfinite(a32[w.n_init_f32:]).all()
