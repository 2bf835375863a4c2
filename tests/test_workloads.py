"""The seeded generators: determinism and the tree shapes the workloads name."""
import hashlib

import numpy as np

import oracle
import workloads as W


def digest(inp):
    h = hashlib.sha256()
    for k in sorted(inp):
        v = inp[k]
        if isinstance(v, np.ndarray):
            h.update(k.encode())
            h.update(v.tobytes())
    return h.hexdigest()


def test_deterministic():
    w = W.WORKLOADS["tree26"].scaled(L=50, V=1000)
    assert digest(W.make_inputs(w)) == digest(W.make_inputs(w))
    assert digest(W.make_inputs(w)) != digest(W.make_inputs(w, seed=99))


def test_tree_shapes():
    t = W.tree_static_scored((4, 3, 2, 1, 1, 1), 26)
    assert len(t) == 26 and W.tree_depths(t).max() == 6 and (t < 0).sum() == 1
    assert oracle.tree_structure(t, 6)["code"] == "ok"
    f = W.tree_forest(8, 64)
    assert len(f) == 512 and (f < 0).sum() == 8 and W.tree_depths(f).max() == 8
    assert oracle.tree_structure(f, 8, forest=True)["code"] == "ok"
    assert oracle.tree_structure(f, 8, forest=False)["code"] == "extra_root"
    rng = np.random.default_rng(0)
    p, tok = W.tree_eagle2(np.random.Generator(np.random.PCG64(1)), 2000, keep=60)
    assert len(p) == 60 and W.tree_depths(p).max() <= 6
    assert oracle.tree_structure(p, 6)["code"] == "ok"
    assert W.tree_tiny().tolist() == [-1, 0, 0, 1, 1, 2, 2, 3]


def test_bf16_rounding():
    x = np.array([1.0, 1.00390625, 1.005859375, -3.3, 0.0], np.float32)
    b = W.f32_to_bf16_bits(x)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1.0); 1.005859375 rounds up
    assert W.bf16_bits_to_f32(b).tolist()[:3] == [1.0, 1.0, 1.0078125]
    assert b[4] == 0


def test_small_workloads_run_through_oracle():
    for name in ("tiny", "tree26", "eagle60", "forest"):
        w = W.WORKLOADS[name]
        w = w.scaled(L=min(w.L, 40), L_lo=None if w.L_lo is None else 10, V=min(w.V, 300),
                     B=min(w.B, 3))
        inp = W.make_inputs(w)
        acc = oracle.accept_greedy(inp)
        assert all(c == "ok" for c in acc["codes"])
        assert ((acc["accept_len"] >= -1) & (acc["accept_len"] <= w.Dmax)).all()
