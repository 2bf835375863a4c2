"""Pins of the threshold-acceptance oracle (oracle/tree_threshold.py)."""
import numpy as np

import oracle
import workloads as W
from oracle import tree_threshold as tt


def _rows(rng, N, V, sigma=2.0):
    return [rng.standard_normal(V) * sigma for _ in range(N)]


def test_tau_zero_accepts_every_node_and_tau_above_one_none():
    rng = np.random.default_rng(0)
    for _ in range(50):
        N = int(rng.integers(1, 30))
        parent = [-1] + [int(rng.integers(0, i)) for i in range(1, N)]
        toks = [int(t) for t in rng.integers(0, 12, size=N)]
        rows = _rows(rng, N, 12)
        depth = W.tree_depths(np.array(parent))
        A, path, em = tt.accept_threshold(parent, toks, rows, 0.0)
        deepest = int(np.argmax(depth))            # the lowest-index node of greatest depth
        assert A == depth.max() and path[-1] == deepest
        A, path, em = tt.accept_threshold(parent, toks, rows, 1.5)
        assert A == 0 and path == [0] and em == [int(np.argmax(rows[0]))]


def test_brute_force_over_root_paths():
    """A node is accepted iff every edge of its root path passes the threshold (written out per
    path, independently of the oracle's topological pass); a* is the deepest such node."""
    rng = np.random.default_rng(1)
    V, T = 8, 0.9
    for _ in range(200):
        N = int(rng.integers(2, 16))
        parent = [-1] + [int(rng.integers(0, i)) for i in range(1, N)]
        toks = [int(t) for t in rng.integers(0, V, size=N)]
        rows = _rows(rng, N, V, 1.0)
        tau = float(rng.choice([0.05, 0.1, 0.2, 0.4]))
        P = [np.exp(np.asarray(r) / T) / np.exp(np.asarray(r) / T).sum() for r in rows]
        best, best_d = 0, 0
        for i in range(N):
            path, n = [i], i
            while parent[n] >= 0:
                n = parent[n]
                path.append(n)
            ok = all(P[parent[c]][toks[c]] >= tau for c in path[:-1])
            if ok and len(path) - 1 > best_d:
                best, best_d = i, len(path) - 1
        A, pth, em = tt.accept_threshold(parent, toks, rows, tau, T)
        assert A == best_d and pth[-1] == best
        assert em[:-1] == [toks[c] for c in pth[1:]]
        assert em[-1] == int(np.argmax(rows[best]))


def test_above_one_half_equals_greedy_on_dominant_rows():
    """With tau > 1/2 only a row's argmax can pass; when every row's argmax holds more than tau,
    threshold acceptance is exactly greedy acceptance (compared with the C greedy oracle)."""
    rng = np.random.default_rng(2)
    parents = [W.tree_static_scored((4, 3, 2, 1, 1, 1), 26), W.tree_tiny(), W.tree_chain(6)] * 3
    inp = W.make_custom_inputs(parents, [1] * len(parents), Hq=2, Hkv=1, d=16, dtype="f32", V=50, seed=3,
                               plant_p=0.7)
    lg = inp["logits"]
    am = lg.argmax(-1)
    for b in range(lg.shape[0]):
        for n in range(lg.shape[1]):
            lg[b, n, am[b, n]] += 12.0                 # argmax probability > 0.99
    ref = oracle.accept_greedy(inp)
    got = tt.accept_threshold_batch(lg, inp["tokens"], inp["parent"], inp["num_nodes"], 0.6, 1.0, int(inp["Dmax"]),
                                    lambda r: np.asarray(r, np.float64))
    assert np.array_equal(got["accept_len"], ref["accept_len"])
    assert np.array_equal(got["path"], ref["path"])
    assert np.array_equal(got["out_tokens"], ref["out_tokens"])


def test_hand_worked_chain():
    # V = 2, T = 1: row logits (0, ln 3) give p = (1/4, 3/4); (ln 3, 0) give (3/4, 1/4)
    l3 = np.log(3.0)
    rows = [np.array([0.0, l3]), np.array([l3, 0.0]), np.array([0.0, 0.0])]
    parent, toks = [-1, 0, 1], [0, 1, 0]
    # edge 0->1: p_0(1) = 3/4; edge 1->2: p_1(0) = 3/4
    assert tt.accept_threshold(parent, toks, rows, 0.7)[:2] == (2, [0, 1, 2])
    assert tt.accept_threshold(parent, toks, rows, 0.8)[:2] == (0, [0])
    toks2 = [0, 0, 0]                                  # edge 0->1: p_0(0) = 1/4
    assert tt.accept_threshold(parent, toks2, rows, 0.2)[:2] == (2, [0, 1, 2])
    assert tt.accept_threshold(parent, toks2, rows, 0.3)[:2] == (0, [0])
    # forest: only the root whose token is the key is accepted; a miss accepts nothing
    fp, ft = [-1, 0, -1, 2], [5, 1, 7, 0]
    frows = [np.array([0.0, 5.0] + [0.0] * 6)] * 4       # p(1) = e^5 / (e^5 + 7) > 0.95, p(0) < 0.01
    assert tt.accept_threshold(fp, ft, frows, 0.5, root_key=5)[:2] == (1, [0, 1])
    assert tt.accept_threshold(fp, ft, frows, 0.5, root_key=7)[:2] == (0, [2])
    assert tt.accept_threshold(fp, ft, frows, 0.5, root_key=9)[0] == -1
