"""Pins of the stochastic tree acceptance oracle (oracle/tree_sample.py)."""
import numpy as np
import pytest
from scipy import stats

from oracle import tree_sample as ts


def _toy(rng, V):
    p = rng.dirichlet(np.ones(V) * 0.7)
    q = rng.dirichlet(np.ones(V) * 0.7)
    return p, q


@pytest.mark.parametrize("m", [1, 2, 4])
def test_first_emitted_token_follows_the_target(m):
    """Root with m children drawn i.i.d. from q: the first emitted token is distributed as p."""
    rng = np.random.default_rng(m)
    V, trials = 8, 40000
    p, q = _toy(rng, V)
    counts = np.zeros(V)
    parent = [-1] + [0] * m
    for _ in range(trials):
        toks = [0] + list(rng.choice(V, size=m, p=q))
        leaf = np.ones(V) / V   # children are leaves: their own rows are irrelevant to the first token
        _, emitted = ts.tree_accept_sample(parent, toks, [p] + [leaf] * m, [q] + [leaf] * m,
                                           rng.random(m + 2))
        counts[emitted[0]] += 1
    chi2, pval = stats.chisquare(counts, p * trials)
    assert pval > 1e-4, (chi2, pval)


def test_first_two_tokens_follow_the_target_on_a_two_level_tree():
    """Root with 2 i.i.d. children, each with 2 i.i.d. children: the pair of the first two emitted
    tokens follows p(x1) p(x2 | x1) for a toy Markov target p(. | x)."""
    rng = np.random.default_rng(11)
    V, trials = 4, 60000
    P = rng.dirichlet(np.ones(V), size=V)          # P[x] = target after token x
    Q = rng.dirichlet(np.ones(V), size=V)          # Q[x] = draft after token x
    root_tok = 0
    counts = np.zeros((V, V))
    parent = [-1, 0, 0, 1, 1, 2, 2]
    for _ in range(trials):
        t1 = list(rng.choice(V, size=2, p=Q[root_tok]))
        t2a = list(rng.choice(V, size=2, p=Q[t1[0]]))
        t2b = list(rng.choice(V, size=2, p=Q[t1[1]]))
        toks = [root_tok] + t1 + t2a + t2b
        tp = [P[t] for t in toks]
        dq = [Q[t] for t in toks]
        _, em = ts.tree_accept_sample(parent, toks, tp, dq, rng.random(8))
        if len(em) >= 2:
            counts[em[0], em[1]] += 1
        else:   # the first token was the final draw: the second is a fresh target draw after it
            counts[em[0], rng.choice(V, p=P[em[0]])] += 1
    expected = (P[root_tok][:, None] * P) * trials
    chi2, pval = stats.chisquare(counts.ravel(), expected.ravel())
    assert pval > 1e-4, (chi2, pval)


def test_single_child_reduces_to_the_chain_rule():
    rng = np.random.default_rng(2)
    V = 10
    for _ in range(200):
        p, q = _toy(rng, V)
        x = int(rng.integers(V))
        u = rng.random(3)
        path, em = ts.tree_accept_sample([-1, 0], [0, x], [p, np.ones(V) / V], [q, np.ones(V) / V], u)
        if u[1] * q[x] < p[x]:
            assert path == [0, 1] and em[0] == x
        else:
            r = np.maximum(p - q, 0)
            assert path == [0] and em == [ts.inverse_cdf(r / r.sum(), u[2])]


def test_special_cases():
    rng = np.random.default_rng(3)
    V = 6
    p, _ = _toy(rng, V)
    # p == q: the first child is always accepted (u q < p for every u < 1)
    for _ in range(50):
        path, _ = ts.tree_accept_sample([-1, 0, 0], [0, 2, 4], [p, p, p], [p, p, p], rng.random(4) * 0.999)
        assert path[:2] == [0, 1]
    # disjoint supports: p has no mass on q's tokens, every child is rejected, the draw is from p
    p2 = np.array([0.5, 0.5, 0, 0, 0, 0])
    q2 = np.array([0, 0, 0.25, 0.25, 0.25, 0.25])
    path, em = ts.tree_accept_sample([-1, 0, 0], [0, 3, 5], [p2, p2, p2], [q2, q2, q2], [0.1, 0.1, 0.1, 0.7])
    assert path == [0] and em == [1]


def test_batch_wrapper_marshals_the_gpu_layout():
    """The batch form (GPU layout: uniforms[c] tests node c, uniforms[0] is the final draw, rows
    of logits per node) gives what the single-tree form gives on the same trees and numbers, and
    one margin per accept test plus one for the final draw."""
    import workloads as W
    parents = [W.tree_static_scored((4, 3, 2, 1, 1, 1), 26), W.tree_tiny(), W.tree_chain(4)]
    inp = W.make_tree_sample_inputs(parents, 50, "f32", seed=4, T=0.8)
    r = ts.tree_accept_sample_batch(inp["z_p"], inp["z_q"], inp["tokens"], inp["parent"], inp["num_nodes"],
                                    inp["u"], 0.8, int(inp["Dmax"]), lambda row: np.asarray(row, np.float32))
    for b, par in enumerate(parents):
        N = len(par)
        u = list(inp["u"][b, :N].astype(np.float64)) + [float(inp["u"][b, 0])]
        P = [ts.softmax(inp["z_p"][b, i].astype(np.float64), 0.8) for i in range(N)]
        Q = [ts.softmax(inp["z_q"][b, i].astype(np.float64), 0.8) for i in range(N)]
        m = []
        path, em = ts.tree_accept_sample([int(x) for x in par], [int(t) for t in inp["tokens"][b, :N]], P, Q, u, m)
        assert r["accept_len"][b] == len(path) - 1
        assert list(r["path"][b, :len(path)]) == [p + 1 for p in path] and (r["path"][b, len(path):] == 0).all()
        assert list(r["out_tokens"][b, :len(em)]) == em and (r["out_tokens"][b, len(em):] == -1).all()
        assert r["margins"][b] == m and len(m) >= 1
