"""Pins of the draft tree build oracle (oracle/draft_tree.py): brute force on tiny vocabularies,
the closure and monotonicity invariants, and an independent restatement (one global sort of all
root->node paths) that shares no code with the oracle's incremental build."""
import itertools

import numpy as np
import pytest

import oracle
from oracle.draft_tree import DraftTree


def _rows(rng, F, V, scale=3.0):
    return (rng.standard_normal((F, V)) * scale).astype(np.float32)


def test_logsumexp_and_top_k_special_cases():
    z = np.array([0.0, 0.0, 0.0, 0.0])
    assert abs(oracle.draft_tree.logsumexp(z) - np.log(4.0)) < 1e-15
    z = np.array([1.0, 3.0, 3.0, -2.0, 2.0])
    assert oracle.draft_tree.top_k_tokens(z, 3) == [1, 2, 4]          # tie -> lower index first
    z = np.array([1e3, 0.0])
    assert abs(oracle.draft_tree.logsumexp(z) - 1e3) < 1e-12           # no overflow


def test_single_expansion_is_the_softmax_top_k():
    rng = np.random.default_rng(0)
    z = rng.standard_normal(50) * 3
    t = DraftTree(7)
    t.expand(z[None, :].astype(np.float32), K=5, F=3)
    p = np.exp(z.astype(np.float32).astype(np.float64))
    p /= p.sum()
    best = np.argsort(-p, kind="stable")[:5]
    assert t.token[1:] == list(best)
    for j, v in enumerate(best):
        assert abs(t.score[1 + j] - np.log(p[v])) < 1e-12
    assert t.frontier == [1, 2, 3]


def test_brute_force_tiny():
    """V=4, K=2, F=2, depth 3: every expansion is checked against an exhaustive enumeration of
    the children the frontier can have, and the final kept set against all generated nodes."""
    rng = np.random.default_rng(3)
    V, K, F, depth, keep = 4, 2, 2, 3, 6
    t = DraftTree(1)
    for d in range(depth):
        rows = _rows(rng, F, V)
        front = list(t.frontier)
        n0 = len(t.parent)
        t.expand(rows, K, F)
        # exhaustive: every (frontier node, token) pair with its exact cumulative log-prob
        allc = []
        for f, p in enumerate(front):
            z = rows[f].astype(np.float64)
            lp = z - np.log(np.exp(z).sum())
            for v in range(V):
                allc.append((t.score[p] + lp[v], f, v, p))
        # the appended children are, per frontier node, its K best tokens in rank order
        k = n0
        for f, p in enumerate(front):
            mine = sorted([c for c in allc if c[1] == f], key=lambda c: (-c[0], c[2]))[:K]
            for c in mine:
                assert t.parent[k] == p and t.token[k] == c[2] and abs(t.score[k] - c[0]) < 1e-12
                k += 1
        # the new frontier is the F best of the appended children
        appended = list(range(n0, k))
        best = sorted(appended, key=lambda i: (-t.score[i], i))[:F]
        assert t.frontier == best
    parent, tokens = t.finalize(keep)
    chosen = sorted(range(1, len(t.score)), key=lambda i: (-t.score[i], i))[: keep - 1]
    assert len(parent) == keep and parent[0] == -1
    assert sorted(tokens[1:].tolist()) == sorted(t.token[i] for i in chosen)
    # every kept non-root node is one of the keep-1 best; every node's parent precedes it
    for i in range(1, keep):
        assert 0 <= parent[i] < i


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_invariants_and_independent_restatement(seed):
    rng = np.random.default_rng(seed)
    V, K, F, depth, keep = 300, 4, 3, 4, 14
    t = DraftTree(5)
    rows_all = []
    for d in range(depth):
        rows = _rows(rng, F, V)
        rows_all.append(rows)
        t.expand(rows, K, F)
    parent, tokens = t.finalize(keep)
    # invariants: a child's score never exceeds its parent's; the kept tree is ancestor-closed,
    # ordered by depth, and its root is the root token
    for i in range(1, len(t.parent)):
        assert t.score[i] <= t.score[t.parent[i]] + 1e-12
    depth_new = np.zeros(len(parent), int)
    for i in range(1, len(parent)):
        assert 0 <= parent[i] < i
        depth_new[i] = depth_new[parent[i]] + 1
    assert np.all(np.diff(depth_new) >= 0) and tokens[0] == 5
    # independent restatement: replay the frontier choices as whole-path scores
    paths = {(): 0.0}
    frontier = [()]
    generated = []
    for rows in rows_all:
        kids = []
        for f, path in enumerate(frontier):
            z = rows[f].astype(np.float64)
            lp = z - np.log(np.exp(z).sum())
            for v in sorted(range(V), key=lambda v: (-lp[v], v))[:K]:
                kid = path + (v,)
                paths[kid] = paths[path] + lp[v]
                kids.append(kid)
        generated.extend(kids)
        order = {kid: n for n, kid in enumerate(generated)}
        frontier = sorted(kids, key=lambda k: (-paths[k], order[k]))[:F]
    order = {kid: n for n, kid in enumerate(generated)}
    chosen = sorted(generated, key=lambda k: (-paths[k], order[k]))[: keep - 1]
    ref = [()] + sorted(chosen, key=lambda k: (len(k), -paths[k], order[k]))
    # rebuild the oracle's kept paths from parent / tokens and compare
    got = [()]
    for i in range(1, len(parent)):
        got.append(got[parent[i]] + (int(tokens[i]),))
    assert got == ref


def test_batch_wrapper_pads_and_reports_margins():
    rng = np.random.default_rng(9)
    B, F, V, K, keep = 2, 2, 40, 2, 5
    logits = [(rng.standard_normal((B, F, V)) * 3).astype(np.float32) for _ in range(2)]
    r = oracle.draft_tree_build([3, 4], logits, K=K, F=F, keep=keep)
    assert r["parent"].shape == (B, keep) and (r["num_nodes"] == keep).all()
    assert r["margin"] > 0
