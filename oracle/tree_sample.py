"""TEST INFRASTRUCTURE ONLY: fp64 CPU oracle of stochastic (multi-branch) tree acceptance.

The pages state rejection sampling for a linear draft ("Acelerando Sonar a traves de la
especulacion", section "Objetivo-Borrador", with the Leviathan et al. rule it cites) and say that
EAGLE explores a tree of draft candidates (section "EAGLE"), but not how a sampled tree is accepted.
The reading restated here is the plainest extension of the cited rule to several candidates: at
a node whose children were drawn independently from the draft distribution q, the children are
tried in index order; child c (token x) is accepted iff u_c q(x) < p(x); after a rejection the
target distribution is replaced by the residual p <- max(p - q, 0) / sum, so that the next child
is tested against what the earlier rejections left.  Acceptance moves to the accepted child and
repeats; when every child of a node is rejected (or the node is a leaf) one more token is drawn
from the current p by the inverse CDF with the sequence's last uniform.  With one child per node
this is exactly the chain rule; with i.i.d. children the emitted tokens follow the target
distribution (tests/test_oracle_tree_sample.py checks it by chi-square).

Uniforms: u[c] for the test of node c (indexed by node, so the allocation does not depend on the
path taken) and u[N] for the final draw.  fp64 throughout; plain loops.

Parity unpinned: none (chi-square of the first emitted token and of the first two on toy trees,
the single-child reduction to the chain sampler, p == q accepting the first child, disjoint
supports rejecting every child).
"""
from __future__ import annotations

import numpy as np


def softmax(z: np.ndarray, T: float) -> np.ndarray:
    x = np.asarray(z, np.float64) / T
    x = np.exp(x - x.max())
    return x / x.sum()


def inverse_cdf(prob: np.ndarray, u: float) -> int:
    total = float(prob.sum())
    thr = u * total
    acc = 0.0
    for t, x in enumerate(prob):
        acc += float(x)
        if acc > thr:
            return t
    return int(np.nonzero(prob > 0)[0][-1])


def tree_accept_sample(parent, tokens, target_probs, draft_probs, u):
    """One tree.  parent[i] < i (root: -1, node 0); tokens[i]; target_probs[i] = p after node i;
    draft_probs[i] = the q node i's children were drawn from; u: N+1 uniforms.

    Returns (path: accepted nodes root first, emitted tokens: accepted drafts below the root and
    the final draw)."""
    N = len(parent)
    children = [[] for _ in range(N)]
    for i in range(1, N):
        children[parent[i]].append(i)
    node = 0
    path = [0]
    emitted = []
    while True:
        p = np.array(target_probs[node], np.float64)
        q = np.array(draft_probs[node], np.float64)
        nxt = None
        for c in children[node]:
            x = tokens[c]
            if u[c] * q[x] < p[x]:
                nxt = c
                break
            r = np.maximum(p - q, 0.0)
            if r.sum() > 0:
                p = r / r.sum()
        if nxt is None:
            emitted.append(inverse_cdf(p, float(u[N])))
            return path, emitted
        path.append(nxt)
        emitted.append(int(tokens[nxt]))
        node = nxt
