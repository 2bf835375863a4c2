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


def inverse_cdf(prob: np.ndarray, u: float, margin: list | None = None) -> int:
    """Smallest t with sum_{v<=t} prob[v] > u * sum(prob), by a sequential fp64 scan.  With
    `margin`, appends the distance of the threshold to the nearest cumulative boundary of the
    chosen token, relative to the total (how far the draw is from choosing a neighbour)."""
    total = float(prob.sum())
    thr = u * total
    acc = 0.0
    for t, x in enumerate(prob):
        prev = acc
        acc += float(x)
        if acc > thr:
            if margin is not None:
                margin.append(min(thr - prev, acc - thr) / total if total > 0 else 0.0)
            return t
    if margin is not None:
        margin.append(0.0)
    return int(np.nonzero(prob > 0)[0][-1])


def tree_accept_sample(parent, tokens, target_probs, draft_probs, u, margins: list | None = None):
    """One tree.  parent[i] < i (root: -1, node 0); tokens[i]; target_probs[i] = p after node i;
    draft_probs[i] = the q node i's children were drawn from; u: N+1 uniforms.

    Returns (path: accepted nodes root first, emitted tokens: accepted drafts below the root and
    the final draw).  With `margins`, appends for every accept test its relative margin
    |u q - p| / max(p, u q) and, last, the final draw's margin (see inverse_cdf): a decision whose
    margin is tiny may legitimately come out the other way under another rounding."""
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
            if margins is not None:
                den = max(p[x], u[c] * q[x])
                margins.append(abs(u[c] * q[x] - p[x]) / den if den > 0 else 0.0)
            if u[c] * q[x] < p[x]:
                nxt = c
                break
            r = np.maximum(p - q, 0.0)
            if r.sum() > 0:
                p = r / r.sum()
        if nxt is None:
            emitted.append(inverse_cdf(p, float(u[N]), margins))
            return path, emitted
        path.append(nxt)
        emitted.append(int(tokens[nxt]))
        node = nxt


class _SoftmaxRows:
    """Rows softmax(z[i] / T) in fp64, computed when first asked for (the walk visits few nodes)."""

    def __init__(self, z: np.ndarray, T: float, widen):
        self.z, self.T, self.widen, self.cache = z, T, widen, {}

    def __getitem__(self, i):
        if i not in self.cache:
            self.cache[i] = softmax(self.widen(self.z[i]), self.T)
        return self.cache[i]


def tree_accept_sample_batch(zp, zq, tokens, parent, num_nodes, uniforms, T: float, Dmax: int, widen):
    """Every sequence of a batch, in the layout of the GPU call: zp / zq [B, N, V] logits (row n =
    after node n), tokens / parent [B, N], uniforms [B, N] with entry c testing node c and entry 0
    the final draw (so the per-tree uniforms are u[c] = uniforms[c], u[N] = uniforms[0]).  `widen`
    maps a stored row to float values.  A walk stops growing at depth Dmax.

    Returns dict(accept_len [B], path [B, Dmax+1] slots, out_tokens [B, Dmax+1], margins: list of
    per-sequence margin lists)."""
    B = zp.shape[0]
    al = np.zeros(B, np.int32)
    path = np.zeros((B, Dmax + 1), np.int32)
    ot = np.full((B, Dmax + 1), -1, np.int32)
    margins = []
    for b in range(B):
        N = int(num_nodes[b])
        par = [int(x) for x in parent[b, :N]]
        if Dmax < max(_depths(par)):
            raise ValueError("tree deeper than Dmax")
        u = np.concatenate([uniforms[b, :N], uniforms[b, :1]]).astype(np.float64)
        m = []
        pth, em = tree_accept_sample(par, [int(t) for t in tokens[b, :N]], _SoftmaxRows(zp[b], T, widen),
                                     _SoftmaxRows(zq[b], T, widen), u, m)
        al[b] = len(pth) - 1
        path[b, :len(pth)] = np.array(pth) + 1
        ot[b, :len(em)] = em
        margins.append(m)
    return {"accept_len": al, "path": path, "out_tokens": ot, "margins": margins}


def _depths(parent):
    d = []
    for i, p in enumerate(parent):
        d.append(0 if p < 0 else d[p] + 1)
    return d
