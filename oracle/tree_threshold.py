"""TEST INFRASTRUCTURE ONLY: fp64 CPU oracle of threshold acceptance over a draft tree.

"Acelerando Sonar a traves de la especulacion" (Perplexity), section "Decodificacion
especulativa", names, beside exact matching, acceptance of the longest prefix whose tokens stay
above an acceptance threshold, and gives no threshold or formula.  Reading restated here (the
plainest one the rest of the page supports): with p_n = softmax(target_logits[n] / T) the target
distribution after node n, a non-root node i is accepted iff its parent is accepted and
p_parent(i)(token[i]) >= tau; a single tree's root is always accepted, a forest's root only when
its token equals root_key (the lowest such root), as in greedy acceptance.  The deepest accepted
node a* (ties -> lowest index) ends the path; the emitted tokens are the accepted drafts below the
root, then the target's own next token, argmax of a*'s row (ties -> lowest id).  tau = 0 accepts
every node; a tau above 1/2 accepts only tokens that are their parent row's argmax.

Plain loops over the nodes, numpy fp64 softmax per row.  Parity unpinned: none
(tests/test_oracle_threshold.py: tau = 0 and tau > 1 closed forms, the tau > 1/2 inclusion in the
greedy result, brute force over every root->node path, hand-worked fixtures).
"""
from __future__ import annotations

import numpy as np


def softmax(z: np.ndarray, T: float) -> np.ndarray:
    x = np.asarray(z, np.float64) / T
    x = np.exp(x - x.max())
    return x / x.sum()


def accept_threshold(parent, tokens, rows, tau: float, T: float = 1.0, root_key=None, margins: list | None = None):
    """One tree: parent[i] < i (roots -1), tokens[i], rows[n] = target logits after node n (float
    values), tau, temperature T.  Returns (accept_len, path nodes root first, emitted tokens); a
    forest miss gives (-1, [], []).  With `margins`, appends |p - tau| / tau of every test made."""
    N = len(parent)
    probs = {}

    def p_of(n):
        if n not in probs:
            probs[n] = softmax(rows[n], T)
        return probs[n]

    acc = [False] * N
    depth = [0] * N
    hit_root = None
    for i in range(N):
        if parent[i] < 0:
            depth[i] = 0
            if root_key is None:
                acc[i] = True
            elif hit_root is None and tokens[i] == root_key:
                acc[i] = True
                hit_root = i
        else:
            depth[i] = depth[parent[i]] + 1
            if acc[parent[i]]:
                pv = float(p_of(parent[i])[tokens[i]])
                if margins is not None and tau > 0:
                    margins.append(abs(pv - tau) / tau)
                acc[i] = pv >= tau
    best = -1
    for i in range(N):
        if acc[i] and (best < 0 or depth[i] > depth[best]):
            best = i
    if best < 0:
        return -1, [], []
    path = [best]
    while parent[path[-1]] >= 0:
        path.append(parent[path[-1]])
    path.reverse()
    row = np.asarray(rows[best], np.float64)
    bonus = int(np.argmax(np.where(np.isnan(row), -np.inf, row)))
    return depth[best], path, [int(tokens[n]) for n in path[1:]] + [bonus]


def accept_threshold_batch(logits, tokens, parent, num_nodes, tau: float, T: float, Dmax: int, widen,
                           root_key=None):
    """Every sequence in the GPU call's layout: logits [B, N, V] (stored rows; `widen` gives float
    values), tokens / parent [B, N].  Returns dict(accept_len, path [B, Dmax+1] slots, out_tokens
    [B, Dmax+1], margins per sequence)."""
    B = logits.shape[0]
    al = np.zeros(B, np.int32)
    path = np.zeros((B, Dmax + 1), np.int32)
    ot = np.full((B, Dmax + 1), -1, np.int32)
    margins = []
    for b in range(B):
        N = int(num_nodes[b])
        m = []
        rk = None if root_key is None else int(root_key[b])
        A, pth, em = accept_threshold([int(x) for x in parent[b, :N]], [int(t) for t in tokens[b, :N]],
                                      _Rows(logits[b], widen), tau, T, rk, m)
        al[b] = A
        path[b, :len(pth)] = np.array(pth, np.int32) + 1
        ot[b, :len(em)] = em
        margins.append(m)
    return {"accept_len": al, "path": path, "out_tokens": ot, "margins": margins}


class _Rows:
    def __init__(self, z, widen):
        self.z, self.widen = z, widen

    def __getitem__(self, i):
        return self.widen(self.z[i])
