"""TEST INFRASTRUCTURE ONLY: fp64 CPU oracle of the device-side draft tree build.

"Acelerando Sonar a traves de la especulacion", section "EAGLE": EAGLE-2 shapes the draft tree
dynamically, taking the Top-K candidates at every node instead of following the single best
token, and the draft sequences are scored.  The pages give no more detail; the reading restated
here (the EAGLE-2 procedure as the rest of the pages' setting implies it) is:

  * the tree starts as the root alone (score 0, depth 0) and the frontier is [root];
  * one expansion consumes the draft logits of every frontier node f (row f): with
    lse_f = log sum_v exp(z_f[v]), the node's K children are its K largest logits (ties -> lower
    token id), each with score = score(f) + z_f[t] - lse_f (cumulative draft log-probability)
    and depth = depth(f) + 1; all n_frontier * K children are appended in frontier order, then
    rank order;
  * the new frontier is the F best children by (score desc, node index asc), in that order;
  * finalisation keeps the root and the keep-1 best non-root nodes by (score desc, node index
    asc) -- ancestor-closed because a child's score never exceeds its parent's and its index is
    larger -- ordered by (depth, score desc, node index) and renumbered, parents remapped.

Plain loops and numpy on small arrays; no blocking or fusion.  Each selection also reports its
margin (the score gap at the selection boundary) for the margin protocol of the parity tests:
the kernels sum fp32 exponentials in fp64, so a decision can differ from this fp64 oracle only
when a margin is below ~1e-6.

Parity unpinned: none (tests/test_oracle_draft_tree.py checks brute-force enumeration on tiny
vocabularies, the closure / monotonicity invariants, and an independent sort-based restatement
of the whole build).
"""
from __future__ import annotations

import numpy as np


def _widen(row: np.ndarray) -> np.ndarray:
    """bf16 bits (uint16) or fp32 -> fp64."""
    if row.dtype == np.uint16:
        return (row.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return row.astype(np.float64)


def logsumexp(z: np.ndarray) -> float:
    m = float(z.max())
    return m + float(np.log(np.exp(z - m).sum()))


def top_k_tokens(z: np.ndarray, K: int) -> list:
    """The K largest entries of z, ties -> lower index, best first (a stable sort of -z)."""
    order = np.lexsort((np.arange(len(z)), -z))
    return [int(v) for v in order[:K]]


class DraftTree:
    def __init__(self, root_token: int):
        self.parent = [-1]
        self.token = [int(root_token)]
        self.score = [0.0]
        self.depth = [0]
        self.frontier = [0]
        self.margins = []

    def expand(self, rows: np.ndarray, K: int, F: int):
        """rows[f] = draft logits after frontier node f (rows past the frontier are ignored)."""
        children = []
        for f, p in enumerate(self.frontier):
            z = _widen(rows[f])
            lse = logsumexp(z)
            for t in top_k_tokens(z, K):
                self.parent.append(p)
                self.token.append(int(t))
                self.score.append(self.score[p] + (z[t] - lse))
                self.depth.append(self.depth[p] + 1)
                children.append(len(self.parent) - 1)
        ranked = sorted(children, key=lambda i: (-self.score[i], i))
        if len(ranked) > F:
            self.margins.append(self._gap(ranked[F - 1], ranked[F]))
        self.frontier = ranked[:F]

    def _gap(self, a: int, b: int) -> float:
        """Score gap of a decision between nodes a and b.  Siblings with equal scores (the same
        draft logit under the same parent) tie exactly on any arithmetic and are ordered by
        index alike everywhere, so they decide nothing; any other gap is the decision margin."""
        if self.parent[a] == self.parent[b] and self.score[a] == self.score[b]:
            return np.inf
        return abs(self.score[a] - self.score[b])

    def finalize(self, keep: int):
        """Returns (parent int32[n], tokens int32[n]) of the kept tree, n = min(keep, nodes)."""
        cand = sorted(range(1, len(self.parent)), key=lambda i: (-self.score[i], i))
        if len(cand) > keep - 1 and keep >= 2:
            self.margins.append(self._gap(cand[keep - 2], cand[keep - 1]))
        chosen = cand[: max(keep - 1, 0)]
        kept = [0] + sorted(chosen, key=lambda i: (self.depth[i], -self.score[i], i))
        # order decisions inside one depth also rest on score comparisons
        for a, b in zip(kept[1:], kept[2:]):
            if self.depth[a] == self.depth[b]:
                self.margins.append(self._gap(a, b))
        remap = {old: new for new, old in enumerate(kept)}
        parent = np.array([-1 if self.parent[o] < 0 else remap[self.parent[o]] for o in kept], np.int32)
        tokens = np.array([self.token[o] for o in kept], np.int32)
        return parent, tokens


def draft_tree_build(root_tokens, logits_per_depth, K: int, F: int, keep: int):
    """Whole build for a batch.  logits_per_depth[d] is [B, F, V] (bf16 bits or fp32).

    Returns dict(parent [B, keep] int32 (-1 root / padding), tokens [B, keep] int32 (0 padding),
    num_nodes [B] int32, margin: smallest decision margin over the batch, trees: the DraftTree
    objects)."""
    B = len(root_tokens)
    parent = np.full((B, keep), -1, np.int32)
    tokens = np.zeros((B, keep), np.int32)
    num = np.zeros(B, np.int32)
    trees = []
    for b in range(B):
        t = DraftTree(int(root_tokens[b]))
        for rows in logits_per_depth:
            t.expand(rows[b], K, F)
        p, tk = t.finalize(keep)
        parent[b, :len(p)] = p
        tokens[b, :len(tk)] = tk
        num[b] = len(p)
        trees.append(t)
    margins = [m for t in trees for m in t.margins]
    return {"parent": parent, "tokens": tokens, "num_nodes": num, "margin": min(margins) if margins else np.inf,
            "trees": trees}
