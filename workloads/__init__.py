"""Seeded synthetic inputs for the tree-verify workloads.

This module draws random numbers and builds draft-tree shapes, nothing else.  It holds
none of the verify arithmetic (no attention, no acceptance rule, no sampling decision, no
commit): the oracle under ``oracle/`` and the CUDA path both consume the arrays it returns,
and neither of them is imported here.

Five workloads are defined, one per synthetic shape of the tree-verify step (sizes below
are the full ones; every generator takes overrides so tests can shrink them):

==========  ======================================================================
``tiny``    B=1, Hq=8, Hkv=2, d=64, fp32, prefix L=128, 8-node tree (depth 3,
            top-2), vocab 256, greedy acceptance + contiguous commit.
``tree26``  Llama-3-8B-shaped: B=1, Hq=32, Hkv=8, d=128, bf16, L=2048, static
            EAGLE-style tree (4,3,2,1,1,1) pruned to 26 nodes, vocab 128256.
``eagle60`` B=16 EAGLE-2-style dynamic trees (top-10 per expanded node, depth 6,
            reranked to 60 nodes), ragged L in [1024, 8192], paged cache (block 16).
``chain5``  70B-shaped chain: B=64, Hq=64, Hkv=8, d=128, L=8192, K=5 drafts,
            temperature 1 rejection sampling.
``forest``  SSD/Saguaro-style forest: B=8, 8 subtrees x 64 nodes (depth 8) per
            sequence, L=32768, paged cache (block 16).
==========  ======================================================================

Planting (so acceptance has something to find): the workload statement fixes "draft token
= target argmax of the parent's row with probability p" for the tiny and tree26 shapes;
this module takes that literally with numpy's ``argmax`` (first maximum) as input
construction, so duplicate sibling tokens can occur.  The eagle60 shape instead raises, for
each internal node with probability 0.75, one uniformly chosen child's token in the
parent's target row above the row maximum.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from fractions import Fraction
from typing import Optional

import numpy as np

BF16_NAN = np.uint16(0x7FC0)


# ----------------------------------------------------------------------------- bf16 bits
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even); return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + r) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bits to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def as_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    """Values of a generated array as float32, whatever its storage."""
    return bf16_bits_to_f32(x) if dtype == "bf16" else np.asarray(x, np.float32)


def _normal(rng: np.random.Generator, shape, sigma: float, dtype: str) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    return f32_to_bf16_bits(x) if dtype == "bf16" else x


def _nan_fill(shape, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return np.full(shape, BF16_NAN, np.uint16)
    return np.full(shape, np.nan, np.float32)


# ----------------------------------------------------------------------------- tree shapes
def tree_tiny() -> np.ndarray:
    """8 nodes, depth 3, top-2: root, 2 children, 4 grandchildren, 1 node at depth 3 (BFS)."""
    return np.array([-1, 0, 0, 1, 1, 2, 2, 3], np.int32)


def tree_chain(n: int) -> np.ndarray:
    """A linear draft: node i's parent is i-1."""
    return np.arange(-1, n - 1, dtype=np.int32)


def tree_star(n: int) -> np.ndarray:
    """A root with n-1 leaf children."""
    p = np.zeros(n, np.int32)
    p[0] = -1
    return p


def _full_tree_bfs(branching):
    parent, rank, depth, frontier = [-1], [0], [0], [0]
    for b in branching:
        nxt = []
        for p in frontier:
            for r in range(b):
                parent.append(p)
                rank.append(r)
                depth.append(depth[p] + 1)
                nxt.append(len(parent) - 1)
        frontier = nxt
    return parent, rank, depth


def tree_static_scored(branching, keep: int) -> np.ndarray:
    """Static EAGLE-style tree: the full tree with the given per-depth branching, scored by
    the product of 1/(1+rank) along each node's path (rank 0 = first child), pruned to the
    `keep` best nodes (ties by BFS position) and returned in BFS order."""
    parent, rank, _ = _full_tree_bfs(branching)
    score = [Fraction(1)]
    for i in range(1, len(parent)):
        score.append(score[parent[i]] * Fraction(1, 1 + rank[i]))
    best = sorted(range(len(parent)), key=lambda i: (-score[i], i))[:keep]
    kept = sorted(best)
    remap = {old: new for new, old in enumerate(kept)}
    out = []
    for o in kept:
        p = parent[o]
        if p >= 0 and p not in remap:
            raise AssertionError("pruned tree is not ancestor-closed")
        out.append(-1 if p < 0 else remap[p])
    return np.array(out, np.int32)


def tree_eagle2(rng: np.random.Generator, V: int, topk: int = 10, depth: int = 6, keep: int = 60,
                sigma: float = 3.0):
    """EAGLE-2-style dynamic draft tree.  Each expanded node draws draft logits ~N(0, sigma)
    over the vocab and gets its top-k tokens as children, scored by cumulative draft
    log-probability; the top-k children of a depth form the next frontier.  After `depth`
    levels all generated nodes are reranked and the best `keep`-1 plus the root are kept,
    ordered by (depth, score desc).  Returns (parent int32[keep], tokens int32[keep])."""
    par, tok, lsc, dep = [-1], [int(rng.integers(0, V))], [0.0], [0]
    frontier = [0]
    for d in range(1, depth + 1):
        children = []
        for p in frontier:
            z = rng.standard_normal(V, dtype=np.float32).astype(np.float64) * sigma
            z -= z.max()
            lp = z - np.log(np.exp(z).sum())
            top = np.argpartition(-lp, topk)[:topk]
            top = top[np.lexsort((top, -lp[top]))]
            for t in top:
                par.append(p)
                tok.append(int(t))
                lsc.append(lsc[p] + float(lp[t]))
                dep.append(d)
                children.append(len(par) - 1)
        frontier = sorted(children, key=lambda i: (-lsc[i], i))[:topk]
    cand = sorted(range(1, len(par)), key=lambda i: (-lsc[i], i))[: keep - 1]
    kept = [0] + sorted(cand, key=lambda i: (dep[i], -lsc[i], i))
    remap = {old: new for new, old in enumerate(kept)}
    parent = np.array([-1 if par[o] < 0 else remap[par[o]] for o in kept], np.int32)
    tokens = np.array([tok[o] for o in kept], np.int32)
    return parent, tokens


def tree_forest(S: int, per: int, branching=(3, 2, 2, 1, 1, 1, 1, 1)) -> np.ndarray:
    """S copies of one pruned subtree packed into one parent[] with S roots at -1."""
    sub = tree_static_scored(branching, per)
    out = []
    for s in range(S):
        out.extend([-1 if p < 0 else p + s * per for p in sub])
    return np.array(out, np.int32)


def tree_depths(parent: np.ndarray) -> np.ndarray:
    """Depth of every node of a topologically ordered parent[] (fixture bookkeeping)."""
    d = np.zeros(len(parent), np.int32)
    for i, p in enumerate(parent):
        d[i] = 0 if p < 0 else d[p] + 1
    return d


# ----------------------------------------------------------------------------- workloads
@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    dtype: str                   # "f32" | "bf16"
    L: int                       # prefix length (upper end when ragged)
    L_lo: Optional[int]          # lower end of a ragged prefix (None = all equal)
    tree: str                    # "tiny" | "static26" | "eagle2" | "chain" | "forest"
    N: int                       # tree nodes per sequence
    Dmax: int                    # maximum node depth (root = 0)
    V: int
    paged: bool
    block_size: int = 16
    accept: str = "greedy"       # "greedy" | "sample"
    K: int = 0                   # chain drafts (sample)
    T: float = 1.0               # sampling temperature
    S: int = 1                   # forest subtrees
    plant_p: float = 0.75
    logit_sigma: float = 3.0
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def forest(self) -> bool:
        return self.tree == "forest"

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, Hq=8, Hkv=2, d=64, dtype="f32", L=128, L_lo=None, tree="tiny",
                     N=8, Dmax=3, V=256, paged=False, plant_p=0.7, logit_sigma=2.0, seed=0),
    "tree26": Workload("tree26", B=1, Hq=32, Hkv=8, d=128, dtype="bf16", L=2048, L_lo=None,
                       tree="static26", N=26, Dmax=6, V=128256, paged=False, plant_p=0.75,
                       logit_sigma=3.0, seed=1),
    "eagle60": Workload("eagle60", B=16, Hq=32, Hkv=8, d=128, dtype="bf16", L=8192, L_lo=1024,
                        tree="eagle2", N=60, Dmax=6, V=128256, paged=True, plant_p=0.75,
                        logit_sigma=3.0, seed=2),
    "chain5": Workload("chain5", B=64, Hq=64, Hkv=8, d=128, dtype="bf16", L=8192, L_lo=None,
                       tree="chain", N=6, Dmax=5, V=128256, paged=False, accept="sample", K=5,
                       T=1.0, logit_sigma=2.0, seed=3),
    "forest": Workload("forest", B=8, Hq=32, Hkv=8, d=128, dtype="bf16", L=32768, L_lo=None,
                       tree="forest", N=512, Dmax=8, V=128256, paged=True, S=8, plant_p=0.75,
                       logit_sigma=3.0, seed=4),
}


def _round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


def make_inputs(w: Workload, seed: Optional[int] = None, nan_guard: bool = True) -> dict:
    """Draw every input of one verify step of workload `w`.

    Storage: bf16 tensors are uint16 bit arrays, fp32 ones float32.  Layouts (row-major):
    q [B,N,Hq,d]; k_tree/v_tree [B,N,Hkv,d]; contiguous cache [B,Hkv,Lmax,d]; paged cache
    [num_blocks,Hkv,block,d] + block_table [B,max_blocks]; logits [B,N,V]; for sampling
    z_p [B,K+1,V], z_q [B,K,V], x [B,K], u [B,K+1] float32.  Cache rows that are not part of
    a sequence's prefix hold NaN when `nan_guard` is set, so any read of them shows up.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    B, N, dt = w.B, w.N, w.dtype
    out: dict = {"workload": w}

    # --- tree shape and tokens
    parents = np.zeros((B, N), np.int32)
    tokens = np.zeros((B, N), np.int32)
    eagle_tokens = None
    if w.tree == "tiny":
        parents[:] = tree_tiny()[:N]
    elif w.tree == "static26":
        parents[:] = tree_static_scored((4, 3, 2, 1, 1, 1), N)
    elif w.tree == "chain":
        parents[:] = tree_chain(N)
    elif w.tree == "forest":
        parents[:] = tree_forest(w.S, N // w.S)
    elif w.tree == "eagle2":
        eagle_tokens = np.zeros((B, N), np.int32)
        for b in range(B):
            p, t = tree_eagle2(rng, w.V, keep=N, depth=w.Dmax)
            parents[b], eagle_tokens[b] = p, t
    elif w.tree == "star":
        parents[:] = tree_star(N)
    else:
        raise ValueError(w.tree)
    out["parent"] = parents
    out["num_nodes"] = np.full(B, N, np.int32)

    # --- prefix lengths
    if w.L_lo is None:
        prefix = np.full(B, w.L, np.int32)
    else:
        prefix = rng.integers(w.L_lo, w.L + 1, size=B).astype(np.int32)
    out["prefix_len"] = prefix
    Lcap = _round_up(int(prefix.max()) + N, 64)

    # --- Q and tree K/V
    out["q"] = _normal(rng, (B, N, w.Hq, w.d), 1.0, dt)
    out["k_tree"] = _normal(rng, (B, N, w.Hkv, w.d), 1.0, dt)
    out["v_tree"] = _normal(rng, (B, N, w.Hkv, w.d), 1.0, dt)

    # --- KV cache
    if not w.paged:
        shape = (B, w.Hkv, Lcap, w.d)
        kc = _nan_fill(shape, dt) if nan_guard else np.zeros(shape, np.uint16 if dt == "bf16" else np.float32)
        vc = kc.copy()
        for b in range(B):
            L = int(prefix[b])
            kc[b, :, :L] = _normal(rng, (w.Hkv, L, w.d), 1.0, dt)
            vc[b, :, :L] = _normal(rng, (w.Hkv, L, w.d), 1.0, dt)
        out["k_cache"], out["v_cache"], out["Lmax"] = kc, vc, Lcap
    else:
        bs = w.block_size
        max_blocks = Lcap // bs if Lcap % bs == 0 else Lcap // bs + 1
        nblk = B * max_blocks + 3          # a few spare blocks nobody owns
        perm = rng.permutation(nblk).astype(np.int32)
        table = perm[: B * max_blocks].reshape(B, max_blocks)
        shape = (nblk, w.Hkv, bs, w.d)
        kp = _nan_fill(shape, dt) if nan_guard else np.zeros(shape, np.uint16 if dt == "bf16" else np.float32)
        vp = kp.copy()
        for b in range(B):
            L = int(prefix[b])
            kk = _normal(rng, (w.Hkv, L, w.d), 1.0, dt)
            vv = _normal(rng, (w.Hkv, L, w.d), 1.0, dt)
            for j in range((L + bs - 1) // bs):
                n = min(bs, L - j * bs)
                blk = table[b, j]
                kp[blk, :, :n] = kk[:, j * bs: j * bs + n]
                vp[blk, :, :n] = vv[:, j * bs: j * bs + n]
        out.update(k_pages=kp, v_pages=vp, block_table=table, num_blocks=nblk, max_blocks=max_blocks,
                   Lmax=max_blocks * bs)

    # --- logits and tokens
    if w.accept == "greedy":
        logits = np.empty((B, N, w.V), np.uint16 if dt == "bf16" else np.float32)
        for b in range(B):
            logits[b] = _normal(rng, (N, w.V), w.logit_sigma, dt)
        lf = lambda b, i: as_f32(logits[b, i], dt)  # noqa: E731
        if w.tree == "eagle2":
            tokens[:] = eagle_tokens
            for b in range(B):
                for p in range(N):
                    kids = np.nonzero(parents[b] == p)[0]
                    if len(kids) == 0 or rng.random() >= w.plant_p:
                        continue
                    c = int(kids[rng.integers(0, len(kids))])
                    row = lf(b, p)
                    val = np.float32(row.max() + np.float32(1.0))
                    if dt == "bf16":
                        bits = f32_to_bf16_bits(np.array([val]))[0]
                        assert bf16_bits_to_f32(np.array([bits]))[0] > row.max()
                        logits[b, p, tokens[b, c]] = bits
                    else:
                        logits[b, p, tokens[b, c]] = val
        else:
            for b in range(B):
                roots = np.nonzero(parents[b] < 0)[0]
                if w.forest:
                    rt = rng.choice(w.V, size=len(roots), replace=False).astype(np.int32)
                    tokens[b, roots] = rt
                else:
                    tokens[b, roots] = rng.integers(0, w.V, size=len(roots))
                for i in range(N):
                    p = parents[b, i]
                    if p < 0:
                        continue
                    if rng.random() < w.plant_p:
                        tokens[b, i] = int(np.argmax(lf(b, p)))
                    else:
                        tokens[b, i] = int(rng.integers(0, w.V))
        out["logits"] = logits
        if w.forest:
            keys = np.zeros(B, np.int32)
            for b in range(B):
                roots = np.nonzero(parents[b] < 0)[0]
                rt = tokens[b, roots]
                if rng.random() < 7.0 / 8.0:
                    keys[b] = rt[rng.integers(0, len(rt))]
                else:
                    while True:
                        t = int(rng.integers(0, w.V))
                        if t not in set(rt.tolist()):
                            break
                    keys[b] = t
            out["root_key"] = keys
        else:
            out["root_key"] = None
    else:  # chain rejection sampling
        K = w.K
        zp = np.empty((B, K + 1, w.V), np.uint16 if dt == "bf16" else np.float32)
        zq = np.empty((B, K, w.V), zp.dtype)
        x = np.zeros((B, K), np.int32)
        for b in range(B):
            zpf = rng.standard_normal((K + 1, w.V), dtype=np.float32) * np.float32(w.logit_sigma)
            zqf = zpf[:K] + rng.standard_normal((K, w.V), dtype=np.float32) * np.float32(0.8)
            zp[b] = f32_to_bf16_bits(zpf) if dt == "bf16" else zpf
            zq[b] = f32_to_bf16_bits(zqf) if dt == "bf16" else zqf
            for k in range(K):  # draft token drawn from softmax(z_q / T) (input construction)
                z = as_f32(zq[b, k], dt).astype(np.float64) / max(w.T, 1e-6)
                pr = np.exp(z - z.max())
                c = np.cumsum(pr)
                x[b, k] = min(int(np.searchsorted(c, rng.random() * c[-1], side="right")), w.V - 1)
        u = rng.random((B, K + 1), dtype=np.float32)
        tokens[:, 0] = rng.integers(0, w.V, size=B)
        tokens[:, 1:K + 1] = x
        out.update(z_p=zp, z_q=zq, x=x, u=u, T=w.T, root_key=None)
    out["tokens"] = tokens
    out["Dmax"] = w.Dmax
    return out


def nbytes_of(inputs: dict) -> int:
    return sum(v.nbytes for v in inputs.values() if isinstance(v, np.ndarray))


def make_custom_inputs(parents, prefix_lens, Hq: int = 4, Hkv: int = 2, d: int = 16, dtype: str = "f32",
                       V: int = 64, seed: int = 0, paged: bool = False, block_size: int = 16,
                       forest: bool = False, Dmax: Optional[int] = None, logit_sigma: float = 2.0,
                       plant_p: float = 0.6, nan_guard: bool = True, Nmax: Optional[int] = None) -> dict:
    """Inputs for hand-picked trees: `parents` is a list of per-sequence parent arrays (they
    may differ in length: the batch is ragged, padded to Nmax with -1 parents), `prefix_lens`
    the per-sequence prefix lengths.  Same storage and layouts as `make_inputs`; tokens are
    planted on parents' argmax rows with probability `plant_p`."""
    rng = np.random.Generator(np.random.PCG64(seed))
    B = len(parents)
    Ns = [len(p) for p in parents]
    Nmax = max(max(Ns), 1) if Nmax is None else Nmax
    if Dmax is None:
        Dmax = max([int(tree_depths(np.asarray(p)).max()) if len(p) else 0 for p in parents])
    parent = np.full((B, Nmax), -1, np.int32)
    for b, p in enumerate(parents):
        parent[b, :len(p)] = p
    prefix = np.asarray(prefix_lens, np.int32)
    w = Workload("custom", B=B, Hq=Hq, Hkv=Hkv, d=d, dtype=dtype, L=int(prefix.max()), L_lo=None,
                 tree="forest" if forest else "custom", N=Nmax, Dmax=Dmax, V=V, paged=paged,
                 block_size=block_size, logit_sigma=logit_sigma, plant_p=plant_p, seed=seed)
    out = {"workload": w, "parent": parent, "num_nodes": np.asarray(Ns, np.int32), "prefix_len": prefix,
           "Dmax": Dmax}
    Lcap = _round_up(int(prefix.max()) + Nmax, 64)
    out["q"] = _normal(rng, (B, Nmax, Hq, d), 1.0, dtype)
    out["k_tree"] = _normal(rng, (B, Nmax, Hkv, d), 1.0, dtype)
    out["v_tree"] = _normal(rng, (B, Nmax, Hkv, d), 1.0, dtype)
    store = np.uint16 if dtype == "bf16" else np.float32
    if not paged:
        shape = (B, Hkv, Lcap, d)
        kc = _nan_fill(shape, dtype) if nan_guard else np.zeros(shape, store)
        vc = kc.copy()
        for b in range(B):
            L = int(prefix[b])
            kc[b, :, :L] = _normal(rng, (Hkv, L, d), 1.0, dtype)
            vc[b, :, :L] = _normal(rng, (Hkv, L, d), 1.0, dtype)
        out.update(k_cache=kc, v_cache=vc, Lmax=Lcap)
    else:
        bs = block_size
        max_blocks = (Lcap + bs - 1) // bs
        nblk = B * max_blocks + 2
        table = rng.permutation(nblk).astype(np.int32)[: B * max_blocks].reshape(B, max_blocks)
        shape = (nblk, Hkv, bs, d)
        kp = _nan_fill(shape, dtype) if nan_guard else np.zeros(shape, store)
        vp = kp.copy()
        for b in range(B):
            L = int(prefix[b])
            kk = _normal(rng, (Hkv, L, d), 1.0, dtype)
            vv = _normal(rng, (Hkv, L, d), 1.0, dtype)
            for j in range((L + bs - 1) // bs):
                n = min(bs, L - j * bs)
                kp[table[b, j], :, :n] = kk[:, j * bs: j * bs + n]
                vp[table[b, j], :, :n] = vv[:, j * bs: j * bs + n]
        out.update(k_pages=kp, v_pages=vp, block_table=table, num_blocks=nblk, max_blocks=max_blocks,
                   Lmax=max_blocks * bs)
    logits = np.empty((B, Nmax, V), store)
    for b in range(B):
        logits[b] = _normal(rng, (Nmax, V), logit_sigma, dtype)
    tokens = np.zeros((B, Nmax), np.int32)
    for b in range(B):
        for i in range(Ns[b]):
            p = parent[b, i]
            if p >= 0 and rng.random() < plant_p:
                tokens[b, i] = int(np.argmax(as_f32(logits[b, p], dtype)))
            else:
                tokens[b, i] = int(rng.integers(0, V))
    out.update(logits=logits, tokens=tokens, root_key=None)
    return out


def make_tree_sample_inputs(parents, V: int, dtype: str = "bf16", seed: int = 0, T: float = 1.0,
                            sigma: float = 2.0, noise: float = 0.8, Nmax: Optional[int] = None) -> dict:
    """Inputs of stochastic tree acceptance for hand-picked trees (ragged, padded with -1 parents):
    target logits z_p [B, Nmax, V] ~ N(0, sigma) per node row, draft logits z_q = z_p + N(0, noise)
    (the chain workload's recipe), every non-root node's token drawn from softmax(z_q[parent] / T)
    -- children of one node drawn independently, as the draft would -- the root's token uniform,
    and uniforms u [B, Nmax] in [0, 1) (entry c for node c's test, entry 0 for the final draw)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    B = len(parents)
    Ns = [len(p) for p in parents]
    Nmax = max(Ns) if Nmax is None else Nmax
    parent = np.full((B, Nmax), -1, np.int32)
    for b, p in enumerate(parents):
        parent[b, :len(p)] = p
    store = np.uint16 if dtype == "bf16" else np.float32
    zp = np.zeros((B, Nmax, V), store)
    zq = np.zeros((B, Nmax, V), store)
    tokens = np.zeros((B, Nmax), np.int32)
    for b in range(B):
        zpf = rng.standard_normal((Nmax, V), dtype=np.float32) * np.float32(sigma)
        zqf = zpf + rng.standard_normal((Nmax, V), dtype=np.float32) * np.float32(noise)
        zp[b] = f32_to_bf16_bits(zpf) if dtype == "bf16" else zpf
        zq[b] = f32_to_bf16_bits(zqf) if dtype == "bf16" else zqf
        tokens[b, 0] = rng.integers(0, V)
        cdf = {}
        for i in range(1, Ns[b]):
            p = int(parent[b, i])
            if p not in cdf:   # draft token drawn from softmax(z_q / T) (input construction)
                z = as_f32(zq[b, p], dtype).astype(np.float64) / T
                cdf[p] = np.cumsum(np.exp(z - z.max()))
            c = cdf[p]
            tokens[b, i] = min(int(np.searchsorted(c, rng.random() * c[-1], side="right")), V - 1)
    u = rng.random((B, Nmax), dtype=np.float32)
    Dmax = max(int(tree_depths(np.asarray(p)).max()) for p in parents)
    return {"parent": parent, "num_nodes": np.asarray(Ns, np.int32), "z_p": zp, "z_q": zq, "tokens": tokens,
            "u": u, "T": T, "Dmax": Dmax, "dtype": dtype}


def make_ssd_inputs(B: int, K: int, V: int, dtype: str = "bf16", seed: int = 0, sigma: float = 3.0,
                    alpha_lo: float = 0.4, alpha_hi: float = 0.9) -> dict:
    """Inputs of the SSD outcome-cache build: draft logits [B, K+1, V] ~ N(0, sigma) (row a = the
    draft distribution at position a+1), a per-sequence acceptance rate alpha ~ U[alpha_lo,
    alpha_hi] (fp32) and uniforms [B, K] in [0, 1) (fp32) for the K draft draws."""
    rng = np.random.Generator(np.random.PCG64(seed))
    z = _normal(rng, (B, K + 1, V), sigma, dtype)
    alpha = rng.uniform(alpha_lo, alpha_hi, size=B).astype(np.float32)
    u = rng.random((B, K), dtype=np.float32)
    return {"draft_logits": z, "alpha": alpha, "u": u, "dtype": dtype, "K": K, "V": V}
