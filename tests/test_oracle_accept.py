"""Oracle pins: greedy tree acceptance.

Pinned against hand-worked cases (tests/golden/accept_tiny.txt) and against brute force:
enumerate every root->node path, keep those that reproduce target argmax decoding token
for token (numpy's argmax as the library routine), and take the deepest (lowest index on
ties) -- a different algorithm from the oracle's topological pass."""
import numpy as np
import pytest

import oracle
import workloads as W
from golden_io import nums, read_cases, rows


def _inp(parent, tokens, logits, Dmax, root_key=None, forest=False):
    w = W.Workload("t", B=1, Hq=1, Hkv=1, d=1, dtype="f32", L=0, L_lo=None,
                   tree="forest" if forest else "x", N=len(parent), Dmax=Dmax, V=logits.shape[-1], paged=False)
    return {"workload": w, "parent": np.array([parent], np.int32), "num_nodes": np.array([len(parent)], np.int32),
            "tokens": np.array([tokens], np.int32), "logits": np.ascontiguousarray(logits[None].astype(np.float32)),
            "Dmax": Dmax, "root_key": None if root_key is None else np.array([root_key], np.int32)}


@pytest.mark.parametrize("case", read_cases("accept_tiny.txt"), ids=lambda c: c["case"])
def test_golden_cases(case):
    parent = nums(case["parent"], int)
    logits = np.stack(rows(case["logits"]))
    rk = None if case["root_key"] == "none" else int(case["root_key"])
    inp = _inp(parent, nums(case["tokens"], int), logits, int(case["Dmax"]), rk, forest=(parent < 0).sum() > 1)
    r = oracle.accept_greedy(inp)
    assert r["accept_len"][0] == int(case["accept_len"])
    assert r["path"][0].tolist() == nums(case["path"], int).tolist()
    assert r["out_tokens"][0].tolist() == nums(case["out_tokens"], int).tolist()


def brute_force(parent, tokens, logits, root_key=None):
    N = len(parent)
    tstar = [int(np.argmax(logits[i])) for i in range(N)]
    best = None
    for end in range(N):
        path = []
        j = end
        while j >= 0:
            path.append(j)
            j = parent[j]
        path = path[::-1]
        root = path[0]
        if root_key is not None:
            roots = [i for i in range(N) if parent[i] < 0 and tokens[i] == root_key]
            if not roots or roots[0] != root:
                continue
        if all(tokens[path[k + 1]] == tstar[path[k]] for k in range(len(path) - 1)):
            if best is None or len(path) > len(best):
                best = path
    if best is None:
        return -1, [], []
    return len(best) - 1, [j + 1 for j in best], [tokens[j] for j in best[1:]] + [tstar[best[-1]]]


@pytest.mark.parametrize("forest", [False, True])
def test_brute_force_random_trees(forest):
    rng = np.random.default_rng(7)
    V = 5                                          # small vocab: many matches and duplicate siblings
    for t in range(300):
        N = int(rng.integers(1, 9))
        parent = [-1] + [int(rng.integers(-1 if forest else 0, i)) for i in range(1, N)]
        logits = rng.integers(-3, 4, size=(N, V)).astype(np.float32)   # integer logits: frequent ties
        tokens = rng.integers(0, V, size=N).astype(np.int32)
        for i in range(1, N):
            if rng.random() < 0.6:
                tokens[i] = int(np.argmax(logits[parent[i]])) if parent[i] >= 0 else tokens[i]
        depth = W.tree_depths(np.array(parent))
        Dmax = int(depth.max())
        rk = int(tokens[0]) if (forest and rng.random() < 0.8) else (V + 3 if forest else None)
        inp = _inp(parent, tokens, logits, Dmax, rk, forest)
        r = oracle.accept_greedy(inp)
        A, path, out = brute_force(parent, tokens, logits, rk)
        assert r["accept_len"][0] == A
        assert r["path"][0][: A + 1].tolist() == path
        assert (r["path"][0][A + 1:] == 0).all()
        assert r["out_tokens"][0][: A + 1].tolist() == out
        assert (r["out_tokens"][0][A + 1:] == -1).all()
        if A >= 0:                                  # n drafts on the path -> n + 1 tokens
            assert A <= Dmax and len(out) == A + 1


def test_full_chain_accepts_all_plus_bonus():
    rng = np.random.default_rng(1)
    K, V = 5, 50
    logits = rng.standard_normal((K + 1, V)).astype(np.float32)
    tokens = [7] + [int(np.argmax(logits[i])) for i in range(K)]
    inp = _inp(list(range(-1, K)), tokens, logits, K)
    r = oracle.accept_greedy(inp)
    assert r["accept_len"][0] == K
    assert r["out_tokens"][0].tolist() == tokens[1:] + [int(np.argmax(logits[K]))]


def test_argmax_first_max_and_nan():
    assert oracle.argmax_row(np.array([1, 3, 3, 2], np.float32)) == 1
    assert oracle.argmax_row(np.array([np.nan, 0, np.inf, np.inf], np.float32)) == 2
    assert oracle.argmax_row(np.array([np.nan, np.nan], np.float32)) == 0
    assert oracle.argmax_row(np.array([-np.inf, -np.inf, -1], np.float32)) == 2
    bits = W.f32_to_bf16_bits(np.array([0.5, 2.0, 2.0, -7.0], np.float32))
    assert oracle.argmax_row(bits) == 1


def test_workload_forest_hit_and_miss():
    w = W.WORKLOADS["forest"].scaled(B=8, L=20, V=300)
    inp = W.make_inputs(w, seed=11)
    r = oracle.accept_greedy(inp)
    for b in range(8):
        roots = np.nonzero(inp["parent"][b] < 0)[0]
        hit = [i for i in roots if inp["tokens"][b, i] == inp["root_key"][b]]
        if hit:
            assert r["path"][b][0] == hit[0] + 1 and r["accept_len"][b] >= 0
        else:
            assert r["accept_len"][b] == -1
