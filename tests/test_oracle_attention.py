"""Oracle pins: tree-masked attention.

Pinned against a library routine (torch's scaled_dot_product_attention in fp64 on the CPU)
on the special cases the tree mask must reduce to, plus a hand-derived closed form:
  * a chain tree is plain causal attention over prefix + draft;
  * a star tree is independent single-query decode over prefix + root + self;
  * every node of every tree with N <= 5 equals decoding that node alone over
    prefix + its root->node path (brute force over all parent[] arrays);
  * changing a non-ancestor's K/V leaves a node's output bit-identical (no leakage).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from golden_io import nums, read_kv
from test_oracle_structure import all_trees


def f64(x, dt):
    return torch.from_numpy(W.as_f32(x, dt).astype(np.float64))


def sdpa(q, k, v, mask=None):
    """q [n, d], k/v [m, d] -> [n, d] (fp64, library routine)."""
    d = q.shape[-1]
    return torch.nn.functional.scaled_dot_product_attention(
        q[None, None], k[None, None], v[None, None], attn_mask=None if mask is None else mask[None, None],
        scale=1.0 / math.sqrt(d))[0, 0]


def rows_by_node(inp, out, rows):
    res = {}
    for r, key in enumerate(rows):
        res[key] = out[r]
    return res


def test_closed_form_golden():
    g = read_kv("attn_closed_form.txt")
    parent = nums(g["parent"], int)
    N = len(parent)
    inp = W.make_custom_inputs([parent], [1], Hq=1, Hkv=1, d=1, dtype="f32", V=4, nan_guard=False)
    inp["k_tree"][0, :, 0, 0] = nums(g["k_tree"])
    inp["v_tree"][0, :, 0, 0] = nums(g["v_tree"])
    inp["k_cache"][0, 0, 0, 0] = nums(g["k_prefix"])[0]
    inp["v_cache"][0, 0, 0, 0] = nums(g["v_prefix"])[0]
    inp["q"][0, :, 0, 0] = nums(g["q"])
    out, lse, rows = oracle.attention_rows(inp)
    assert [r[1] for r in rows] == list(range(N))
    np.testing.assert_allclose(out[:, 0], nums(g["out"]), rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(lse, nums(g["lse"]), rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_chain_equals_causal(dt):
    N = 7
    inp = W.make_custom_inputs([W.tree_chain(N), W.tree_chain(N)], [37, 0], Hq=4, Hkv=2, d=16, dtype=dt, seed=3)
    out, _, rows = oracle.attention_rows(inp)
    got = rows_by_node(inp, out, rows)
    G = 2
    for b in range(2):
        L = int(inp["prefix_len"][b])
        for h in range(4):
            g = h // G
            k = torch.cat([f64(inp["k_cache"][b, g, :L], dt), f64(inp["k_tree"][b, :N, g], dt)])
            v = torch.cat([f64(inp["v_cache"][b, g, :L], dt), f64(inp["v_tree"][b, :N, g], dt)])
            q = f64(inp["q"][b, :N, h], dt)
            mask = torch.ones(N, L + N, dtype=torch.bool)
            mask[:, L:] = torch.tril(torch.ones(N, N, dtype=torch.bool))
            ref = sdpa(q, k, v, mask).numpy()
            for i in range(N):
                np.testing.assert_allclose(got[(b, i, h)], ref[i], rtol=0, atol=1e-12)


def test_star_equals_independent_decode():
    N = 6
    inp = W.make_custom_inputs([W.tree_star(N)], [21], Hq=6, Hkv=3, d=8, dtype="bf16", seed=4)
    out, _, rows = oracle.attention_rows(inp)
    got = rows_by_node(inp, out, rows)
    L = 21
    for h in range(6):
        g = h // 2
        kp, vp = f64(inp["k_cache"][0, g, :L], "bf16"), f64(inp["v_cache"][0, g, :L], "bf16")
        kt, vt = f64(inp["k_tree"][0, :N, g], "bf16"), f64(inp["v_tree"][0, :N, g], "bf16")
        for i in range(N):
            sel = [0] if i == 0 else [0, i]
            q = f64(inp["q"][0, i:i + 1, h], "bf16")
            ref = sdpa(q, torch.cat([kp, kt[sel]]), torch.cat([vp, vt[sel]]))[0].numpy()
            np.testing.assert_allclose(got[(0, i, h)], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n,forest", [(3, False), (4, False), (5, False), (4, True)])
def test_every_node_equals_path_decode(n, forest):
    trees = list(all_trees(n, forest))
    for t, parent in enumerate(trees):
        L = (7 * t) % 13          # includes an empty prefix
        inp = W.make_custom_inputs([parent], [L], Hq=2, Hkv=1, d=8, dtype="f32", seed=100 + t, forest=forest)
        out, _, rows = oracle.attention_rows(inp)
        got = rows_by_node(inp, out, rows)
        kp, vp = f64(inp["k_cache"][0, 0, :L], "f32"), f64(inp["v_cache"][0, 0, :L], "f32")
        kt, vt = f64(inp["k_tree"][0, :n, 0], "f32"), f64(inp["v_tree"][0, :n, 0], "f32")
        for i in range(n):
            path = []
            j = i
            while j >= 0:
                path.append(j)
                j = parent[j]
            path = path[::-1]
            for h in range(2):
                q = f64(inp["q"][0, i:i + 1, h], "f32")
                ref = sdpa(q, torch.cat([kp, kt[path]]), torch.cat([vp, vt[path]]))[0].numpy()
                np.testing.assert_allclose(got[(0, i, h)], ref, rtol=0, atol=1e-12)


def test_no_cross_branch_leakage():
    parent = W.tree_static_scored((4, 3, 2, 1, 1, 1), 26)
    inp = W.make_custom_inputs([parent], [19], Hq=4, Hkv=2, d=16, dtype="bf16", seed=5)
    out0, _, rows = oracle.attention_rows(inp)
    M = oracle.tree_structure(parent, 6)["M"]
    rng = np.random.default_rng(0)
    for i in [0, 5, 13, 25]:
        pert = {k: v.copy() if isinstance(v, np.ndarray) else v for k, v in inp.items()}
        others = np.nonzero(M[i] == 0)[0]
        pert["k_tree"][0, others] = W.f32_to_bf16_bits(rng.standard_normal(pert["k_tree"][0, others].shape) * 5)
        pert["v_tree"][0, others] = W.f32_to_bf16_bits(rng.standard_normal(pert["v_tree"][0, others].shape) * 5)
        out1, _, _ = oracle.attention_rows(pert)
        for r, (b, ii, h) in enumerate(rows):
            if ii == i:
                assert np.array_equal(out0[r], out1[r])
        # and the perturbation does reach nodes that do see those rows
        changed = [r for r, (b, ii, h) in enumerate(rows) if not np.array_equal(out0[r], out1[r])]
        assert all(M[rows[r][1]][others].any() for r in changed)
        assert changed


def test_paged_equals_contiguous():
    parent = W.tree_tiny()
    a = W.make_custom_inputs([parent, parent[:5]], [40, 3], Hq=4, Hkv=2, d=8, dtype="bf16", seed=9)
    p = W.make_custom_inputs([parent, parent[:5]], [40, 3], Hq=4, Hkv=2, d=8, dtype="bf16", seed=9, paged=True,
                             block_size=16)
    # same q / tree; copy the contiguous prefix into the pages
    for key in ("q", "k_tree", "v_tree"):
        p[key] = a[key]
    for b in range(2):
        L = int(a["prefix_len"][b])
        for pos in range(L):
            blk = p["block_table"][b, pos // 16]
            p["k_pages"][blk, :, pos % 16] = a["k_cache"][b, :, pos]
            p["v_pages"][blk, :, pos % 16] = a["v_cache"][b, :, pos]
    oa, la, _ = oracle.attention_rows(a)
    op, lp, _ = oracle.attention_rows(p)
    assert np.array_equal(oa, op) and np.array_equal(la, lp)
