"""Oracle pins: tree structure (shifted indices, ancestor tables, invariant checks).

Pinned against a hand-derived fixture, hand-made malformed trees and a brute-force
reachability closure computed by boolean matrix powers (a different route from the
oracle's upward walk)."""
import itertools

import numpy as np
import pytest

import oracle
from golden_io import nums, read_kv, rows


def test_shifted_indices_golden():
    g = read_kv("shifted_indices.txt")
    parent = nums(g["parent"], int)
    st = oracle.tree_structure(parent, int(g["Dmax"]))
    assert st["code"] == "ok"
    assert st["parent_s"].tolist() == nums(g["parent_s"], int).tolist()
    assert st["depth"].tolist() == nums(g["depth_s"], int).tolist()
    assert st["anc"].tolist() == [r.tolist() for r in rows(g["anc"], int)]
    assert st["M"].tolist() == [r.tolist() for r in rows(g["M"], int)]
    # no negative index anywhere in what the kernels consume
    assert (st["parent_s"] >= 0).all() and (st["anc"] >= 0).all()


@pytest.mark.parametrize("parent,Dmax,forest,code,node", [
    ([0, 0], 4, False, "bad_parent", 0),          # node 0 must be a root
    ([-1, 1], 4, False, "bad_parent", 1),         # self-parent (cycle)
    ([-1, 0, 3, 1], 4, False, "bad_parent", 2),   # forward reference (parent >= i)
    ([-1, -2], 4, False, "bad_parent", 1),        # negative other than -1
    ([-1, 0, -1], 4, False, "extra_root", 2),     # two roots outside forest mode
    ([-1, 0, 1, 2, 3], 3, False, "too_deep", 4),  # depth 4 > Dmax 3
    ([-1, 0, 1, -1, 3, 4, 5, 6], 3, True, "too_deep", 7),
    ([-1, 0, -1, 2], 4, True, "ok", 0),           # forest is fine
    ([], 3, False, "ok", 0),                      # empty tree
])
def test_invariants(parent, Dmax, forest, code, node):
    st = oracle.tree_structure(np.array(parent, np.int32), Dmax, forest)
    assert st["code"] == code
    assert st["bad_node"] == node


def all_trees(n, forest=False):
    choices = [[-1]] + [list(range(-1 if forest else 0, i)) for i in range(1, n)]
    for p in itertools.product(*choices):
        yield np.array(p, np.int32)


@pytest.mark.parametrize("n,forest", [(1, False), (4, False), (5, False), (4, True), (5, True)])
def test_ancestor_matrix_brute_force(n, forest):
    for parent in all_trees(n, forest):
        st = oracle.tree_structure(parent, n, forest)
        assert st["code"] == "ok"
        A = np.zeros((n, n), bool)              # edge i -> parent(i), plus identity
        for i, p in enumerate(parent):
            A[i, i] = True
            if p >= 0:
                A[i, p] = True
        R = A.copy()
        for _ in range(n):                      # transitive closure by repeated squaring-ish
            R = (R.astype(int) @ R.astype(int)) > 0
        assert (st["M"].astype(bool) == R).all(), parent
        depth = R.sum(1) - 1                    # ancestors other than self
        assert st["depth"][1:].tolist() == depth.tolist()
        for i in range(n):                      # anc row = root->node slots ordered by depth
            anc_nodes = sorted(np.nonzero(R[i])[0], key=lambda j: depth[j])
            row = st["anc"][i + 1]
            assert row[: depth[i] + 1].tolist() == [j + 1 for j in anc_nodes]
            assert (row[depth[i] + 1:] == 0).all()
