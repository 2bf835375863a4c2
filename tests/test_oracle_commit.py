"""Oracle pins: branch KV commit.

Invariants that pin it: after the commit the cache rows L..L+A equal the tree rows named by
the path byte for byte; no other tree row appears anywhere in the cache; rows below L and
above L+A are untouched; the three modes agree (path gather from the scratch tree, in-place
compaction of a tree stored after the prefix, and the chain's length mode); the paged
cache agrees with the contiguous one."""
import numpy as np
import pytest

import oracle
import workloads as W


def _case(paged, dtype="bf16", seed=0):
    parents = [W.tree_static_scored((4, 3, 2, 1, 1, 1), 26), W.tree_tiny(), W.tree_chain(5)]
    return W.make_custom_inputs(parents, [33, 0, 70], Hq=4, Hkv=2, d=16, dtype=dtype, seed=seed, paged=paged,
                                nan_guard=False)


def _rows(inp, kc, b, lo, hi):
    if "k_pages" in inp:
        bs = kc.shape[2]
        pos = np.arange(lo, hi)
        return kc[inp["block_table"][b, pos // bs], :, pos % bs]
    return np.moveaxis(kc[b, :, lo:hi], 0, 1)


@pytest.mark.parametrize("paged", [False, True])
def test_commit_path_invariants(paged):
    inp = _case(paged)
    acc = oracle.accept_greedy(inp)
    kc, vc, pl, st = oracle.kv_commit(inp, acc["accept_len"], acc["path"], "path")
    k0 = inp["k_pages"] if paged else inp["k_cache"]
    for b in range(3):
        A, L = int(acc["accept_len"][b]), int(inp["prefix_len"][b])
        assert st[b] == "ok" and pl[b] == L + A + 1
        nodes = [int(s) - 1 for s in acc["path"][b][: A + 1]]
        got = _rows(inp, kc, b, L, L + A + 1)
        assert np.array_equal(got, inp["k_tree"][b, nodes])
        assert np.array_equal(_rows(inp, vc, b, L, L + A + 1), inp["v_tree"][b, nodes])
        cap = k0.shape[2] if not paged else inp["block_table"].shape[1] * k0.shape[2]
        assert np.array_equal(_rows(inp, kc, b, 0, L), _rows(inp, k0, b, 0, L))
        assert np.array_equal(_rows(inp, kc, b, L + A + 1, cap), _rows(inp, k0, b, L + A + 1, cap))
        # no non-path tree row anywhere in this sequence's cache
        allrows = _rows(inp, kc, b, 0, cap).reshape(cap, -1)
        others = set(range(int(inp["num_nodes"][b]))) - set(nodes)
        for j in others:
            assert not (allrows == inp["k_tree"][b, j].reshape(-1)).all(1).any()


@pytest.mark.parametrize("paged", [False, True])
def test_inplace_equals_path(paged):
    inp = _case(paged, seed=1)
    acc = oracle.accept_greedy(inp)
    ref = oracle.kv_commit(inp, acc["accept_len"], acc["path"], "path")
    # lay the tree K/V into the cache right after each prefix, then compact in place
    kc = (inp["k_pages"] if paged else inp["k_cache"]).copy()
    vc = (inp["v_pages"] if paged else inp["v_cache"]).copy()
    for b in range(3):
        L, N = int(inp["prefix_len"][b]), int(inp["num_nodes"][b])
        for j in range(N):
            if paged:
                bs = kc.shape[2]
                blk = inp["block_table"][b, (L + j) // bs]
                kc[blk, :, (L + j) % bs] = inp["k_tree"][b, j]
                vc[blk, :, (L + j) % bs] = inp["v_tree"][b, j]
            else:
                kc[b, :, L + j] = inp["k_tree"][b, j]
                vc[b, :, L + j] = inp["v_tree"][b, j]
    got = oracle.kv_commit(inp, acc["accept_len"], acc["path"], "inplace", k_cache=kc, v_cache=vc)
    assert np.array_equal(got[2], ref[2])
    for b in range(3):
        L, A = int(inp["prefix_len"][b]), int(acc["accept_len"][b])
        assert np.array_equal(_rows(inp, got[0], b, 0, L + A + 1), _rows(inp, ref[0], b, 0, L + A + 1))
        assert np.array_equal(_rows(inp, got[1], b, 0, L + A + 1), _rows(inp, ref[1], b, 0, L + A + 1))


def test_length_mode_is_identity_path():
    inp = _case(False, seed=2)
    A = np.array([3, 0, 4], np.int32)
    path = np.zeros((3, 7), np.int32)
    for b in range(3):
        path[b, : A[b] + 1] = np.arange(1, A[b] + 2)
    a = oracle.kv_commit(inp, A, None, "length")
    p = oracle.kv_commit(inp, A, path, "path")
    assert all(np.array_equal(x, y) for x, y in zip(a[:3], p[:3]))


def test_miss_capacity_and_bad_path_leave_cache_untouched():
    inp = _case(False, seed=3)
    path = np.zeros((3, 7), np.int32)
    path[0, :2] = [1, 99]                 # node 98 does not exist
    A = np.array([1, -1, 2], np.int32)    # seq 1: miss; seq 2: capacity (below)
    pl = inp["prefix_len"].copy()
    pl[2] = inp["k_cache"].shape[2] - 2
    kc, vc, pl2, st = oracle.kv_commit(inp, A, path, "path", prefix_len=pl)
    assert st == ["bad_path", "ok", "capacity"]
    assert np.array_equal(pl2, pl)
    assert np.array_equal(kc, inp["k_cache"]) and np.array_equal(vc, inp["v_cache"])
