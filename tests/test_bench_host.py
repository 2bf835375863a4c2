"""bench.py's host-side accounting: the algorithmic bytes and flops it divides by, checked against
definitions written out from the oracle's explicit ancestor matrix."""
import numpy as np

import bench
import oracle
import workloads as W


def test_algorithmic_flops_and_bytes_match_their_definitions():
    for name in ("tiny", "forest"):
        w = W.WORKLOADS[name]
        if name == "forest":
            w = w.scaled(B=2, L=100)
        inp = W.make_inputs(w, nan_guard=False)
        B, N, Hq, d = inp["q"].shape
        Hkv = inp["k_tree"].shape[2]
        es = 2 if inp["q"].dtype == np.uint16 else 4
        flops = 0
        nbytes = 0
        for b in range(B):
            n, L = int(inp["num_nodes"][b]), int(inp["prefix_len"][b])
            M = oracle.tree_structure(inp["parent"][b, :n], int(inp["Dmax"]), bool(getattr(w, "forest", False)))["M"]
            keys = L + M.sum(axis=1)          # prefix + the node's own root->node path
            flops += int(4 * d * Hq * keys.sum())
            nbytes += Hkv * (L + n) * d * es * 2 + n * Hq * d * es * 2
        assert bench.attn_algorithmic_flops(inp) == flops
        assert bench.attn_algorithmic_bytes(inp) == nbytes
