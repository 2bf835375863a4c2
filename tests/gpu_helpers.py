"""Shared helpers of the GPU parity tests: move generated inputs to the device, run the
library through its binding, and compare with the oracle at the stated tolerances."""
import os

import numpy as np
import torch

import oracle
import tree_speculative_decoding_06_b200 as tsd
import workloads as W
from tree_speculative_decoding_06_b200.step import to_device

# attention tolerances: |gpu - ref| <= ATOL + RTOL * |ref| (bf16: 2e-2 / 1e-2; fp32: 1e-4 / 1e-4)
TOL = {"bf16": (2e-2, 1e-2), "f32": (1e-4, 1e-4)}


def dtype_of(inp):
    return "bf16" if inp["q"].dtype == np.uint16 else "f32"


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def lay_tree_in_cache(inp):
    """Copy every sequence's tree K/V into its cache right after the prefix (in-place layout)."""
    out = dict(inp)
    paged = "k_pages" in inp
    kc = (inp["k_pages"] if paged else inp["k_cache"]).copy()
    vc = (inp["v_pages"] if paged else inp["v_cache"]).copy()
    for b in range(inp["parent"].shape[0]):
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
    out["k_pages" if paged else "k_cache"] = kc
    out["v_pages" if paged else "v_cache"] = vc
    return out


def gpu_prepare(x, forest):
    return tsd.tree_prepare(x["parent"], x["num_nodes"], int(x["Dmax"]), forest)


def forced_split_workspace(inp):
    """A zeroed workspace holding TSD_ATTN_SPLITS partials (the split-count knob only takes effect
    when the workspace has room for them), or None when the knob is not set."""
    n = int(os.environ.get("TSD_ATTN_SPLITS", "0"))
    if n <= 1:
        return None
    B, Nmax, Hq, d = inp["q"].shape
    Hkv = inp["k_tree"].shape[2]
    dt = tsd.TSD_BF16 if dtype_of(inp) == "bf16" else tsd.TSD_F32
    if "block_table" in inp:
        planned = tsd.tree_verify_attn_paged_workspace_size(B, Nmax, Hq, Hkv, d, inp["block_table"].shape[1],
                                                            inp["k_pages"].shape[2], dt)
    else:
        planned = tsd.tree_verify_attn_workspace_size(B, Nmax, Hq, Hkv, d, inp["k_cache"].shape[2], dt)
    # at least what the planner asks for, or the binding would allocate a workspace of its own
    nbytes = max(planned, tsd.tree_verify_attn_ticket_bytes() + B * Hkv * n * (Hq // Hkv) * Nmax * (d + 2) * 4)
    return torch.zeros(nbytes, dtype=torch.uint8, device="cuda")


def gpu_attention(inp, tree_in_cache=False, want_lse=True, workspace=None):
    x = to_device(inp)
    forest = bool(getattr(inp["workload"], "forest", False))
    prep = gpu_prepare(x, forest)
    kt, vt = (None, None) if tree_in_cache else (x["k_tree"], x["v_tree"])
    if workspace is None:
        workspace = forced_split_workspace(inp)
    if "k_pages" in x:
        out, lse = tsd.tree_verify_attn_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["prefix_len"],
                                              kt, vt, prep["parent_s"], x["num_nodes"], int(x["Dmax"]),
                                              status=prep["status"], want_lse=want_lse, workspace=workspace)
    else:
        out, lse = tsd.tree_verify_attn(x["q"], x["k_cache"], x["v_cache"], x["prefix_len"], kt, vt,
                                        prep["parent_s"], x["num_nodes"], int(x["Dmax"]), status=prep["status"],
                                        want_lse=want_lse, workspace=workspace)
    torch.cuda.synchronize()
    return to_np(out), (lse.cpu().numpy() if lse is not None else None), prep["status"].cpu().numpy()


def check_attention(inp, out, lse, rows=None, tree_in_cache=False):
    ref, ref_lse, rows = oracle.attention_rows(inp, rows, tree_in_cache=tree_in_cache)
    got = np.stack([out[b, i, h] for (b, i, h) in rows])
    atol, rtol = TOL[dtype_of(inp)]
    err = np.abs(got - ref)
    bad = err > atol + rtol * np.abs(ref)
    assert not np.isnan(got).any(), "NaN in GPU attention output"
    assert not bad.any(), (f"attention mismatch: {bad.sum()} elements, max abs err {err.max():.3e}, "
                           f"first bad row {rows[int(np.nonzero(bad.any(1))[0][0])]}")
    if lse is not None:
        gl = np.array([lse[b, i, h] for (b, i, h) in rows])
        np.testing.assert_allclose(gl, ref_lse, rtol=1e-4, atol=1e-3)
    return float(err.max())


def sample_rows(inp, n, seed=0):
    rng = np.random.default_rng(seed)
    B, _, Hq, _ = inp["q"].shape
    rows = set()
    for b in range(B):
        N = int(inp["num_nodes"][b])
        rows.add((b, 0, 0))
        rows.add((b, N - 1, Hq - 1))
    while len(rows) < n:
        b = int(rng.integers(0, B))
        rows.add((b, int(rng.integers(0, int(inp["num_nodes"][b]))), int(rng.integers(0, Hq))))
    return sorted(rows)
