"""GPU parity of the device-side EAGLE-2 draft tree build (tsd_draft_tree_*) against the oracle:
the kept tree (parent[], tokens, node count) bit-exact whenever every selection clears its margin
(the kernels sum fp32 exponentials in fp64; the oracle is fp64 throughout)."""
import numpy as np
import pytest
import torch

import oracle
import tree_speculative_decoding_06_b200 as tsd
import workloads as W

pytestmark = pytest.mark.gpu

MARGIN = 1e-5   # log-probability gap below which a selection may legitimately differ


def _logits(rng, B, F, V, dtype):
    z = (rng.standard_normal((B, F, V), dtype=np.float32) * 3.0).astype(np.float32)
    return W.f32_to_bf16_bits(z) if dtype == "bf16" else z


def _dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def _build_gpu(roots, logits, K, F, keep, max_nodes):
    B = len(roots)
    t = tsd.DraftTree(B, F, max_nodes)
    t.init(torch.from_numpy(np.asarray(roots, np.int32)).cuda())
    for rows in logits:
        t.expand(_dev(rows), K)
    out = t.finalize(keep)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}, t


@pytest.mark.parametrize("dtype,V,B,F,K,depth,keep,seed", [
    ("bf16", 128256, 4, 10, 10, 6, 60, 0),   # the EAGLE-2 workload's shape
    ("bf16", 40000, 3, 4, 5, 4, 17, 1),      # several chunks and a partial last chunk
    ("f32", 1001, 3, 3, 4, 4, 14, 2),        # V not a multiple of 8 (scalar loads)
    ("f32", 20, 2, 2, 16, 3, 40, 3),         # K = 16 (the maximum), fewer tokens than a chunk
])
def test_draft_tree_matches_oracle(dtype, V, B, F, K, depth, keep, seed):
    rng = np.random.default_rng(seed)
    roots = rng.integers(0, V, size=B).astype(np.int32)
    logits = [_logits(rng, B, F, V, dtype) for _ in range(depth)]
    ref = oracle.draft_tree_build(roots, logits, K=K, F=F, keep=keep)
    assert ref["margin"] > MARGIN, "seed too close to a selection boundary"
    max_nodes = 1 + depth * F * K
    got, t = _build_gpu(roots, logits, K, F, keep, max_nodes)
    assert (t.status.cpu().numpy() == 0).all()
    assert np.array_equal(got["num_nodes"], ref["num_nodes"])
    assert np.array_equal(got["parent"], ref["parent"])
    assert np.array_equal(got["tokens"], ref["tokens"])
    # the device-side scores of the generated nodes agree with the oracle's to fp64 rounding of
    # fp32 exponentials
    sc = t.score.cpu().numpy()
    for b in range(B):
        tr = ref["trees"][b]
        n = len(tr.score)
        assert np.max(np.abs(sc[b, :n] - np.array(tr.score))) < 1e-5


def test_draft_tree_feeds_the_verify_step():
    """A finalised tree is a valid verify input: tree_prepare accepts it, depth-ordered."""
    rng = np.random.default_rng(5)
    B, F, K, V, keep = 2, 10, 10, 4096, 60
    roots = rng.integers(0, V, size=B).astype(np.int32)
    logits = [_logits(rng, B, F, V, "bf16") for _ in range(6)]
    got, _ = _build_gpu(roots, logits, K, F, keep, 1 + 6 * F * K)
    parent = torch.from_numpy(got["parent"]).cuda()
    prep = tsd.tree_prepare(parent, torch.from_numpy(got["num_nodes"]).cuda(), 6, False)
    torch.cuda.synchronize()
    assert (prep["status"].cpu().numpy() == 0).all()


def test_draft_tree_capacity_flag():
    rng = np.random.default_rng(7)
    B, F, K, V = 2, 4, 4, 500
    t = tsd.DraftTree(B, F, max_nodes=1 + F * K)          # room for one full expansion only
    t.init(torch.zeros(B, dtype=torch.int32, device="cuda"))
    t.expand(_dev(_logits(rng, B, F, V, "f32")), K)          # 1 frontier node -> 4 children: fits
    n1 = t.num_nodes.cpu().numpy().copy()
    t.expand(_dev(_logits(rng, B, F, V, "f32")), K)          # 4 x 4 more: does not fit
    torch.cuda.synchronize()
    assert (t.status.cpu().numpy() == 6).all()
    assert np.array_equal(t.num_nodes.cpu().numpy(), n1)
    out = t.finalize(8)
    torch.cuda.synchronize()
    assert (out["num_nodes"].cpu().numpy() == 0).all()
