"""GPU parity of stochastic tree acceptance (tsd_tree_accept_sample) against the fp64 oracle in
oracle/tree_sample.py, with the chain sampler's margin protocol: bit-exact on every sequence whose
decisions all clear their margins, a validity check otherwise; and the target distribution of the
emitted tokens on the GPU (chi-square on a vocabulary of 16)."""
import numpy as np
import pytest
import torch
from scipy import stats

import tree_speculative_decoding_06_b200 as tsd
import workloads as W
from oracle import tree_sample as ots

pytestmark = pytest.mark.gpu

# the chain sampler's thresholds: fp32 exponentials (~1e-7 relative, independent per token),
# everything else fp64
ACC_MARGIN = 1e-5
CDF_MARGIN = 2e-7


def _dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run_gpu(inp, status=None):
    parent = torch.from_numpy(inp["parent"]).cuda()
    nn = torch.from_numpy(inp["num_nodes"]).cuda()
    prep = tsd.tree_prepare(parent, nn, int(inp["Dmax"]), False)
    st = prep["status"] if status is None else torch.from_numpy(status).cuda()
    r = tsd.tree_accept_sample(_dev(inp["z_p"]), _dev(inp["z_q"]), torch.from_numpy(inp["tokens"]).cuda(),
                               prep["parent_s"], torch.from_numpy(inp["u"]).cuda(), inp["T"], num_nodes=nn,
                               Dmax=int(inp["Dmax"]), status=st)
    torch.cuda.synchronize()
    out = {k: v.cpu().numpy() for k, v in r.items()}
    out["status"] = st.cpu().numpy()
    return out


def run_oracle(inp):
    dt = inp["dtype"]
    return ots.tree_accept_sample_batch(inp["z_p"], inp["z_q"], inp["tokens"], inp["parent"], inp["num_nodes"],
                                        inp["u"], inp["T"], int(inp["Dmax"]), lambda row: W.as_f32(row, dt))


def compare(got, ref, inp):
    """Returns the number of sequences with a decision inside its margin (checked for validity)."""
    near = 0
    for b in range(inp["parent"].shape[0]):
        m = ref["margins"][b]
        if all(x >= ACC_MARGIN for x in m[:-1]) and m[-1] >= CDF_MARGIN:
            assert got["accept_len"][b] == ref["accept_len"][b], b
            assert np.array_equal(got["path"][b], ref["path"][b]), b
            assert np.array_equal(got["out_tokens"][b], ref["out_tokens"][b]), b
            continue
        near += 1
        # a valid outcome: a root-down chain of parent -> child slots, its tokens, then a token
        A = int(got["accept_len"][b])
        pth = got["path"][b]
        assert pth[0] == 1 and 0 <= A <= int(inp["Dmax"])
        for j in range(1, A + 1):
            assert inp["parent"][b, pth[j] - 1] == pth[j - 1] - 1
            assert got["out_tokens"][b, j - 1] == inp["tokens"][b, pth[j] - 1]
        assert 0 <= got["out_tokens"][b, A] < inp["z_p"].shape[2]
        assert (got["out_tokens"][b, A + 1:] == -1).all() and (pth[A + 1:] == 0).all()
    return near


def _random_tree(rng, n):
    return np.array([-1] + [int(rng.integers(0, i)) for i in range(1, n)], np.int32)


@pytest.mark.parametrize("V,dt", [(16, "f32"), (1001, "bf16"), (20000, "bf16"), (4096, "f32")])
def test_tree_sample_matches_oracle(V, dt):
    rng = np.random.default_rng(V)
    shapes = [W.tree_static_scored((4, 3, 2, 1, 1, 1), 26), W.tree_tiny(), W.tree_chain(6), W.tree_star(10),
              np.array([-1], np.int32)]
    parents = [shapes[i % len(shapes)] for i in range(25)] + [_random_tree(rng, int(rng.integers(2, 40)))
                                                              for _ in range(25)]
    for T in (1.0, 0.7):
        inp = W.make_tree_sample_inputs(parents, V, dt, seed=V + int(10 * T), T=T)
        got = run_gpu(inp)
        assert (got["status"] == 0).all()
        ref = run_oracle(inp)
        assert compare(got, ref, inp) <= 3
        assert len(set(ref["accept_len"].tolist())) > 1


def test_tree_sample_full_size_eagle2_trees():
    """B = 16 EAGLE-2 trees of 60 nodes over the 128256-token vocabulary (bf16)."""
    w = W.WORKLOADS["eagle60"].scaled(L=16, L_lo=8)
    base = W.make_inputs(w, nan_guard=False)
    parents = [base["parent"][b, :int(base["num_nodes"][b])] for b in range(w.B)]
    inp = W.make_tree_sample_inputs(parents, 128256, "bf16", seed=5, T=1.0)
    got = run_gpu(inp)
    assert (got["status"] == 0).all()
    ref = run_oracle(inp)
    assert compare(got, ref, inp) <= 1


def test_single_child_trees_equal_the_chain_sampler():
    """A chain through the tree sampler takes the chain sampler's decisions (uniform c tests node c,
    the chain's last uniform is the tree's entry 0)."""
    K, V, B = 5, 3000, 64
    inp = W.make_tree_sample_inputs([W.tree_chain(K + 1)] * B, V, "bf16", seed=3)
    got = run_gpu(inp)
    zq_chain = np.ascontiguousarray(inp["z_q"][:, :K])
    u_chain = np.concatenate([inp["u"][:, 1:K + 1], inp["u"][:, :1]], axis=1)
    ch = tsd.chain_accept_sample(_dev(inp["z_p"]), _dev(zq_chain), torch.from_numpy(inp["tokens"][:, 1:]).cuda(),
                                 torch.from_numpy(np.ascontiguousarray(u_chain)).cuda(), 1.0)
    torch.cuda.synchronize()
    ref = run_oracle(inp)
    far = np.array([all(x >= ACC_MARGIN for x in m[:-1]) and m[-1] >= CDF_MARGIN for m in ref["margins"]])
    assert far.sum() >= B - 2
    assert np.array_equal(got["accept_len"][far], ch["accept_len"].cpu().numpy()[far])
    assert np.array_equal(got["out_tokens"][far, :K + 1], ch["out_tokens"].cpu().numpy()[far])


def _toy_logits(probs):
    return np.log(np.maximum(probs, 1e-30)).astype(np.float32)


def test_first_emitted_token_follows_the_target_on_the_gpu():
    """Root with 3 children drawn i.i.d. from q (V = 16): the first emitted token is distributed
    as p (chi-square)."""
    rng = np.random.default_rng(7)
    V, n, m = 16, 60000, 3
    p = rng.dirichlet(np.ones(V) * 0.7)
    q = rng.dirichlet(np.ones(V) * 0.7)
    N = m + 1
    zp = np.broadcast_to(_toy_logits(p), (n, N, V)).copy()
    zq = np.broadcast_to(_toy_logits(q), (n, N, V)).copy()
    tokens = np.zeros((n, N), np.int32)
    tokens[:, 1:] = rng.choice(V, size=(n, m), p=q)
    inp = {"parent": np.tile(np.array([-1] + [0] * m, np.int32), (n, 1)), "num_nodes": np.full(n, N, np.int32),
           "z_p": zp, "z_q": zq, "tokens": tokens, "u": rng.random((n, N), dtype=np.float32), "T": 1.0,
           "Dmax": 1, "dtype": "f32"}
    got = run_gpu(inp)
    counts = np.bincount(got["out_tokens"][:, 0], minlength=V)
    exp = p * n
    keep = exp >= 5
    obs = np.append(counts[keep], counts[~keep].sum())
    ex = np.append(exp[keep], exp[~keep].sum())
    obs, ex = obs[ex > 0], ex[ex > 0]
    assert stats.chisquare(obs, ex).pvalue > 1e-4


def test_first_two_tokens_follow_the_target_on_a_two_level_tree_gpu():
    """Root with 2 i.i.d. children, each with 2 i.i.d. children, Markov target P[x] and draft Q[x]
    (V = 4): the first two emitted tokens follow p(x1) p(x2 | x1)."""
    rng = np.random.default_rng(12)
    V, n = 4, 60000
    P = rng.dirichlet(np.ones(V), size=V)
    Q = rng.dirichlet(np.ones(V), size=V)
    parent = np.array([-1, 0, 0, 1, 1, 2, 2], np.int32)
    tokens = np.zeros((n, 7), np.int32)
    t1 = np.stack([rng.choice(V, size=n, p=Q[0]) for _ in range(2)], 1)
    tokens[:, 1:3] = t1
    for j, c in ((0, 3), (1, 5)):
        cum = np.cumsum(Q[t1[:, j]], axis=1)
        for k in range(2):
            r = rng.random(n)[:, None]
            tokens[:, c + k] = np.minimum((cum <= r).sum(1), V - 1)
    zp = _toy_logits(P[tokens])          # row n = the target after node n's token
    zq = _toy_logits(Q[tokens])
    inp = {"parent": np.tile(parent, (n, 1)), "num_nodes": np.full(n, 7, np.int32), "z_p": zp, "z_q": zq,
           "tokens": tokens, "u": rng.random((n, 7), dtype=np.float32), "T": 1.0, "Dmax": 2, "dtype": "f32"}
    got = run_gpu(inp)
    em = got["out_tokens"]
    A = got["accept_len"]
    second = np.where(A >= 1, em[:, 1], -1)
    # when the first token was the final draw, the second is a fresh target draw after it
    fresh = A == 0
    cumP = np.cumsum(P, axis=1)
    r = rng.random(n)
    second[fresh] = np.minimum((cumP[em[fresh, 0]] <= r[fresh, None]).sum(1), V - 1)
    counts = np.zeros((V, V))
    np.add.at(counts, (em[:, 0], second), 1)
    expected = (P[0][:, None] * P) * n
    assert stats.chisquare(counts.ravel(), expected.ravel()).pvalue > 1e-4


def test_flagged_and_too_wide_sequences():
    V = 64
    parents = [W.tree_static_scored((4, 3, 2, 1, 1, 1), 26), W.tree_star(300), W.tree_tiny()]
    inp = W.make_tree_sample_inputs(parents, V, "f32", seed=1)
    st = np.array([0, 0, 3 | (5 << 8)], np.int32)        # sequence 2 was flagged earlier
    got = run_gpu(inp, status=st)
    assert got["accept_len"][1] == -1 and got["accept_len"][2] == -1
    assert got["status"][1] == 1 and got["status"][2] == (3 | (5 << 8))   # 300 children > 256 at the root
    assert (got["out_tokens"][1:] == -1).all() and (got["path"][1:] == 0).all()
    ref = run_oracle({**inp, "parent": inp["parent"][:1], "num_nodes": inp["num_nodes"][:1], "z_p": inp["z_p"][:1],
                      "z_q": inp["z_q"][:1], "tokens": inp["tokens"][:1], "u": inp["u"][:1]})
    if all(x >= ACC_MARGIN for x in ref["margins"][0][:-1]):
        assert got["accept_len"][0] == ref["accept_len"][0]
