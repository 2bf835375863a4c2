"""GPU parity of the SSD / Saguaro outcome-cache build (tsd_ssd_cache_build) against the fp64
oracle in oracle/ssd_cache.py: the fan-out and the outcome keys bit-exact (the fan-out wherever no
share sits within rounding of an integer or of another remainder), the Saguaro draws bit-exact
where their inverse-CDF margin clears 2e-7 (the chain sampler's protocol); the draws' distribution
on the GPU (chi-square), and a forest rooted at the keys accepted by the greedy verify."""
import numpy as np
import pytest
import torch
from scipy import stats

import oracle
import tree_speculative_decoding_06_b200 as tsd
import workloads as W
from oracle import ssd_cache as sc

pytestmark = pytest.mark.gpu

CDF_MARGIN = 2e-7
FANOUT_MARGIN = 1e-9


def _dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run_gpu(inp, S, beta, T=1.0):
    r = tsd.ssd_cache_build(_dev(inp["draft_logits"]), torch.from_numpy(inp["alpha"]).cuda(), beta,
                            torch.from_numpy(inp["u"]).cuda() if inp["K"] > 0 else torch.zeros(
                                (inp["draft_logits"].shape[0], 1), dtype=torch.float32, device="cuda"),
                            S, T)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in r.items()}


def fanout_margin(S, alpha, K):
    """Smallest distance of a share S P(a) to an integer, or between two remainders: below rounding
    level the apportionment is not decided by the mathematics alone."""
    share = S * sc.length_probs(float(alpha), K)
    rem = share - np.floor(share)
    dist = np.minimum(rem, 1 - rem)
    d = dist[dist > 0].min(initial=1.0)        # exact integers (alpha 0, 1/2, 1) are computed alike
    r = np.sort(rem)
    gaps = np.diff(r)
    return min(d, gaps[gaps > 0].min(initial=1.0))


def compare(got, inp, S, beta, T=1.0):
    widen = (lambda z: W.as_f32(z, inp["dtype"]))
    B, K = inp["draft_logits"].shape[0], inp["K"]
    near = 0
    for b in range(B):
        m = []
        ref = sc.build_and_draft(widen(inp["draft_logits"][b]).astype(np.float64), S, float(inp["alpha"][b]), beta,
                                 inp["u"][b].astype(np.float64), T, m)
        if fanout_margin(S, inp["alpha"][b], K) < FANOUT_MARGIN:
            assert got["slots"][b].sum() == S
            near += 1
            continue
        assert got["slots"][b].tolist() == ref["n"].tolist(), b
        assert list(zip(got["key_len"][b].tolist(), got["key_tok"][b].tolist())) == ref["keys"], b
        for j in range(K):
            if m[j] >= CDF_MARGIN:
                assert got["draft_tokens"][b, j] == ref["tokens"][j], (b, j)
            else:
                near += 1
                assert ref["probs"][j][got["draft_tokens"][b, j]] > 0
    return near


@pytest.mark.parametrize("V,dt,K,S,beta", [(1000, "bf16", 4, 8, 0.5), (4096, "f32", 6, 32, 0.2),
                                           (20001, "bf16", 7, 64, 0.0), (300, "f32", 3, 256, 1.0),
                                           (50, "bf16", 0, 20, 0.5)])
def test_ssd_cache_matches_oracle(V, dt, K, S, beta):
    inp = W.make_ssd_inputs(24, K, V, dt, seed=V + K)
    inp["alpha"][:3] = [0.0, 1.0, 0.5]          # closed forms: everything at length 0 / K, exact halves
    got = run_gpu(inp, S, beta, T=0.8 if dt == "f32" else 1.0)
    assert compare(got, inp, S, beta, T=0.8 if dt == "f32" else 1.0) <= 2
    assert got["slots"][0].tolist() == [S] + [0] * K
    assert got["slots"][1].tolist() == [0] * K + [S]


def test_ssd_cache_full_size():
    """8 sequences, 7-token drafts, 8 outcome slots each, the 128256-token vocabulary (bf16)."""
    inp = W.make_ssd_inputs(8, 7, 128256, "bf16", seed=11)
    got = run_gpu(inp, 8, 0.5)
    assert compare(got, inp, 8, 0.5) <= 2   # two of the 56 draws of this fixture sit within 2e-7 of a boundary


def test_ties_go_to_the_lower_token():
    inp = W.make_ssd_inputs(4, 2, 640, "bf16", seed=3)
    z = inp["draft_logits"]
    top = W.f32_to_bf16_bits(np.array([20.0], np.float32))[0]
    z[:, :, [5, 77, 300, 301, 639]] = top             # five equal maxima in every row
    inp["alpha"][:] = 0.5
    got = run_gpu(inp, 6, 0.5)
    assert compare(got, inp, 6, 0.5) == 0
    for b in range(4):   # length 0 has 3 slots, length 1 two, length 2 one: the lowest tied ids
        assert got["key_tok"][b].tolist() == [5, 77, 300, 5, 77, 5]


def test_saguaro_draws_follow_the_reweighted_draft():
    """Many draws from one row (V = 16): chi-square against q' (beta on the 3 cached tokens)."""
    rng = np.random.default_rng(4)
    n, V = 40000, 16
    z = (rng.standard_normal(V) * 1.5).astype(np.float32)
    inp = {"draft_logits": np.broadcast_to(z, (n, 2, V)).copy(), "alpha": np.full(n, 0.5, np.float32),
           "u": rng.random((n, 1), dtype=np.float32), "dtype": "f32", "K": 1, "V": V}
    got = run_gpu(inp, 6, 0.25)                         # alpha 1/2, K 1: 3 slots per length
    cached = got["key_tok"][0, :3].tolist()
    qp = sc.saguaro_probs(z.astype(np.float64), cached, 0.25)
    counts = np.bincount(got["draft_tokens"][:, 0], minlength=V)
    keep = qp * n >= 5
    obs = np.append(counts[keep], counts[~keep].sum())
    ex = np.append(qp[keep] * n, qp[~keep].sum() * n)
    obs, ex = obs[ex > 0], ex[ex > 0]
    assert stats.chisquare(obs, ex).pvalue > 1e-4


def test_forest_rooted_at_the_keys_is_verified_by_the_greedy_step():
    """The keys of the likeliest accepted length root a forest of pre-drafted chains; the greedy
    verify with the real outcome token as root_key hits the subtree of that key (or misses)."""
    inp = W.make_ssd_inputs(6, 3, 512, "bf16", seed=8)
    got = run_gpu(inp, 8, 0.5)
    parents, roots_tok = [], []
    for b in range(6):
        a0 = int(np.argmax(got["slots"][b]))
        keys = [t for L, t in zip(got["key_len"][b], got["key_tok"][b]) if L == a0]
        par = []
        for r, _ in enumerate(keys):      # each root followed by a chain of 2 pre-drafted tokens
            base = len(par)
            par.extend([-1, base, base + 1])
        parents.append(np.array(par, np.int32))
        roots_tok.append(keys)
    x = W.make_custom_inputs(parents, [4] * 6, Hq=2, Hkv=1, d=64, dtype="bf16", V=512, seed=9, forest=True,
                             plant_p=0.9)
    for b in range(6):
        for r, t in enumerate(roots_tok[b]):
            x["tokens"][b, 3 * r] = t
    rk = [roots_tok[b][b % len(roots_tok[b])] if b < 5 else 511 - 0 for b in range(6)]
    if rk[5] in roots_tok[5]:
        rk[5] = -7
    x["root_key"] = np.array(rk, np.int32)
    ref = oracle.accept_greedy(x)
    xd = {k: (torch.from_numpy(v).cuda() if isinstance(v, np.ndarray) and v.dtype in (np.int32,) else v)
          for k, v in x.items()}
    prep = tsd.tree_prepare(xd["parent"], xd["num_nodes"], int(x["Dmax"]), True)
    r = tsd.tree_accept_greedy(_dev(x["logits"]), xd["tokens"], prep["parent_s"], xd["num_nodes"], xd["root_key"],
                               int(x["Dmax"]), status=prep["status"])
    torch.cuda.synchronize()
    assert np.array_equal(r["accept_len"].cpu().numpy(), ref["accept_len"])
    assert np.array_equal(r["out_tokens"].cpu().numpy(), ref["out_tokens"])
    assert (ref["accept_len"][:5] >= 0).all() and ref["accept_len"][5] == -1
