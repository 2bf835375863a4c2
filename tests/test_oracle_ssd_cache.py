"""Pins of the SSD / Saguaro outcome-cache oracle (oracle/ssd_cache.py)."""
import numpy as np
import pytest
from scipy import stats

from oracle import ssd_cache as sc


def test_length_probabilities_sum_to_one_and_are_geometric():
    for alpha in (0.0, 0.3, 0.8, 1.0):
        P = sc.length_probs(alpha, 5)
        assert abs(P.sum() - 1.0) < 1e-15
        if 0.0 < alpha < 1.0:
            assert np.allclose(P[1:5] / P[:4], alpha)


def test_fanout_closed_forms_and_hand_example():
    assert sc.geometric_fanout(8, 0.0, 4).tolist() == [8, 0, 0, 0, 0]     # every draft rejected at once
    assert sc.geometric_fanout(8, 1.0, 4).tolist() == [0, 0, 0, 0, 8]     # every draft accepted
    # alpha = 1/2, K = 3: P = (1/2, 1/4, 1/8, 1/8) -> 8 slots split 4, 2, 1, 1 exactly
    assert sc.geometric_fanout(8, 0.5, 3).tolist() == [4, 2, 1, 1]
    # remainders: alpha = 0.6, K = 2, S = 5: S P = (2.0, 1.2, 1.8) -> (2, 1, 2)
    assert sc.geometric_fanout(5, 0.6, 2).tolist() == [2, 1, 2]


@pytest.mark.parametrize("S,alpha,K", [(8, 0.7, 5), (64, 0.55, 7), (3, 0.9, 6), (100, 0.2, 4)])
def test_fanout_is_a_largest_remainder_apportionment(S, alpha, K):
    n = sc.geometric_fanout(S, alpha, K)
    share = S * sc.length_probs(alpha, K)
    assert n.sum() == S and (n >= 0).all()
    assert np.all(np.abs(n - share) < 1.0)                 # within one slot of the exact share
    # no length whose remainder is smaller got the extra slot while a larger one did not
    got = n - np.floor(share)
    rem = share - np.floor(share)
    for a in range(K + 1):
        for b in range(K + 1):
            if got[a] == 1 and got[b] == 0:
                assert rem[a] > rem[b] or (rem[a] == rem[b] and a < b)


def test_cache_keys_are_the_top_tokens_per_length():
    rng = np.random.default_rng(0)
    z = rng.standard_normal((4, 30))
    n = np.array([3, 0, 2, 1])
    keys = sc.cache_keys(z, n)
    assert [a for a, _ in keys] == [0, 0, 0, 2, 2, 3]
    for a, cnt in enumerate(n):
        mine = [t for b, t in keys if b == a]
        assert mine == list(np.argsort(-z[a], kind="stable")[:cnt])


def test_saguaro_special_cases_and_residual_mass():
    rng = np.random.default_rng(1)
    z = rng.standard_normal(50) * 2
    q = sc.softmax(z, 1.0)
    cached = [3, 7, 11]
    assert np.allclose(sc.saguaro_probs(z, cached, 1.0), q)                 # beta = 1: plain draft
    q0 = sc.saguaro_probs(z, cached, 0.0)                                    # beta = 0: cached removed
    assert (q0[cached] == 0).all() and abs(q0.sum() - 1) < 1e-15
    assert np.allclose(q0[[i for i in range(50) if i not in cached]],
                       q[[i for i in range(50) if i not in cached]] / (1 - q[cached].sum()))
    # the pages' claim: lowering q on the cached tokens raises the residual max(p - q, 0) there
    for _ in range(20):
        p = sc.softmax(rng.standard_normal(50) * 2, 1.0)
        r_before = np.maximum(p - q, 0)[cached].sum()
        for beta in (0.7, 0.3, 0.0):
            r_after = np.maximum(p - sc.saguaro_probs(z, cached, beta), 0)[cached].sum()
            assert r_after >= r_before - 1e-15


def test_inverse_cdf_draws_follow_the_reweighted_draft():
    rng = np.random.default_rng(2)
    z = rng.standard_normal(8)
    qp = sc.saguaro_probs(z, [0, 5], 0.25)
    n = 40000
    draws = np.array([sc.inverse_cdf(qp, u) for u in rng.random(n)])
    counts = np.bincount(draws, minlength=8)
    chi2, pval = stats.chisquare(counts, qp * n)
    assert pval > 1e-4
    assert sc.inverse_cdf(qp, 0.0) == int(np.nonzero(qp > 0)[0][0])


def test_build_and_draft_one_sequence():
    rng = np.random.default_rng(3)
    K, V = 4, 64
    z = rng.standard_normal((K + 1, V)) * 2
    r = sc.build_and_draft(z, S=8, alpha=0.6, beta=0.5, u=rng.random(K))
    assert r["n"].sum() == 8 and len(r["keys"]) == 8 and r["tokens"].shape == (K,)
    for j in range(K):
        cached = [t for a, t in r["keys"] if a == j]
        assert np.allclose(r["probs"][j], sc.saguaro_probs(z[j], cached, 0.5))
