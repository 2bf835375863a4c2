"""TEST INFRASTRUCTURE ONLY: fp64 CPU oracle of the SSD / Saguaro outcome-cache construction.

"Speculative Speculative Decoding", technical summary sec. 2 and sec. 3 A-B: while the target
verifies round T, the draft predicts the verification outcome -- how many draft tokens will be
accepted and which bonus token the target will add -- and pre-drafts a continuation for each
likely outcome (the outcome cache; a hit sends the pre-drafted tokens straight to verification).
Cache construction spends a fixed budget unevenly: a geometric fan-out gives more of it to the
accepted lengths the acceptance rate makes likely.  Saguaro sampling lowers, while drafting, the
draft probability of the tokens the cache holds, which raises the residual mass the target's
bonus draw uses on exactly those tokens.

Reading restated here (the pages give the ideas, not the formulas):

  * accepted length a in 0..K for a K-token draft with per-token acceptance rate alpha:
    P(a) = alpha^a (1 - alpha) for a < K, P(K) = alpha^K;
  * fan-out: the S cache slots are apportioned to the lengths in proportion to P(a) by the
    largest-remainder rule (floor(S P(a)) each, then one more slot to the lengths with the
    largest remainders, ties -> shorter length);
  * keys: the n_a slots of length a go to the n_a most likely tokens (ties -> lower id) of the
    draft distribution at position a+1 (temperature T softmax of the draft logits) -- the
    position whose draft token a rejection at a+1 replaces, or the free token when a = K;
  * Saguaro: the draft token at position a+1 is drawn from q' proportional to q times beta on
    the tokens cached for length a (0 <= beta <= 1) and times 1 elsewhere, by the inverse CDF
    with a uniform u: the smallest t with sum_{v<=t} q'(v) > u sum_v q'(v).

Plain loops and numpy on small arrays.  Parity unpinned: none (tests/test_oracle_ssd_cache.py:
closed forms at alpha = 0 and 1 and a hand-worked apportionment, the proportionality bound,
beta = 1 and beta = 0 special cases, the residual-mass monotonicity the pages state, and a
chi-square of the draws against q').
"""
from __future__ import annotations

import numpy as np


def length_probs(alpha: float, K: int) -> np.ndarray:
    """P(a), a = 0..K, of the accepted length under a per-token acceptance rate alpha."""
    p = np.array([alpha ** a * (1.0 - alpha) for a in range(K)] + [alpha ** K], np.float64)
    return p


def geometric_fanout(S: int, alpha: float, K: int) -> np.ndarray:
    """Slots per accepted length (int64[K+1], summing to S), largest-remainder apportionment."""
    P = length_probs(alpha, K)
    share = S * P
    n = np.floor(share).astype(np.int64)
    left = S - int(n.sum())
    rem = share - n
    order = sorted(range(K + 1), key=lambda a: (-rem[a], a))
    for a in order[:left]:
        n[a] += 1
    return n


def softmax(z: np.ndarray, T: float) -> np.ndarray:
    x = z.astype(np.float64) / T
    x = np.exp(x - x.max())
    return x / x.sum()


def cache_keys(draft_logits: np.ndarray, n: np.ndarray, T: float = 1.0) -> list:
    """draft_logits [K+1, V]: row a = the draft distribution at position a+1.  Returns the
    outcome keys [(a, token)] ordered by length, then rank."""
    keys = []
    for a, cnt in enumerate(n):
        if cnt <= 0:
            continue
        q = softmax(draft_logits[a], T)
        order = np.lexsort((np.arange(len(q)), -q))
        keys.extend((a, int(t)) for t in order[:cnt])
    return keys


def saguaro_probs(logits: np.ndarray, cached, beta: float, T: float = 1.0) -> np.ndarray:
    """q' = q * (beta on the cached tokens, 1 elsewhere), renormalised (fp64)."""
    q = softmax(logits, T)
    w = np.ones_like(q)
    for t in cached:
        w[t] = beta
    qp = q * w
    s = qp.sum()
    return qp / s if s > 0 else q


def inverse_cdf(prob: np.ndarray, u: float, margin: list | None = None) -> int:
    """Smallest t with sum_{v<=t} prob[v] > u * sum(prob) (sequential scan).  With `margin`,
    appends the distance of the threshold to the nearest cumulative boundary of the chosen
    token, relative to the total."""
    total = float(prob.sum())
    thr = u * total
    acc = 0.0
    for t, x in enumerate(prob):
        prev = acc
        acc += float(x)
        if acc > thr:
            if margin is not None:
                margin.append(min(thr - prev, acc - thr) / total if total > 0 else 0.0)
            return t
    if margin is not None:
        margin.append(0.0)
    return int(np.nonzero(prob > 0)[0][-1])


def build_and_draft(draft_logits: np.ndarray, S: int, alpha: float, beta: float, u: np.ndarray, T: float = 1.0,
                    margins: list | None = None):
    """One sequence: fan-out, keys, and the K Saguaro-sampled draft tokens (u: K uniforms).

    Returns dict(n, keys, tokens, probs) with probs[j] = q' of position j+1; with `margins`,
    appends each draw's margin (see inverse_cdf)."""
    K = draft_logits.shape[0] - 1
    n = geometric_fanout(S, alpha, K)
    keys = cache_keys(draft_logits, n, T)
    tokens, probs = [], []
    for j in range(K):
        cached = [t for a, t in keys if a == j]
        qp = saguaro_probs(draft_logits[j], cached, beta, T)
        probs.append(qp)
        tokens.append(inverse_cdf(qp, float(u[j]), margins))
    return {"n": n, "keys": keys, "tokens": np.array(tokens, np.int32), "probs": probs}
