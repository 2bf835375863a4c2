"""GPU parity: greedy tree acceptance and chain sampling (bit-exact, with the margin protocol for
sampling decisions) and the KV commit (byte-exact), through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import tree_speculative_decoding_06_b200 as tsd
import workloads as W
from gpu_helpers import gpu_prepare
from tree_speculative_decoding_06_b200.step import to_device, VerifyStep

pytestmark = pytest.mark.gpu

# Decision margins below which the kernel's arithmetic (fp32 exponentials, ~1e-7 relative and
# independent per token; everything else fp64) may legitimately land on the other side of a
# boundary than the fp64 oracle: an accept test |u q - p| / max(p, u q), and the distance of the
# inverse-CDF threshold to the nearest cumulative boundary relative to the total mass.
ACC_MARGIN = 1e-5
CDF_MARGIN = 2e-7


def gpu_accept(inp):
    x = to_device(inp)
    forest = bool(getattr(inp["workload"], "forest", False))
    prep = gpu_prepare(x, forest)
    r = tsd.tree_accept_greedy(x["logits"], x["tokens"], prep["parent_s"], x["num_nodes"], x.get("root_key"),
                               int(x["Dmax"]), status=prep["status"])
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in r.items()}, prep["status"].cpu().numpy()


def assert_accept_equal(got, ref):
    assert np.array_equal(got["accept_len"], ref["accept_len"]), (got["accept_len"], ref["accept_len"])
    assert np.array_equal(got["path"], ref["path"])
    assert np.array_equal(got["out_tokens"], ref["out_tokens"])


@pytest.mark.parametrize("name", ["tiny", "tree26", "eagle60", "forest"])
def test_accept_greedy_full(name):
    inp = W.make_inputs(W.WORKLOADS[name])
    got, st = gpu_accept(inp)
    assert (st == 0).all()
    ref = oracle.accept_greedy(inp)
    assert_accept_equal(got, ref)
    if name == "forest":   # the fixture hits some roots and misses others
        assert (ref["accept_len"] == -1).any() and (ref["accept_len"] >= 0).any()


def test_accept_greedy_edge_cases():
    rng = np.random.default_rng(3)
    V = 1001                                            # not a multiple of 8: scalar path
    parents = [W.tree_chain(1), W.tree_tiny(), W.tree_static_scored((4, 3, 2, 1, 1, 1), 26), W.tree_chain(7)]
    inp = W.make_custom_inputs(parents, [1, 1, 1, 1], Hq=2, Hkv=1, d=64, dtype="bf16", V=V, seed=2, plant_p=0.9)
    lg = inp["logits"]
    lg[1, 0, 5:9] = W.f32_to_bf16_bits(np.array([30, 30, 30, 30], np.float32))   # 4-way tie -> lowest (5)
    lg[2, 0] = W.BF16_NAN                                                             # all-NaN row -> 0
    lg[2, 1, :] = W.f32_to_bf16_bits(np.full(V, -np.inf, np.float32))               # all -inf -> 0
    lg[3, 2, 700] = W.BF16_NAN
    inp["tokens"][1, 1] = 5
    inp["tokens"][1, 2] = 5                                  # duplicate sibling tokens, both match
    got, st = gpu_accept(inp)
    ref = oracle.accept_greedy(inp)
    assert_accept_equal(got, ref)
    # fp32 logits and V % 8 == 0
    inp = W.make_custom_inputs(parents, [1, 1, 1, 1], Hq=2, Hkv=1, d=64, dtype="f32", V=4096, seed=4, plant_p=0.8)
    got, _ = gpu_accept(inp)
    assert_accept_equal(got, oracle.accept_greedy(inp))


def test_accept_forest_hit_each_root_and_miss():
    w = W.WORKLOADS["forest"].scaled(B=10, L=4, V=4000)
    inp = W.make_inputs(w, seed=21)
    roots = np.nonzero(inp["parent"][0] < 0)[0]
    keys = [int(inp["tokens"][b, roots[b % len(roots)]]) for b in range(8)] + [-5, 3999999]
    inp["root_key"] = np.array(keys, np.int32)
    inp["tokens"][8:, roots] = inp["tokens"][0, roots]
    got, _ = gpu_accept(inp)
    ref = oracle.accept_greedy(inp)
    assert_accept_equal(got, ref)
    assert (ref["accept_len"][8:] == -1).all() and (ref["accept_len"][:8] >= 0).all()


def gpu_sample(zp, zq, x, u, T):
    dev = lambda a: (torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16) if a.dtype == np.uint16
                     else torch.from_numpy(a).cuda())
    r = tsd.chain_accept_sample(dev(zp), dev(zq), torch.from_numpy(x).cuda(), torch.from_numpy(u).cuda(), T)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in r.items()}


def final_interval_distance(zp, zq, u, T, b, j, tok):
    """Validity of a near-boundary draw: distance (relative to the total mass) between the
    threshold u_K * R and the cumulative interval the GPU's token owns under the fp64
    distribution; 0 when the token is the oracle's own choice."""
    dt = "bf16" if zp.dtype == np.uint16 else "f32"
    K = zq.shape[1]
    zpj = W.as_f32(zp[b, j], dt).astype(np.float64) / T
    p = np.exp(zpj - zpj.max())
    p /= p.sum()
    r = p
    if j < K:
        zqj = W.as_f32(zq[b, j], dt).astype(np.float64) / T
        q = np.exp(zqj - zqj.max())
        q /= q.sum()
        r = np.maximum(p - q, 0.0)
        if r.sum() <= 0:
            r = p
    R = r.sum()
    c = np.cumsum(r)
    thr = float(u[b, K]) * R
    lo = c[tok - 1] if tok > 0 else 0.0
    hi = c[tok]
    if r[tok] <= 0:
        return np.inf
    return 0.0 if lo <= thr < hi else min(abs(thr - lo), abs(thr - hi)) / R


def final_distribution_mass(zp, zq, T, b, j, tok):
    """fp64 mass of `tok` under the distribution the final draw at position j samples from: the
    residual max(p_j - q_j, 0) after a rejection at j < K (p_j if that residual is empty), p_K
    when every draft was accepted.  A drawn token must have positive mass there."""
    dt = "bf16" if zp.dtype == np.uint16 else "f32"
    K = zq.shape[1]
    zpj = W.as_f32(zp[b, j], dt).astype(np.float64) / T
    p = np.exp(zpj - zpj.max())
    p /= p.sum()
    if j == K:
        return float(p[tok])
    zqj = W.as_f32(zq[b, j], dt).astype(np.float64) / T
    q = np.exp(zqj - zqj.max())
    q /= q.sum()
    r = np.maximum(p - q, 0.0)
    return float(r[tok] if r.sum() > 0 else p[tok])


def compare_sampling(got, ref, K, zp=None, zq=None, u=None, T=None, x=None):
    """Bit-exact on every sequence whose decisions all clear their margins.  A sequence with a
    decision near its margin is checked for validity instead:
      * accept tests: every test before the first near one clears its margin, so the kernel must
        accept exactly as the oracle did up to there (A >= that index); the A emitted tokens
        before the draw are the drafts x[:A]; the drawn token has positive fp64 mass under the
        distribution the draw at A samples from; every entry past A is -1;
      * a near final draw with clear tests: the same accept decisions, and a token whose
        cumulative interval lies within CDF_MARGIN of the threshold.
    Returns the number of near-margin sequences."""
    m = ref["margin"]
    acc_near = (m[:, :K] < ACC_MARGIN).any(1)
    cdf_near = m[:, K] < CDF_MARGIN
    far = ~(acc_near | cdf_near)
    assert np.array_equal(got["accept_len"][far], ref["accept_len"][far])
    assert np.array_equal(got["out_tokens"][far], ref["out_tokens"][far])
    A = got["accept_len"]
    assert ((A >= 0) & (A <= K)).all()
    for b in np.nonzero(acc_near)[0]:
        j0 = int(np.nonzero(m[b, :K] < ACC_MARGIN)[0][0])
        a = int(A[b])
        assert a >= j0, (b, a, j0)
        if x is not None:
            assert np.array_equal(got["out_tokens"][b, :a], x[b, :a])
        else:
            n = min(a, int(ref["accept_len"][b]))
            assert np.array_equal(got["out_tokens"][b, :n], ref["out_tokens"][b, :n])
        assert (got["out_tokens"][b, a + 1:] == -1).all()
        tok = int(got["out_tokens"][b, a])
        assert 0 <= tok < (zp.shape[2] if zp is not None else np.iinfo(np.int32).max)
        if zp is not None:
            assert final_distribution_mass(zp, zq, T, b, a, tok) > 0.0, (b, a, tok)
    for b in np.nonzero(cdf_near & ~acc_near)[0]:
        j = int(ref["accept_len"][b])
        assert got["accept_len"][b] == j
        assert np.array_equal(got["out_tokens"][b, :j], ref["out_tokens"][b, :j])
        if zp is not None:
            assert final_interval_distance(zp, zq, u, T, b, j, int(got["out_tokens"][b, j])) <= CDF_MARGIN
    return int((~far).sum())


def test_chain_sample_full_size():
    inp = W.make_inputs(W.WORKLOADS["chain5"])
    got = gpu_sample(inp["z_p"], inp["z_q"], inp["x"], inp["u"], 1.0)
    ref = oracle.chain_sample(inp["z_p"], inp["z_q"], inp["x"], inp["u"], 1.0)
    n_near = compare_sampling(got, ref, 5, inp["z_p"], inp["z_q"], inp["u"], 1.0, inp["x"])
    assert n_near <= 2
    assert len(set(ref["accept_len"].tolist())) > 1   # the fixture exercises several accepted lengths


@pytest.mark.parametrize("V,dt", [(16, "f32"), (1001, "bf16"), (20000, "bf16"), (8192, "f32")])
def test_chain_sample_small(V, dt):
    rng = np.random.default_rng(V)
    B, K = 300, 4
    zpf = rng.standard_normal((B, K + 1, V)).astype(np.float32) * 2
    zqf = zpf[:, :K] + rng.standard_normal((B, K, V)).astype(np.float32) * 0.8
    zp = W.f32_to_bf16_bits(zpf) if dt == "bf16" else zpf
    zq = W.f32_to_bf16_bits(zqf) if dt == "bf16" else zqf
    x = rng.integers(0, V, size=(B, K)).astype(np.int32)
    am = W.as_f32(zq, dt).argmax(-1)
    x = np.where(rng.random((B, K)) < 0.7, am, x).astype(np.int32)
    u = rng.random((B, K + 1), dtype=np.float32)
    for T in (1.0, 0.7):
        got = gpu_sample(zp, zq, x, u, T)
        ref = oracle.chain_sample(zp, zq, x, u, T)
        assert compare_sampling(got, ref, K, zp, zq, u, T, x) <= 3
    got = gpu_sample(zp, zq, x, u, 0.0)
    ref = oracle.chain_sample(zp, zq, x, u, 0.0)
    assert np.array_equal(got["accept_len"], ref["accept_len"])
    assert np.array_equal(got["out_tokens"], ref["out_tokens"])


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_chain_sample_masked_vocabulary(dt):
    """-inf logits (a masked vocabulary, 30% of the tokens) in every target and draft row, at
    T = 0.7 (an exponent constant whose fp32 split has a negative low part) and T = 1: the masked
    tokens carry no mass, are never emitted, and every decision is the oracle's."""
    rng = np.random.default_rng(23)
    B, K, V = 128, 4, 4096
    zpf = rng.standard_normal((B, K + 1, V)).astype(np.float32) * 2
    zqf = zpf[:, :K] + rng.standard_normal((B, K, V)).astype(np.float32) * 0.8
    masked = rng.random(V) < 0.3
    zpf[..., masked] = -np.inf
    zqf[..., masked] = -np.inf
    zp = W.f32_to_bf16_bits(zpf) if dt == "bf16" else zpf
    zq = W.f32_to_bf16_bits(zqf) if dt == "bf16" else zqf
    open_ids = np.nonzero(~masked)[0]
    x = open_ids[rng.integers(0, len(open_ids), size=(B, K))].astype(np.int32)
    am = W.as_f32(zq, dt).argmax(-1)
    x = np.where(rng.random((B, K)) < 0.7, am, x).astype(np.int32)
    u = rng.random((B, K + 1), dtype=np.float32)
    for T in (0.7, 1.0):
        got = gpu_sample(zp, zq, x, u, T)
        ref = oracle.chain_sample(zp, zq, x, u, T)
        assert compare_sampling(got, ref, K, zp, zq, u, T, x) <= 3
        emitted = got["out_tokens"][got["out_tokens"] >= 0]
        assert not masked[emitted].any()


def test_chain_sample_distribution_gpu():
    """The GPU sampler preserves the target distribution (chi-square, vocab 16, K = 3, toy
    Markov target and draft as in the oracle's own distribution test)."""
    from scipy import stats
    from test_oracle_sample import markov_tables, draw
    Vs, K = 16, 3
    P, Q = markov_tables(0)
    rng = np.random.default_rng(11)
    n = 60000
    firsts = []
    for _ in range(3):
        x0 = np.full(n, 3)
        xs = [x0]
        for _ in range(K):
            xs.append(draw(rng, Q[xs[-1]]))
        ctx = np.stack(xs, 1)
        zp = np.log(P[ctx]).astype(np.float32)
        zq = np.ascontiguousarray(np.log(Q[ctx[:, :K]]).astype(np.float32))
        got = gpu_sample(zp, zq, np.ascontiguousarray(ctx[:, 1:].astype(np.int32)),
                         rng.random((n, K + 1)).astype(np.float32), 1.0)
        firsts.append(got["out_tokens"][:, 0])
    t1 = np.concatenate(firsts)
    exp = P[3] * len(t1)
    keep = exp >= 5
    assert stats.chisquare(np.bincount(t1, minlength=Vs)[keep], exp[keep] * keep.sum() / keep.sum()
                           * len(t1) / exp[keep].sum()).pvalue > 1e-4


def test_chain_sample_p_equals_q_accepts_all():
    rng = np.random.default_rng(9)
    B, K, V = 64, 5, 3000
    z = W.f32_to_bf16_bits(rng.standard_normal((B, K + 1, V)).astype(np.float32))
    x = rng.integers(0, V, size=(B, K)).astype(np.int32)
    u = rng.random((B, K + 1), dtype=np.float32) * np.float32(0.999)
    got = gpu_sample(z, np.ascontiguousarray(z[:, :K]), x, u, 1.0)
    assert (got["accept_len"] == K).all()


# ----------------------------------------------------------------------------- commit
def _commit_case(paged, dtype="bf16", seed=0):
    parents = [W.tree_static_scored((4, 3, 2, 1, 1, 1), 26), W.tree_tiny(), W.tree_chain(5), W.tree_tiny()]
    return W.make_custom_inputs(parents, [33, 0, 70, 15], Hq=4, Hkv=2, d=128 if dtype == "bf16" else 64,
                                dtype=dtype, seed=seed, paged=paged, nan_guard=False, plant_p=0.8)


def gpu_commit(inp, accept_len, path, mode, k_cache=None, v_cache=None, prefix_len=None, status=None):
    x = to_device(inp)
    paged = "k_pages" in x
    kc = torch.from_numpy((k_cache if k_cache is not None else (inp["k_pages"] if paged else inp["k_cache"]))
                          .view(np.int16) if inp["q"].dtype == np.uint16 else
                          (k_cache if k_cache is not None else (inp["k_pages"] if paged else inp["k_cache"]))).cuda()
    vc = torch.from_numpy((v_cache if v_cache is not None else (inp["v_pages"] if paged else inp["v_cache"]))
                          .view(np.int16) if inp["q"].dtype == np.uint16 else
                          (v_cache if v_cache is not None else (inp["v_pages"] if paged else inp["v_cache"]))).cuda()
    if inp["q"].dtype == np.uint16:
        kc, vc = kc.view(torch.bfloat16), vc.view(torch.bfloat16)
    pl = torch.from_numpy((inp["prefix_len"] if prefix_len is None else prefix_len).copy()).cuda()
    st = torch.from_numpy(np.zeros(len(pl), np.int32) if status is None else status.copy()).cuda()
    al = torch.from_numpy(np.asarray(accept_len, np.int32)).cuda()
    pa = None if path is None else torch.from_numpy(np.asarray(path, np.int32)).cuda()
    kt, vt = (None, None) if mode == "inplace" else (x["k_tree"], x["v_tree"])
    if paged:
        tsd.kv_commit_paged(kc, vc, x["block_table"], pl, kt, vt, pa, al, x["num_nodes"], int(inp["Dmax"]), mode,
                            status=st, Nmax=inp["parent"].shape[1])
    else:
        tsd.kv_commit(kc, vc, pl, kt, vt, pa, al, x["num_nodes"], int(inp["Dmax"]), mode, status=st,
                      Nmax=inp["parent"].shape[1])
    torch.cuda.synchronize()
    cast = (lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)) if inp["q"].dtype == np.uint16 else \
        (lambda t: t.cpu().numpy())
    return cast(kc), cast(vc), pl.cpu().numpy(), st.cpu().numpy()


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_commit_path_matches_oracle(paged, dtype):
    inp = _commit_case(paged, dtype)
    acc = oracle.accept_greedy(inp)
    kc, vc, pl, st = gpu_commit(inp, acc["accept_len"], acc["path"], "path")
    rk, rv, rpl, rst = oracle.kv_commit(inp, acc["accept_len"], acc["path"], "path")
    assert (st == 0).all() and np.array_equal(pl, rpl)
    assert np.array_equal(kc, rk) and np.array_equal(vc, rv)   # byte-exact, guard rows included


@pytest.mark.parametrize("paged", [False, True])
def test_commit_inplace_and_length(paged):
    inp = _commit_case(paged, seed=1)
    acc = oracle.accept_greedy(inp)
    from gpu_helpers import lay_tree_in_cache
    lay = lay_tree_in_cache(inp)
    key = "k_pages" if paged else "k_cache"
    vkey = "v_pages" if paged else "v_cache"
    kc, vc, pl, st = gpu_commit(inp, acc["accept_len"], acc["path"], "inplace", k_cache=lay[key], v_cache=lay[vkey])
    rk, rv, rpl, _ = oracle.kv_commit(inp, acc["accept_len"], acc["path"], "inplace", k_cache=lay[key],
                                      v_cache=lay[vkey])
    assert (st == 0).all() and np.array_equal(pl, rpl)
    assert np.array_equal(kc, rk) and np.array_equal(vc, rv)
    A = np.array([3, 0, 4, 2], np.int32)
    kc, vc, pl, st = gpu_commit(inp, A, None, "length")
    rk, rv, rpl, _ = oracle.kv_commit(inp, A, None, "length")
    assert np.array_equal(kc, rk) and np.array_equal(vc, rv) and np.array_equal(pl, rpl)


def test_commit_errors_leave_cache_untouched():
    inp = _commit_case(False, seed=3)
    path = np.zeros((4, 7), np.int32)
    path[0, :2] = [1, 99]
    path[3, :2] = [1, 2]
    A = np.array([1, -1, 2, 1], np.int32)
    pl = inp["prefix_len"].copy()
    pl[2] = inp["k_cache"].shape[2] - 2
    status = np.array([0, 0, 0, 3], np.int32)            # sequence 3 was flagged earlier
    kc, vc, pl2, st = gpu_commit(inp, A, path, "path", prefix_len=pl, status=status)
    assert st.tolist() == [1, 0, 6, 3]
    assert np.array_equal(pl2, pl)
    assert np.array_equal(kc, inp["k_cache"]) and np.array_equal(vc, inp["v_cache"])


# ----------------------------------------------------------------------------- whole step
_STEP_CASES = {}


def _step_case(name):
    """Inputs of the whole-step test and the oracle's outputs on them (attention of every row,
    acceptance, commit), computed once per workload and shared by the three schedules."""
    if name not in _STEP_CASES:
        w = W.WORKLOADS[name]
        if name == "forest":       # 2 x 512 nodes x 32 heads: every row is checked
            w = w.scaled(B=2, L=700)
        elif name in ("chain5", "eagle60"):
            w = w.scaled(B=min(w.B, 4), L=min(w.L, 3000), L_lo=None if w.L_lo is None else 500)
        inp = W.make_inputs(w, nan_guard=False)
        att = oracle.attention_rows(inp)
        if w.accept == "greedy":
            acc = oracle.accept_greedy(inp)
            com = oracle.kv_commit(inp, acc["accept_len"], acc["path"], "path")
        else:
            acc = oracle.chain_sample(inp["z_p"], inp["z_q"], inp["x"], inp["u"], inp["T"])
            com = oracle.kv_commit(inp, acc["accept_len"], None, "length")
        _STEP_CASES[name] = (w, inp, att, acc, com)
    return _STEP_CASES[name]


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.cpu().numpy()


@pytest.mark.parametrize("name,schedule", [(n, s) for n in ("tiny", "tree26", "eagle60", "forest")
                                            for s in ("overlap", "fused", "serial")] +
                         [("chain5", "overlap"), ("chain5", "serial")])
def test_verify_step_matches_oracle(name, schedule):
    """The whole step under each schedule: the attention output of every row within tolerance,
    acceptance bit-exact (margin protocol for sampling), and the K and V caches byte-exact after
    the commit (guard rows included), with prefix_len advanced as the oracle's commit does."""
    from gpu_helpers import TOL
    w, inp, (ref_o, _, rows), ref, (rk, rv, rpl, _) = _step_case(name)
    x = to_device(inp)
    step = VerifyStep.for_inputs(x, schedule=schedule)
    res = step.run(x)
    torch.cuda.synchronize()
    assert (res["status"].cpu().numpy() == 0).all()
    out = res["out"].float().cpu().numpy().astype(np.float64)
    got_o = np.stack([out[b, i, h] for (b, i, h) in rows])
    atol, rtol = TOL["bf16" if w.dtype == "bf16" else "f32"]
    assert not np.isnan(got_o).any()
    assert (np.abs(got_o - ref_o) <= atol + rtol * np.abs(ref_o)).all(), np.abs(got_o - ref_o).max()
    if w.accept == "greedy":
        assert np.array_equal(res["accept_len"].cpu().numpy(), ref["accept_len"])
        assert np.array_equal(res["path"].cpu().numpy(), ref["path"])
        assert np.array_equal(res["out_tokens"].cpu().numpy(), ref["out_tokens"])
    else:
        got = {"accept_len": res["accept_len"].cpu().numpy(), "out_tokens": res["out_tokens"].cpu().numpy()}
        assert compare_sampling(got, ref, w.K, inp["z_p"], inp["z_q"], inp["u"], inp["T"], inp["x"]) <= 1
        if not np.array_equal(got["accept_len"], ref["accept_len"]):
            pytest.skip("a near-margin sampling decision differs from the oracle's: caches not comparable")
    assert np.array_equal(x["prefix_len"].cpu().numpy(), rpl)
    kkey, vkey = ("k_pages", "v_pages") if w.paged else ("k_cache", "v_cache")
    assert np.array_equal(_bits(x[kkey]), rk)
    assert np.array_equal(_bits(x[vkey]), rv)


def test_schedules_agree_on_a_sequence_the_attention_flags():
    """A bad block id inside one sequence's prefix makes the attention flag that sequence
    (TSD_ERR_CAPACITY) while the acceptance may already be running on the side stream.  Every
    schedule must leave the same status, caches and prefix lengths, the flagged sequence's cache
    untouched and its attention rows zero, and agree with the oracle on the other sequences."""
    w = W.WORKLOADS["eagle60"].scaled(B=3, L=600, L_lo=300)
    inp = W.make_inputs(w, nan_guard=False)
    bad_b = 1
    inp["block_table"] = inp["block_table"].copy()
    inp["block_table"][bad_b, 2] = 1 << 30              # inside its prefix: prefix_len >= 300 > 2 * 16
    ref = oracle.accept_greedy(inp)
    outcomes = []
    for schedule in ("overlap", "fused", "serial"):
        x = to_device(inp)
        step = VerifyStep.for_inputs(x, schedule=schedule)
        res = step.run(x)
        torch.cuda.synchronize()
        st = res["status"].cpu().numpy()
        assert (st & 0xFF).tolist() == [0 if b != bad_b else 6 for b in range(w.B)], st
        good = st == 0
        assert np.array_equal(res["accept_len"].cpu().numpy()[good], ref["accept_len"][good])
        assert np.array_equal(res["out_tokens"].cpu().numpy()[good], ref["out_tokens"][good])
        assert (res["out"][bad_b].float() == 0).all()
        outcomes.append((st, x["prefix_len"].cpu().numpy(), _bits(x["k_pages"]), _bits(x["v_pages"])))
    for o in outcomes[1:]:
        for a, b in zip(outcomes[0], o):
            assert np.array_equal(a, b)
    assert outcomes[0][1][bad_b] == inp["prefix_len"][bad_b]
