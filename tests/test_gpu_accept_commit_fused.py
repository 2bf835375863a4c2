"""GPU parity of the fused acceptance + commit call (tsd_tree_accept_commit) and of the
device-resident decoding loop it enables: the acceptance outputs bit-exact and the cache bytes,
prefix lengths and token history byte-exact against the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import tree_speculative_decoding_06_b200 as tsd
import workloads as W
from gpu_helpers import gpu_prepare, lay_tree_in_cache, sample_rows, to_np
from tree_speculative_decoding_06_b200.step import to_device, VerifyStep

pytestmark = pytest.mark.gpu


def _case(paged, dtype="bf16", seed=0):
    parents = [W.tree_static_scored((4, 3, 2, 1, 1, 1), 26), W.tree_tiny(), W.tree_chain(5), W.tree_tiny()]
    return W.make_custom_inputs(parents, [33, 0, 70, 15], Hq=4, Hkv=2, d=128 if dtype == "bf16" else 64,
                                dtype=dtype, seed=seed, paged=paged, nan_guard=False, plant_p=0.8)


def _cache_np(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.cpu().numpy()


def _fused(inp, mode="path", history=None, history_len=None, status=None, x=None):
    x = to_device(inp) if x is None else x
    forest = bool(getattr(inp["workload"], "forest", False))
    prep = gpu_prepare(x, forest)
    if status is not None:
        prep["status"].copy_(torch.from_numpy(status))
    paged = "k_pages" in x
    kc, vc = (x["k_pages"], x["v_pages"]) if paged else (x["k_cache"], x["v_cache"])
    kt, vt = (None, None) if mode == "inplace" else (x["k_tree"], x["v_tree"])
    r = tsd.tree_accept_commit(x["logits"], x["tokens"], prep["parent_s"], kc, vc, x["prefix_len"], kt, vt,
                               x["num_nodes"], x.get("root_key"), int(inp["Dmax"]), mode,
                               block_table=x.get("block_table"), history=history, history_len=history_len,
                               status=prep["status"])
    torch.cuda.synchronize()
    acc = {k: v.cpu().numpy() for k, v in r.items()}
    return acc, _cache_np(kc), _cache_np(vc), x["prefix_len"].cpu().numpy(), prep["status"].cpu().numpy()


def _assert_acc(got, ref):
    for k in ("accept_len", "path", "out_tokens"):
        assert np.array_equal(got[k], ref[k]), (k, got[k], ref[k])


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fused_path_matches_oracle(paged, dtype):
    inp = _case(paged, dtype)
    acc, kc, vc, pl, st = _fused(inp)
    ref = oracle.accept_greedy(inp)
    rk, rv, rpl, _ = oracle.kv_commit(inp, ref["accept_len"], ref["path"], "path")
    assert (st == 0).all()
    _assert_acc(acc, ref)
    assert np.array_equal(pl, rpl)
    assert np.array_equal(kc, rk) and np.array_equal(vc, rv)   # byte-exact, rows beyond L+A+1 included


@pytest.mark.parametrize("paged", [False, True])
def test_fused_inplace_matches_oracle(paged):
    inp = lay_tree_in_cache(_case(paged, seed=1))
    acc, kc, vc, pl, st = _fused(inp, mode="inplace")
    ref = oracle.accept_greedy(inp)
    rk, rv, rpl, _ = oracle.kv_commit(inp, ref["accept_len"], ref["path"], "inplace")
    assert (st == 0).all()
    _assert_acc(acc, ref)
    assert np.array_equal(pl, rpl) and np.array_equal(kc, rk) and np.array_equal(vc, rv)


@pytest.mark.parametrize("name", ["tree26", "eagle60", "forest"])
def test_fused_workloads(name):
    w = W.WORKLOADS[name]
    if name != "tree26":
        w = w.scaled(B=min(w.B, 4), L=min(w.L, 3000), L_lo=None if w.L_lo is None else 500)
    inp = W.make_inputs(w, nan_guard=False)
    acc, kc, vc, pl, st = _fused(inp)
    ref = oracle.accept_greedy(inp)
    rk, rv, rpl, _ = oracle.kv_commit(inp, ref["accept_len"], ref["path"], "path")
    assert (st == 0).all()
    _assert_acc(acc, ref)
    assert np.array_equal(pl, rpl) and np.array_equal(kc, rk) and np.array_equal(vc, rv)
    if name == "forest":   # misses commit nothing and leave prefix_len as it was
        miss = ref["accept_len"] < 0
        assert np.array_equal(pl[miss], inp["prefix_len"][miss])


def test_fused_history_splice_and_errors():
    inp = _case(False, seed=2)
    ref = oracle.accept_greedy(inp)
    B = inp["parent"].shape[0]
    cap = 16
    hist0 = np.arange(B * cap, dtype=np.int32).reshape(B, cap) + 1000
    A = ref["accept_len"]
    hl0 = np.array([0, 5, 3, cap - A[3]], np.int32)   # sequence 3: one history slot short
    pl0 = inp["prefix_len"].copy()
    status = np.array([0, 0, 0, 0], np.int32)
    hist = torch.from_numpy(hist0.copy()).cuda()
    hl = torch.from_numpy(hl0.copy()).cuda()
    acc, kc, vc, pl, st = _fused(inp, history=hist, history_len=hl, status=status)
    _assert_acc(acc, ref)
    h, hlen = hist.cpu().numpy(), hl.cpu().numpy()
    for b in range(B):
        if b == 3:
            assert st[b] == 6 and hlen[b] == hl0[b] and np.array_equal(h[b], hist0[b]) and pl[b] == pl0[b]
            continue
        assert st[b] == 0
        a = int(A[b])
        assert hlen[b] == hl0[b] + a + 1
        assert np.array_equal(h[b, hl0[b]:hl0[b] + a + 1], ref["out_tokens"][b, :a + 1])
        keep = np.ones(cap, bool)
        keep[hl0[b]:hl0[b] + a + 1] = False
        assert np.array_equal(h[b][keep], hist0[b][keep])
    # the refused sequence's cache rows are untouched; the others are committed
    rk, rv, rpl, _ = oracle.kv_commit(inp, np.where(np.arange(B) == 3, -1, A), ref["path"], "path")
    assert np.array_equal(pl, rpl) and np.array_equal(kc, rk) and np.array_equal(vc, rv)


def test_fused_flagged_sequence_is_skipped():
    inp = _case(False, seed=3)
    status = np.array([0, 5, 0, 0], np.int32)   # sequence 1 flagged before acceptance
    acc, kc, vc, pl, st = _fused(inp, status=status)
    assert st.tolist() == [0, 5, 0, 0]
    ref = oracle.accept_greedy(inp)
    assert acc["accept_len"][1] == -1 and (acc["out_tokens"][1] == -1).all()
    A = ref["accept_len"].copy()
    A[1] = -1
    rk, rv, rpl, _ = oracle.kv_commit(inp, A, ref["path"], "path")
    assert np.array_equal(pl, rpl) and np.array_equal(kc, rk)


@pytest.mark.parametrize("paged,schedule,graph", [(False, "fused", False), (True, "fused", False),
                                                  (False, "overlap", False), (True, "overlap", True),
                                                  (False, "fused", True)])
def test_device_resident_loop(paged, schedule, graph):
    """Three verify steps back to back with nothing read back in between: each step's commit
    advances prefix_len on the device and the next step's attention reads the grown cache.
    Every step is checked against the oracle applied to the cache the previous step left.  With
    graph=True the three steps are captured into one CUDA graph and replayed once."""
    parents = [W.tree_static_scored((4, 3, 2, 1, 1, 1), 26), W.tree_chain(4)]
    inp = W.make_custom_inputs(parents, [40, 75], Hq=8, Hkv=2, d=128, dtype="bf16", seed=5, paged=paged,
                               nan_guard=False, plant_p=0.9)
    x = to_device(inp)
    fused = schedule == "fused"
    step = VerifyStep.for_inputs(x, schedule=schedule, history_cap=64 if fused else 0)
    outs = [{"out": torch.empty_like(step.out), "accept_len": torch.empty_like(step.accept_len),
             "out_tokens": torch.empty_like(step.out_tokens)} for _ in range(3)]

    def three_steps():
        for o in outs:
            res = step.run(x)
            for k in o:
                o[k].copy_(res[k])

    if graph:
        s = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            three_steps()
        g.replay()
    else:
        three_steps()
    torch.cuda.synchronize()
    assert (step.status.cpu().numpy() == 0).all()
    cur = dict(inp)
    hist = [[] for _ in range(2)]
    key, vkey = ("k_pages", "v_pages") if paged else ("k_cache", "v_cache")
    for o in outs:
        rows = sample_rows(cur, 48, seed=1)
        ro, _, rows = oracle.attention_rows(cur, rows)
        got = to_np(o["out"]).astype(np.float64)
        gv = np.stack([got[b, i, h] for b, i, h in rows])
        assert np.max(np.abs(gv - ro)) < 2e-2
        ref = oracle.accept_greedy(cur)
        assert np.array_equal(o["accept_len"].cpu().numpy(), ref["accept_len"])
        assert np.array_equal(o["out_tokens"].cpu().numpy(), ref["out_tokens"])
        rk, rv, rpl, _ = oracle.kv_commit(cur, ref["accept_len"], ref["path"], "path")
        for b in range(2):
            hist[b] += ref["out_tokens"][b, :ref["accept_len"][b] + 1].tolist()
        cur = dict(cur)
        cur[key], cur[vkey], cur["prefix_len"] = rk, rv, rpl
    assert np.array_equal(x["prefix_len"].cpu().numpy(), cur["prefix_len"])
    assert np.array_equal(_cache_np(x[key]), cur[key]) and np.array_equal(_cache_np(x[vkey]), cur[vkey])
    if fused:
        hl = step.history_len.cpu().numpy()
        h = step.history.cpu().numpy()
        for b in range(2):
            assert hl[b] == len(hist[b]) and h[b, :hl[b]].tolist() == hist[b]
