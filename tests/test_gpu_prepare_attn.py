"""GPU parity: tree_prepare (bit-exact) and tree_verify_attn (stated tolerance) against the oracle,
called through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import tree_speculative_decoding_06_b200 as tsd
import workloads as W
from gpu_helpers import check_attention, forced_split_workspace, gpu_attention, lay_tree_in_cache, sample_rows
from test_oracle_structure import all_trees

pytestmark = pytest.mark.gpu

CODE = {"ok": 0, "bad_parent": 3, "too_deep": 4, "extra_root": 5}


def test_prepare_matches_oracle():
    rng = np.random.default_rng(0)
    trees = []
    for n in range(1, 6):
        trees += [(t, False) for t in all_trees(n)]
    trees += [(t, True) for t in all_trees(4, True)]
    for _ in range(60):
        n = int(rng.integers(1, 40))
        forest = bool(rng.random() < 0.3)
        p = [-1] + [int(rng.integers(-1 if forest else 0, i)) for i in range(1, n)]
        if rng.random() < 0.3:                       # corrupt one entry
            k = int(rng.integers(0, n))
            p[k] = int(rng.integers(-3, n + 2))
        trees.append((np.array(p, np.int32), forest))
    trees += [(W.tree_static_scored((4, 3, 2, 1, 1, 1), 26), False), (W.tree_forest(8, 64), True),
              (W.tree_forest(8, 64), False), (W.tree_chain(12), False)]
    for forest in (False, True):
        group = [t for t, f in trees if f == forest]
        B = len(group)
        Nmax = max(len(t) for t in group)
        Dmax = 6
        parent = np.full((B, Nmax), -1, np.int32)
        nn = np.array([len(t) for t in group], np.int32)
        for b, t in enumerate(group):
            parent[b, :len(t)] = t
        res = tsd.tree_prepare(torch.from_numpy(parent).cuda(), torch.from_numpy(nn).cuda(), Dmax, forest,
                               want_bits=True)
        torch.cuda.synchronize()
        st = res["status"].cpu().numpy()
        ps, ds, anc = (res[k].cpu().numpy() for k in ("parent_s", "depth", "anc"))
        bits = res["anc_bits"].cpu().numpy().view(np.uint32)
        for b, t in enumerate(group):
            o = oracle.tree_structure(t, Dmax, forest)
            assert st[b] & 0xFF == CODE[o["code"]], (t, o["code"], st[b])
            if o["code"] != "ok":
                assert st[b] >> 8 == o["bad_node"]
                assert (ps[b] == 0).all() and (anc[b] == 0).all()
                continue
            n = len(t)
            assert (ps[b, :n + 1] == o["parent_s"]).all() and (ps[b, n + 1:] == 0).all()
            assert (ds[b, :n + 1] == o["depth"]).all()
            assert (anc[b, :n + 1] == o["anc"]).all() and (anc[b, n + 1:] == 0).all()
            for i in range(n):                        # bits of slot i+1 = ancestors (as slots) from M
                want = np.zeros(bits.shape[2] * 32, bool)
                want[np.nonzero(o["M"][i])[0] + 1] = True
                got = np.unpackbits(bits[b, i + 1].view(np.uint8), bitorder="little").astype(bool)
                assert (got == want).all()


def test_prepare_rejects_bad_num_nodes():
    parent = torch.full((2, 4), -1, dtype=torch.int32, device="cuda")
    parent[:, 1:] = 0
    nn = torch.tensor([5, 4], dtype=torch.int32, device="cuda")
    res = tsd.tree_prepare(parent, nn, 3, False)
    assert res["status"].cpu().tolist() == [1, 0]


SMALL = {
    "tiny": W.WORKLOADS["tiny"],
    "tree26": W.WORKLOADS["tree26"].scaled(L=300, V=512),
    "eagle60": W.WORKLOADS["eagle60"].scaled(B=3, L=700, L_lo=0, V=3000),
    "chain5": W.WORKLOADS["chain5"].scaled(B=3, L=257, V=700),
    "forest": W.WORKLOADS["forest"].scaled(B=2, L=130, V=600),
}


def _use_path(monkeypatch, param):
    for k in ("TSD_ATTN_PATH", "TSD_ATTN_SPLITS", "TSD_ATTN_MERGE"):
        monkeypatch.delenv(k, raising=False)
    if param == "mma":
        monkeypatch.setenv("TSD_ATTN_PATH", "mma")
    if param.startswith("split3"):
        monkeypatch.setenv("TSD_ATTN_SPLITS", "3")
    if param.endswith("kernel"):
        monkeypatch.setenv("TSD_ATTN_MERGE", "kernel")
    elif param.startswith("split3") or param == "fused":
        monkeypatch.setenv("TSD_ATTN_MERGE", "fused")
    return param


@pytest.fixture(params=["auto", "mma", "split3", "split3_merge_kernel"])
def attn_path(request, monkeypatch):
    """Run a test on the default kernel choice (tcgen05 where it applies), with the warp-level
    mma.sync kernel forced, and with the tcgen05 kernel's keys split three ways, merged in the
    kernel by the last CTA of each query block (forced for every shape) and by the separate merge
    kernel, so every bf16 kernel and both merges stay covered."""
    return _use_path(monkeypatch, request.param)


@pytest.fixture(params=["auto", "mma", "merge_kernel", "fused"])
def attn_path_full(request, monkeypatch):
    """Full-size shapes at the planner's split counts (every bench shape splits its keys): the
    default merge choice, the separate merge kernel and the in-kernel merge forced for every shape,
    and the mma.sync kernel."""
    return _use_path(monkeypatch, request.param)


@pytest.mark.parametrize("name", list(SMALL))
def test_attention_small(name, attn_path):
    inp = W.make_inputs(SMALL[name])
    out, lse, st = gpu_attention(inp)
    assert (st == 0).all()
    check_attention(inp, out, lse)


@pytest.mark.parametrize("name", ["tree26", "eagle60"])
def test_attention_tree_in_cache(name):
    inp = lay_tree_in_cache(W.make_inputs(SMALL[name]))
    out, lse, st = gpu_attention(inp, tree_in_cache=True)
    assert (st == 0).all()
    check_attention(inp, out, lse, tree_in_cache=True)


@pytest.mark.parametrize("dtype,d,Hq,Hkv,paged", [
    ("bf16", 64, 6, 2, False), ("bf16", 128, 5, 5, True), ("f32", 128, 12, 4, True), ("f32", 64, 3, 1, False),
    ("bf16", 64, 48, 1, False), ("bf16", 128, 8, 8, True), ("bf16", 128, 64, 1, False), ("bf16", 128, 16, 2, True),
])
def test_attention_shapes_and_ragged(dtype, d, Hq, Hkv, paged, attn_path):
    # ragged batch: empty prefix, a prefix that ends mid-tile, a long one; trees of different sizes
    parents = [W.tree_chain(1), W.tree_static_scored((4, 3, 2, 1, 1, 1), 26), W.tree_tiny(), W.tree_chain(70)]
    inp = W.make_custom_inputs(parents, [0, 63, 200, 129], Hq=Hq, Hkv=Hkv, d=d, dtype=dtype, seed=7, paged=paged,
                               Dmax=69)
    out, lse, st = gpu_attention(inp)
    assert (st == 0).all()
    check_attention(inp, out, lse)


def test_attention_idle_sequence_and_flagged_tree():
    parents = [W.tree_tiny(), [], np.array([-1, 0, 5, 1], np.int32)]   # N=0 slot; a malformed tree
    inp = W.make_custom_inputs([parents[0], parents[0][:0], parents[0][:4]], [40, 10, 20], Hq=4, Hkv=2, d=64,
                               dtype="bf16", seed=3)
    inp["parent"][2, :4] = parents[2]
    x_out, _, st = gpu_attention(inp)
    assert st[0] == 0 and st[1] == 0 and (st[2] & 0xFF) == 3 and (st[2] >> 8) == 2
    assert (x_out[2, :4] == 0).all()
    inp2 = dict(inp)
    inp2["num_nodes"] = np.array([8, 0, 0], np.int32)
    check_attention(inp2, x_out, None, rows=[(0, i, h) for i in range(8) for h in range(4)])


def test_attention_capacity_flag():
    inp = W.make_custom_inputs([W.tree_tiny(), W.tree_tiny()], [30, 40], Hq=4, Hkv=2, d=64, dtype="bf16", seed=5)
    inp["prefix_len"] = inp["prefix_len"].copy()
    inp["prefix_len"][1] = inp["k_cache"].shape[2] + 1          # past the cache capacity
    out, _, st = gpu_attention(inp)
    assert st[0] == 0 and st[1] == 6
    assert (out[1] == 0).all()


@pytest.mark.parametrize("Hq", [8, 16])   # 104 query rows per KV head (one tile), 208 (two tiles)
def test_no_cross_branch_leakage_gpu(Hq):
    parent = W.tree_static_scored((4, 3, 2, 1, 1, 1), 26)
    inp = W.make_custom_inputs([parent], [150], Hq=Hq, Hkv=2, d=128, dtype="bf16", seed=11)
    out0, _, _ = gpu_attention(inp)
    M = oracle.tree_structure(parent, 6)["M"]
    rng = np.random.default_rng(1)
    for i in (3, 17, 25):
        pert = dict(inp)
        for key in ("k_tree", "v_tree"):
            pert[key] = inp[key].copy()
            others = np.nonzero(M[i] == 0)[0]
            pert[key][0, others] = W.f32_to_bf16_bits(rng.standard_normal(pert[key][0, others].shape) * 4)
        out1, _, _ = gpu_attention(pert)
        assert np.array_equal(out0[0, i], out1[0, i])


FULL = ["tree26", "eagle60", "chain5", "forest"]


@pytest.mark.parametrize("name", FULL)
def test_attention_full_size_sampled(name, attn_path_full):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w)
    out, lse, st = gpu_attention(inp)
    assert (st == 0).all()
    rows = sample_rows(inp, 48 if name != "forest" else 24, seed=1)
    check_attention(inp, out, lse, rows=rows)
    # properties at every row: finite, bounded by the largest |V| of the sequence's keys
    assert np.isfinite(out).all()


def _ticket_words(ws):
    return ws[:tsd.tree_verify_attn_ticket_bytes()].view(torch.int32)


@pytest.mark.parametrize("name", ["tree26", "eagle60"])
def test_merge_tickets_return_to_zero_and_garbage_is_reported(name, monkeypatch):
    """The in-kernel split merge counts the CTAs of each query block on ticket words at the start of
    the workspace: after a call they are all zero again, so back-to-back calls on one workspace
    stay correct; a workspace whose ticket words were never zeroed is reported as
    TSD_ERR_WORKSPACE in status[] (nothing is read or written out of place)."""
    monkeypatch.setenv("TSD_ATTN_SPLITS", "3")
    monkeypatch.setenv("TSD_ATTN_MERGE", "fused")
    inp = W.make_inputs(SMALL[name])
    ws = forced_split_workspace(inp)
    for _ in range(3):
        out, lse, st = gpu_attention(inp, workspace=ws)
        assert (st == 0).all()
        assert int(_ticket_words(ws).abs().sum()) == 0
    check_attention(inp, out, lse)
    ws[:tsd.tree_verify_attn_ticket_bytes()].fill_(0x7F)     # count 0x7f7f7f7f: no call leaves that
    _, _, st = gpu_attention(inp, workspace=ws)
    assert ((st & 0xFF) == 9).all(), st
    ws.zero_()
    out, lse, st = gpu_attention(inp, workspace=ws)
    assert (st == 0).all()
    check_attention(inp, out, lse)


@pytest.mark.parametrize("paged", [False, True])
def test_merge_in_kernel_with_flagged_sequences(paged, monkeypatch):
    """The in-kernel split merge on the sequences a call must zero: one whose tree prepare flags on
    entry (a malformed parent) and one past the cache capacity.  Every CTA of such a row block
    leaves early but still takes its ticket, the last one zeroes the rows, the ticket words return
    to zero, and the other sequences are exact (two query tiles per CTA: 26 nodes x 8 heads)."""
    monkeypatch.setenv("TSD_ATTN_SPLITS", "3")
    monkeypatch.setenv("TSD_ATTN_MERGE", "fused")
    tree = W.tree_static_scored((4, 3, 2, 1, 1, 1), 26)
    inp = W.make_custom_inputs([tree] * 4, [300, 500, 200, 420], Hq=32, Hkv=4, d=128, dtype="bf16", seed=9,
                               paged=paged)
    inp["parent"] = inp["parent"].copy()
    inp["parent"][1, 5] = 9                               # a forward parent: prepare flags sequence 1
    inp["prefix_len"] = inp["prefix_len"].copy()
    inp["prefix_len"][2] = inp["Lmax"] + 1                # past the capacity: the attention flags sequence 2
    ws = forced_split_workspace(inp)
    for _ in range(2):
        out, lse, st = gpu_attention(inp, workspace=ws)
        assert st[0] == 0 and st[3] == 0 and (st[1] & 0xFF) == 3 and (st[2] & 0xFF) == 6, st
        assert (out[1] == 0).all() and (out[2] == 0).all()
        assert int(_ticket_words(ws).abs().sum()) == 0
    check_attention(inp, out, lse, rows=[(b, i, h) for b in (0, 3) for i in range(26) for h in range(0, 32, 5)])
