"""GPU parity of threshold acceptance (tsd_tree_accept_threshold) against the fp64 oracle in
oracle/tree_threshold.py: bit-exact on every sequence whose edge tests clear the margin
|p - tau| / tau >= 1e-5 (the kernel's probabilities carry ~1e-7 relative error from fp32
exponentials), a valid path otherwise."""
import numpy as np
import pytest
import torch

import tree_speculative_decoding_06_b200 as tsd
import workloads as W
from gpu_helpers import gpu_prepare
from oracle import tree_threshold as tt
from tree_speculative_decoding_06_b200.step import to_device

pytestmark = pytest.mark.gpu

MARGIN = 1e-5


def run(inp, tau, T):
    x = to_device(inp)
    forest = bool(getattr(inp["workload"], "forest", False))
    prep = gpu_prepare(x, forest)
    r = tsd.tree_accept_threshold(x["logits"], x["tokens"], prep["parent_s"], tau, T, num_nodes=x["num_nodes"],
                                  root_key=x.get("root_key"), Dmax=int(x["Dmax"]), status=prep["status"])
    torch.cuda.synchronize()
    got = {k: v.cpu().numpy() for k, v in r.items()}
    dt = "bf16" if inp["logits"].dtype == np.uint16 else "f32"
    ref = tt.accept_threshold_batch(inp["logits"], inp["tokens"], inp["parent"], inp["num_nodes"], tau, T,
                                    int(inp["Dmax"]), lambda row: W.as_f32(row, dt).astype(np.float64),
                                    inp.get("root_key"))
    return got, ref


def compare(got, ref, inp):
    near = 0
    for b in range(inp["parent"].shape[0]):
        if all(m >= MARGIN for m in ref["margins"][b]):
            assert got["accept_len"][b] == ref["accept_len"][b], b
            assert np.array_equal(got["path"][b], ref["path"][b]), b
            assert np.array_equal(got["out_tokens"][b], ref["out_tokens"][b]), b
        else:
            near += 1
            A = int(got["accept_len"][b])
            for j in range(1, A + 1):
                assert inp["parent"][b, got["path"][b, j] - 1] == got["path"][b, j - 1] - 1
    return near


@pytest.mark.parametrize("name", ["tree26", "eagle60", "forest"])
@pytest.mark.parametrize("tau", [0.0, 1e-4, 0.01, 0.3, 0.6])
def test_threshold_full_size(name, tau):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w.scaled(L=16, L_lo=None if w.L_lo is None else 8), nan_guard=False)
    got, ref = run(inp, tau, 1.0)
    assert compare(got, ref, inp) <= 1
    if tau == 0.0 and name != "forest":   # every node accepted: the deepest (lowest index) node
        depth = [W.tree_depths(inp["parent"][b, :int(inp["num_nodes"][b])]) for b in range(inp["parent"].shape[0])]
        assert got["accept_len"].tolist() == [int(d.max()) for d in depth]


@pytest.mark.parametrize("V,dt,T", [(1001, "bf16", 1.0), (4096, "f32", 0.5), (50, "f32", 2.0)])
def test_threshold_small_vocabularies(V, dt, T):
    rng = np.random.default_rng(V)
    parents = [W.tree_static_scored((4, 3, 2, 1, 1, 1), 26), W.tree_tiny(), W.tree_chain(7)] * 4
    parents += [np.array([-1] + [int(rng.integers(0, i)) for i in range(1, n)], np.int32)
                for n in rng.integers(2, 30, size=12)]
    inp = W.make_custom_inputs(parents, [1] * len(parents), Hq=2, Hkv=1, d=16, dtype=dt, V=V, seed=V,
                               plant_p=0.8, logit_sigma=1.0)
    for tau in (0.002, 0.02, 0.2):
        got, ref = run(inp, tau, T)
        assert compare(got, ref, inp) <= 2
