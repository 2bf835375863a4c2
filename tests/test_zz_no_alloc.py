"""tsd_tree_accept_greedy_noalloc: greedy acceptance for callers that may not allocate device
memory (for example a serving engine that gave every free byte to its KV-cache pool at start-up,
or a plug-in handed device pointers but no allocator).  The call uses the library's own fixed
scratch array instead of a caller workspace.  Its results must equal those of
tsd_tree_accept_greedy, bit for bit, on consecutive calls (the shared array keeps the previous
call's contents, which must not leak into the next one).  Collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import tree_speculative_decoding_06_b200 as tsd
import workloads as W
from tree_speculative_decoding_06_b200.step import to_device

pytestmark = pytest.mark.gpu


def _both(inp):
    x = to_device(inp)
    forest = bool(getattr(inp["workload"], "forest", False))
    prep = tsd.tree_prepare(x["parent"], x["num_nodes"], int(x["Dmax"]), forest)
    ref = tsd.tree_accept_greedy(x["logits"], x["tokens"], prep["parent_s"], x["num_nodes"], x.get("root_key"),
                                 int(x["Dmax"]), status=prep["status"].clone())
    got = tsd.tree_accept_greedy_noalloc(x["logits"], x["tokens"], prep["parent_s"], x["num_nodes"],
                                         x.get("root_key"), int(x["Dmax"]), status=prep["status"].clone())
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in ref.items()}, {k: v.cpu().numpy() for k, v in got.items()}


def test_noalloc_equals_workspace_call_on_consecutive_calls():
    cases = [W.make_inputs(W.WORKLOADS["forest"].scaled(L=8, V=128256)),     # 4096 rows: 512 KiB of scratch
             W.make_inputs(W.WORKLOADS["tree26"].scaled(L=8, V=50000)),      # then a smaller, different batch
             W.make_inputs(W.WORKLOADS["tiny"])]
    for inp in cases:
        ref, got = _both(inp)
        for k in ("accept_len", "path", "out_tokens"):
            assert np.array_equal(ref[k], got[k]), k


def test_noalloc_refuses_batches_beyond_its_scratch():
    B, Nmax, V = 16, 600, 128256           # 16*600 rows x 16 chunks x 8 B > 1 MiB
    assert tsd.tree_accept_greedy_workspace_size(B, Nmax, V) > tsd.accept_noalloc_scratch_bytes()
    logits = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    i32 = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(i32.data_ptr())
    rc = tsd.lib().tsd_tree_accept_greedy_noalloc(ctypes.c_void_p(logits.data_ptr()), 1, V, p, p, None, None, B, Nmax,
                                                  8, p, p, p, p, None)
    assert tsd.status_str(rc) == "TSD_ERR_WORKSPACE"
