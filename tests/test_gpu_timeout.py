"""The tcgen05 attention's bounded waits: when a key tile never arrives, every wait on it gives up
after its cycle limit and the call reports TSD_ERR_TIMEOUT in status[] with the affected rows
zeroed, instead of stalling; the context stays usable and the next call is correct.

The missing tile is made on the host side of the kernel (a test hook in the launch,
TSD_TEST_WITHHOLD_TILE, makes the K producer skip that tile and shortens the limit to 10^5
cycles); nothing faults, traps or spins without a bound."""
import os

import numpy as np
import pytest
import torch

import tree_speculative_decoding_06_b200 as tsd
import workloads as W
from gpu_helpers import check_attention, forced_split_workspace, gpu_attention

pytestmark = pytest.mark.gpu

TIMEOUT = 7


@pytest.mark.parametrize("name,scale", [("tree26", dict(L=600, V=64)),               # several key splits
                                         ("chain5", dict(B=48, L=900, V=64)),        # more row blocks
                                         ("eagle60", dict(B=3, L=700, L_lo=300, V=64))])   # paged, two query tiles
def test_withheld_tile_times_out_and_the_next_call_is_correct(name, scale):
    inp = W.make_inputs(W.WORKLOADS[name].scaled(**scale), nan_guard=False)
    os.environ["TSD_TEST_WITHHOLD_TILE"] = "1"
    os.environ["TSD_ATTN_SPLITS"] = "2"     # the in-kernel split merge on the time-out path too
    os.environ["TSD_ATTN_MERGE"] = "fused"
    ws = forced_split_workspace(inp)
    try:
        out, lse, st = gpu_attention(inp, workspace=ws)
    finally:
        del os.environ["TSD_TEST_WITHHOLD_TILE"]
        del os.environ["TSD_ATTN_SPLITS"]
        del os.environ["TSD_ATTN_MERGE"]
    assert ((st & 0xFF) == TIMEOUT).all(), st
    # every CTA took its ticket on the way out: the merge words are zero for the next call
    assert int(ws[:tsd.tree_verify_attn_ticket_bytes()].view(torch.int32).abs().sum()) == 0
    for b in range(inp["q"].shape[0]):
        n = int(inp["num_nodes"][b])
        assert (out[b, :n] == 0).all() and (lse[b, :n] == 0).all()
    # the same call again, without the hook, on the same device and stream: clean and correct
    out, lse, st = gpu_attention(inp)
    assert (st == 0).all()
    check_attention(inp, out, lse, rows=None if name != "chain5" else
                    [(b, i, h) for b in range(0, 48, 7) for i in range(6) for h in range(64)])
    torch.cuda.synchronize()
