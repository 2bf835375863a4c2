"""The C-ABI library: it loads without a GPU, exports every entry point include/tsd.h
declares, and its host-side argument checks answer without touching the device."""
import ctypes
import os
import re

import pytest

import tree_speculative_decoding_06_b200 as tsd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "tsd.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tsd_[a-z_0-9]+)\s*\(", src)) - {"tsd_status"})


def test_library_exports_every_declared_symbol():
    lib = tsd.lib()
    names = declared_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(tsd._SIGS), "binding signatures and header disagree"


def test_status_strings_and_version():
    assert tsd.lib().tsd_abi_version() == 2
    for code, name in tsd.STATUS.items():
        assert tsd.status_str(code) == name
    assert tsd.status_str(3 | (17 << 8)) == "TSD_ERR_BAD_TREE"


def test_host_argument_checks():
    L = tsd.lib()
    assert L.tsd_tree_prepare(None, None, -1, 4, 3, 0, None, None, None, None, None, None) == 1
    assert L.tsd_tree_prepare(None, None, 0, 4, 3, 0, None, None, None, None, None, None) == 0   # empty batch
    assert L.tsd_tree_prepare(None, None, 1, 4, 300, 0, None, None, None, None, None, None) == 1  # Dmax > 255
    # attention: d not in {64,128}, Hq % Hkv, bad dtype, missing workspace
    args = dict(q=None, kc=None, vc=None, Lmax=16, pl=None, kt=None, vt=None, ps=None, nn=None)
    assert L.tsd_tree_verify_attn(None, None, None, 16, None, None, None, None, None, 1, 4, 8, 2, 96, 3, 1, 1.0,
                                  None, None, None, 0, None, None) == 1
    assert L.tsd_tree_verify_attn(None, None, None, 16, None, None, None, None, None, 1, 4, 8, 3, 64, 3, 1, 1.0,
                                  None, None, None, 0, None, None) == 1
    assert L.tsd_tree_verify_attn(None, None, None, 16, None, None, None, None, None, 1, 4, 8, 2, 64, 3, 7, 1.0,
                                  None, None, None, 0, None, None) == 2
    assert L.tsd_tree_verify_attn(None, None, None, 16, None, None, None, None, None, 0, 4, 8, 2, 64, 3, 1, 1.0,
                                  None, None, None, 0, None, None) == 0
    assert L.tsd_tree_verify_attn_paged(None, None, None, 4, 12, None, 2, None, None, None, None, None, 1, 4, 8, 2,
                                        64, 3, 1, 1.0, None, None, None, 0, None, None) == 1   # block 12
    assert L.tsd_chain_accept_sample(None, None, 1, 16, None, None, -1.0, 1, 3, None, None, None, 0, None) == 1
    assert L.tsd_kv_commit(None, None, 16, None, None, None, None, None, None, 1, 4, 2, 64, 3, 1, 9, None, None) == 1
    # a non-null but too small workspace is refused before any launch
    buf = ctypes.create_string_buffer(8)
    p = ctypes.cast(buf, ctypes.c_void_p)
    ws = tsd.tree_verify_attn_workspace_size(1, 26, 32, 8, 128, 2112, 1)
    assert ws > 8
    assert L.tsd_tree_verify_attn(p, p, p, 2112, p, p, p, p, None, 1, 26, 32, 8, 128, 6, 1, 0.1, p, None, p, 8, p,
                                  None) == 9


def test_workspace_sizes_are_consistent():
    # the paged query plans for ragged lengths (more splits), so it never asks for less than the
    # contiguous one at the same capacity; both cover the partials of every split the plan makes
    a = tsd.tree_verify_attn_workspace_size(16, 60, 32, 8, 128, 8320, 1)
    b = tsd.tree_verify_attn_paged_workspace_size(16, 60, 32, 8, 128, 520, 16, 1)
    tk = tsd.tree_verify_attn_ticket_bytes()
    assert tk >= 4 * 16 * 8 and tk % 256 == 0        # one ticket word per (sequence, KV head, row block)
    assert b >= a and (b - tk) % (16 * 8 * 240 * 130 * 4) == 0
    assert tsd.tree_accept_greedy_workspace_size(8, 512, 128256) == 8 * 512 * 16 * 8
    assert tsd.chain_accept_sample_workspace_size(64, 5, 128256) > 64 * 11 * 16 * 8


def test_host_checks_of_the_fused_and_draft_tree_entry_points():
    L = tsd.lib()
    cache = tsd.KVCacheDesc(None, None, None, 16, None, 0, 0, 0)
    # fused acceptance + commit: a null cache struct, an empty batch, a missing pointer
    assert L.tsd_tree_accept_commit(None, 1, 16, None, None, None, None, 1, 4, 3, None, None, None, 2, 64, 1, 0,
                                    None, 0, None, None, None, None, None, 0, None, None) == 1
    assert L.tsd_tree_accept_commit(None, 1, 16, None, None, None, None, 0, 4, 3, ctypes.byref(cache), None, None, 2,
                                    64, 1, 0, None, 0, None, None, None, None, None, 0, None, None) == 0
    assert L.tsd_tree_accept_commit(None, 1, 16, None, None, None, None, 1, 4, 3, ctypes.byref(cache), None, None, 2,
                                    64, 1, 0, None, 0, None, None, None, None, None, 0, None, None) == 1
    assert L.tsd_tree_accept_commit(None, 7, 16, None, None, None, None, 1, 4, 3, ctypes.byref(cache), None, None, 2,
                                    64, 1, 0, None, 0, None, None, None, None, None, 0, None, None) == 2
    # draft tree: frontier width and K limits, K above V, empty batches, workspace
    d = tsd.DraftTreeDesc(None, None, None, None, None, None, None, 64, 4)
    assert L.tsd_draft_tree_init(ctypes.byref(d), None, 0, None, None) == 0
    assert L.tsd_draft_tree_init(ctypes.byref(d), None, 1, None, None) == 1          # null arrays
    wide = tsd.DraftTreeDesc(None, None, None, None, None, None, None, 64, 17)
    assert L.tsd_draft_tree_init(ctypes.byref(wide), None, 0, None, None) == 1       # F > 16
    assert L.tsd_draft_tree_expand(ctypes.byref(d), None, 1, 100, 17, 0, None, 0, None, None) == 1   # K > 16
    assert L.tsd_draft_tree_expand(ctypes.byref(d), None, 1, 8, 10, 0, None, 0, None, None) == 1     # K > V
    assert L.tsd_draft_tree_expand(ctypes.byref(d), None, 9, 100, 4, 0, None, 0, None, None) == 2    # dtype
    assert L.tsd_draft_tree_finalize(ctypes.byref(d), 0, 0, None, None, None, None, None) == 1        # keep 0
    big = tsd.DraftTreeDesc(None, None, None, None, None, None, None, 5000, 4)
    assert L.tsd_draft_tree_finalize(ctypes.byref(big), 0, 8, None, None, None, None, None) == 1      # > 4096 nodes
    # one record of (2 x 4 + 16) bytes rounded to 16, per (sequence, row, 16384-token chunk)
    assert tsd.lib().tsd_draft_tree_expand_workspace_size(2, 10, 10, 128256) == 2 * 10 * 8 * 96


def test_split_planner_choices_for_the_bench_workloads():
    """The planner's split counts (read back through the workspace size: splits * rows * (d + 2)
    fp32 per KV head and sequence) for the four bench shapes on a 148-SM device: tree26 9 (a sweep
    of 3..17 on B200 found 9 fastest), eagle60 2 (paged: planned for ragged lengths, each split an
    equal share of its own sequence, longest sequences first; a B200 sweep of 2..8 found 2 fastest
    with the splits merged in the kernel), chain5 2, forest 2 (a sweep of 1..4: 2)."""
    def splits(ws, B, Hkv, R, d=128):   # the ticket words come first, then the partials
        return (ws - tsd.tree_verify_attn_ticket_bytes()) // (B * Hkv * R * (d + 2) * 4) if ws else 1
    assert splits(tsd.tree_verify_attn_workspace_size(1, 26, 32, 8, 128, 2112, 1), 1, 8, 104) == 9
    assert splits(tsd.tree_verify_attn_paged_workspace_size(16, 60, 32, 8, 128, 520, 16, 1), 16, 8, 240) == 2
    assert splits(tsd.tree_verify_attn_workspace_size(64, 6, 64, 8, 128, 8256, 1), 64, 8, 48) == 2
    assert splits(tsd.tree_verify_attn_paged_workspace_size(8, 512, 32, 8, 128, 2080, 16, 1), 8, 8, 2048) == 2


def test_misaligned_tensor_pointers_are_refused_before_any_launch():
    """Every pointer the kernels move in 16-byte pieces must be 16-byte aligned; a view at an odd
    storage offset is refused with a status code on the host instead of reaching a kernel."""
    L = tsd.lib()
    buf = ctypes.create_string_buffer(1 << 16)
    base = (ctypes.addressof(buf) + 255) & ~255
    p, odd = ctypes.c_void_p(base), ctypes.c_void_p(base + 4)
    ws = tsd.tree_verify_attn_workspace_size(1, 26, 32, 8, 128, 2112, 1)
    # attention: Q, a cache or the output off a 16-byte boundary -> INVALID_ARG; workspace -> WORKSPACE
    for i in (0, 1, 2, 5, 6, 17):
        a = [p] * 23
        a[i] = odd
        rc = L.tsd_tree_verify_attn(a[0], a[1], a[2], 2112, p, a[5], a[6], p, None, 1, 26, 32, 8, 128, 6, 1, 0.1,
                                    a[17], None, p, ws, p, None)
        assert rc == 1, i
    assert L.tsd_tree_verify_attn(p, p, p, 2112, p, p, p, p, None, 1, 26, 32, 8, 128, 6, 1, 0.1, p, None, odd, ws,
                                  p, None) == 9
    # commit: cache or tree rows off a 16-byte boundary
    assert L.tsd_kv_commit(odd, p, 16, p, p, p, p, p, None, 1, 4, 2, 64, 3, 1, 0, p, None) == 1
    assert L.tsd_kv_commit(p, p, 16, p, odd, p, p, p, None, 1, 4, 2, 64, 3, 1, 0, p, None) == 1
    # acceptance workspace
    need = tsd.tree_accept_greedy_workspace_size(1, 4, 64)
    assert L.tsd_tree_accept_greedy(p, 1, 64, p, p, None, None, 1, 4, 3, p, p, p, odd, need, p, None) == 9
    assert tsd.accept_noalloc_scratch_bytes() == 1 << 20


def test_attention_kernel_count_query(monkeypatch):
    """Kernels per attention call, as the bench counts them: the two-tile tcgen05 kernel merges its
    key splits itself (eagle60, forest: one launch), the one-tile kernel (tree26, chain5) and the
    mma.sync path are followed by the merge kernel; TSD_ATTN_MERGE forces either merge."""
    monkeypatch.delenv("TSD_ATTN_MERGE", raising=False)
    monkeypatch.delenv("TSD_ATTN_PATH", raising=False)
    q = tsd.tree_verify_attn_kernels
    assert q(1, 26, 32, 8, 128, 2112, 1) == 2                    # tree26: 9 splits, merge kernel
    assert q(16, 60, 32, 8, 128, 520 * 16, 1, 16) == 1           # eagle60 (paged): merged in the kernel
    assert q(64, 6, 64, 8, 128, 8256, 1) == 2                    # chain5
    assert q(8, 512, 32, 8, 128, 2080 * 16, 1, 16) == 1          # forest (paged)
    assert q(1, 8, 8, 2, 64, 128, 0) in (1, 2)                   # fp32 FFMA path
    assert q(16, 60, 32, 8, 128, 8320, 1, 0, True) in (1, 2)     # tree K/V in the cache: mma.sync path
    monkeypatch.setenv("TSD_ATTN_MERGE", "kernel")
    assert q(16, 60, 32, 8, 128, 520 * 16, 1, 16) == 2
    monkeypatch.setenv("TSD_ATTN_MERGE", "fused")
    assert q(1, 26, 32, 8, 128, 2112, 1) == 1
    assert q(0, 26, 32, 8, 128, 2112, 1) == 0


def test_attention_grid_query():
    """CTAs of the split kernel for the bench shapes (B x KV heads x row blocks x key splits): the
    step launches an attention grid smaller than the GPU before the acceptance, a larger one after."""
    q = tsd.tree_verify_attn_ctas
    assert q(1, 26, 32, 8, 128, 2112, 1) == 1 * 8 * 1 * 9           # tree26
    assert q(16, 60, 32, 8, 128, 520 * 16, 1, 16) == 16 * 8 * 1 * 2  # eagle60: two query tiles per CTA
    assert q(64, 6, 64, 8, 128, 8256, 1) == 64 * 8 * 1 * 2           # chain5
    assert q(8, 512, 32, 8, 128, 2080 * 16, 1, 16) == 8 * 8 * 8 * 2  # forest: 8 row blocks of 256 rows
    assert q(0, 26, 32, 8, 128, 2112, 1) == 0
