"""TEST INFRASTRUCTURE ONLY: the fp64 CPU oracle of the tree-verify step.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import this package.  The product library
(``tree_speculative_decoding_06_b200``) never imports it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain single-threaded C, fp64; see its header for the
passages each routine restates).  This module compiles it with gcc on first use, marshals
numpy arrays into it, and adds the KV commit, which is a plain row copy written here with
numpy slicing:

  commit [EAGLE-Pangu, technical summary sec. 2, branchable KV cache]: for j = 0..A the
  cache row at position L + j receives the tree row of path slot path[j] (node path[j]-1),
  for K and V and every KV head; afterwards L grows by A + 1.  LENGTH mode takes node j;
  INPLACE mode reads the source rows from cache positions L + path[j] - 1 (all sources are
  read before any row is written).  A miss (A < 0), a flagged sequence, a path entry outside
  1..N, or L + A + 1 beyond the cache capacity leaves that sequence untouched.

Parity unpinned: none.  Every routine is checked by ``tests/test_oracle_*.py`` against closed
forms, library routines on special cases, brute force or hand-worked fixtures.
"""
from __future__ import annotations

import ctypes as C
import hashlib
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = None

DT = {"f32": 0, "bf16": 1}
CODE_NAMES = {0: "ok", 1: "bad_parent", 2: "too_deep", 3: "extra_root", 4: "bad_arg"}


def build(force: bool = False) -> str:
    """Compile oracle.c into a shared object (keyed by the source hash); return its path."""
    with open(_SRC, "rb") as f:
        tag = hashlib.sha256(f.read()).hexdigest()[:16]
    so = os.path.join(_BUILD, f"liboracle_{tag}.so")
    if force or not os.path.exists(so):
        os.makedirs(_BUILD, exist_ok=True)
        tmp = so + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, so)
    return so


def lib() -> C.CDLL:
    global _LIB
    if _LIB is None:
        L = C.CDLL(build())
        P, I, Lg, D = C.c_void_p, C.c_int, C.c_long, C.c_double
        L.orc_tree_structure.argtypes = [P, I, I, I, P, P, P, P, P]
        L.orc_tree_structure.restype = I
        L.orc_attn_row.argtypes = [P, I, P, P, I, Lg, P, P, Lg, P, I, I, D, P, P]
        L.orc_attn_row.restype = None
        L.orc_argmax_row.argtypes = [P, I, Lg]
        L.orc_argmax_row.restype = Lg
        L.orc_accept_greedy.argtypes = [P, I, Lg, P, P, I, I, I, P, P, P, P]
        L.orc_accept_greedy.restype = I
        L.orc_chain_sample.argtypes = [P, P, I, Lg, I, P, P, D, P, P, P]
        L.orc_chain_sample.restype = I
        L.orc_chain_sample_many.argtypes = [I, P, P, I, Lg, I, P, P, D, P, P, P]
        L.orc_chain_sample_many.restype = I
        _LIB = L
    return _LIB


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return C.c_void_p(a.ctypes.data)


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return 1
    if a.dtype == np.float32:
        return 0
    raise TypeError(f"oracle takes float32 or bf16-bit (uint16) arrays, got {a.dtype}")


# ----------------------------------------------------------------------------- structure
def tree_structure(parent, Dmax: int, forest: bool = False) -> dict:
    parent = np.ascontiguousarray(parent, np.int32)
    N = int(parent.shape[0])
    ps = np.zeros(N + 1, np.int32)
    ds = np.zeros(N + 1, np.int32)
    anc = np.zeros((N + 1, Dmax + 1), np.int32)
    M = np.zeros((max(N, 1), max(N, 1)), np.uint8)
    bad = np.zeros(1, np.int32)
    code = lib().orc_tree_structure(_p(parent), N, Dmax, int(forest), _p(ps), _p(ds), _p(anc), _p(M), _p(bad))
    return {"code": CODE_NAMES[code], "bad_node": int(bad[0]), "parent_s": ps, "depth": ds, "anc": anc,
            "M": M[:N, :N].copy()}


# ----------------------------------------------------------------------------- attention
def _prefix_rows(inp: dict, b: int, g: int, start: int, count: int, which: str) -> np.ndarray:
    """Rows [start, start+count) of KV head g of sequence b's cache, as one contiguous array."""
    if "k_cache" in inp:
        return np.ascontiguousarray(inp[which + "_cache"][b, g, start:start + count])
    bs = inp[which + "_pages"].shape[2]
    pos = np.arange(start, start + count)
    blk = inp["block_table"][b, pos // bs]
    return np.ascontiguousarray(inp[which + "_pages"][blk, g, pos % bs])


def attention_rows(inp: dict, rows=None, tree_in_cache: bool = False, scale=None):
    """Attention outputs of the requested (b, i, h) rows (default: every valid row).

    Returns (out float64 [len(rows), d], lse float64 [len(rows)], rows)."""
    w = inp["workload"]
    parent, nn, pl = inp["parent"], inp["num_nodes"], inp["prefix_len"]
    q = inp["q"]
    B, Nmax, Hq, d = q.shape
    Hkv = inp["k_tree"].shape[2]
    G = Hq // Hkv
    dt = _dt(q)
    scale = (1.0 / np.sqrt(d)) if scale is None else float(scale)
    if rows is None:
        rows = [(b, i, h) for b in range(B) for i in range(int(nn[b])) for h in range(Hq)]
    out = np.zeros((len(rows), d), np.float64)
    lse = np.zeros(len(rows), np.float64)
    L_ = lib()
    cache = {}
    for r, (b, i, h) in enumerate(rows):
        g = h // G
        N = int(nn[b])
        L = int(pl[b])
        if (b, "M") not in cache:
            st = tree_structure(parent[b, :N], int(inp["Dmax"]), bool(getattr(w, "forest", False)))
            assert st["code"] == "ok", st
            cache[(b, "M")] = st["M"]
        if (b, g) not in cache:
            kp = _prefix_rows(inp, b, g, 0, L, "k")
            vp = _prefix_rows(inp, b, g, 0, L, "v")
            if tree_in_cache:
                kt = _prefix_rows(inp, b, g, L, N, "k")
                vt = _prefix_rows(inp, b, g, L, N, "v")
            else:
                kt = np.ascontiguousarray(inp["k_tree"][b, :N, g])
                vt = np.ascontiguousarray(inp["v_tree"][b, :N, g])
            cache[(b, g)] = (kp, vp, kt, vt)
        kp, vp, kt, vt = cache[(b, g)]
        mrow = np.ascontiguousarray(cache[(b, "M")][i])
        qrow = np.ascontiguousarray(q[b, i, h])
        o = np.zeros(d, np.float64)
        l_ = np.zeros(1, np.float64)
        L_.orc_attn_row(_p(qrow), dt, _p(kp) if L else None, _p(vp) if L else None, L, d,
                        _p(kt), _p(vt), d, _p(mrow), N, d, scale, _p(o), _p(l_))
        out[r] = o
        lse[r] = l_[0]
    return out, lse, rows


# ----------------------------------------------------------------------------- acceptance
def argmax_row(row: np.ndarray) -> int:
    row = np.ascontiguousarray(row)
    return int(lib().orc_argmax_row(_p(row), _dt(row), row.shape[-1]))


def accept_greedy(inp: dict, logits=None, tokens=None):
    """Greedy tree acceptance for every sequence.  Returns dict(accept_len, path, out_tokens, codes)."""
    w = inp["workload"]
    logits = inp["logits"] if logits is None else logits
    tokens = inp["tokens"] if tokens is None else tokens
    parent, nn, Dmax = inp["parent"], inp["num_nodes"], int(inp["Dmax"])
    B, Nmax, V = logits.shape
    rk = inp.get("root_key")
    al = np.zeros(B, np.int32)
    path = np.zeros((B, Dmax + 1), np.int32)
    ot = np.zeros((B, Dmax + 1), np.int32)
    codes = []
    for b in range(B):
        N = int(nn[b])
        lg = np.ascontiguousarray(logits[b, :N]) if N else np.zeros((1, V), logits.dtype)
        tk = np.ascontiguousarray(tokens[b, :N]) if N else np.zeros(1, np.int32)
        pa = np.ascontiguousarray(parent[b, :N]) if N else np.zeros(1, np.int32)
        key = None if rk is None else np.array([rk[b]], np.int32)
        a = np.zeros(1, np.int32)
        code = lib().orc_accept_greedy(_p(lg), _dt(lg), V, _p(tk), _p(pa), N, Dmax,
                                       int(bool(getattr(w, "forest", False))),
                                       _p(key) if key is not None else None, _p(a),
                                       _p(path[b]), _p(ot[b]))
        al[b] = a[0]
        codes.append(CODE_NAMES[code])
    return {"accept_len": al, "path": path, "out_tokens": ot, "codes": codes}


def chain_sample(zp: np.ndarray, zq: np.ndarray, x: np.ndarray, u: np.ndarray, T: float):
    """Chain rejection sampling for every sequence: zp [B,K+1,V], zq [B,K,V], x [B,K], u [B,K+1]."""
    zp, zq = np.ascontiguousarray(zp), np.ascontiguousarray(zq)
    x = np.ascontiguousarray(x, np.int32)
    u = np.ascontiguousarray(u, np.float32)
    B, K1, V = zp.shape
    K = K1 - 1
    al = np.zeros(B, np.int32)
    ot = np.zeros((B, K + 1), np.int32)
    mg = np.zeros((B, K + 1), np.float64)
    code = lib().orc_chain_sample_many(B, _p(zp), _p(zq) if K else None, _dt(zp), V, K, _p(x) if K else None,
                                       _p(u), float(T), _p(al), _p(ot), _p(mg))
    assert code == 0
    return {"accept_len": al, "out_tokens": ot, "margin": mg}


# ----------------------------------------------------------------------------- commit
def kv_commit(inp: dict, accept_len, path, mode: str = "path", status=None, k_cache=None, v_cache=None,
              prefix_len=None):
    """Commit the accepted rows; returns (k_cache', v_cache', prefix_len', statuses) as copies.

    Works on the contiguous cache (k_cache/v_cache [B,Hkv,Lmax,d]) or the paged one
    (k_pages/v_pages [blocks,Hkv,bs,d] + block_table), whichever `inp` holds."""
    paged = "k_pages" in inp
    kc = (inp["k_pages"] if paged else inp["k_cache"]) if k_cache is None else k_cache
    vc = (inp["v_pages"] if paged else inp["v_cache"]) if v_cache is None else v_cache
    kc, vc = kc.copy(), vc.copy()
    pl = (inp["prefix_len"] if prefix_len is None else prefix_len).copy()
    kt, vt, nn = inp["k_tree"], inp["v_tree"], inp["num_nodes"]
    B = pl.shape[0]
    if paged:
        bs = kc.shape[2]
        table = inp["block_table"]
        cap = table.shape[1] * bs
    else:
        cap = kc.shape[2]
    st = ["ok"] * B

    def rows_at(arr, b, pos):           # view of cache rows at logical positions, all heads
        if paged:
            return arr[table[b, pos // bs], :, pos % bs]
        return arr[b, :, pos]

    def put(arr, b, pos, val):
        if paged:
            arr[table[b, pos // bs], :, pos % bs] = val
        else:
            arr[b, :, pos] = val

    for b in range(B):
        A = int(accept_len[b])
        if (status is not None and int(status[b]) != 0) or A < 0:
            continue
        L = int(pl[b])
        N = int(nn[b])
        if L + A + 1 > cap:
            st[b] = "capacity"
            continue
        if mode == "length":
            src = list(range(A + 1))
        else:
            src = [int(path[b][j]) - 1 for j in range(A + 1)]
            if any(s < 0 or s >= N for s in src):
                st[b] = "bad_path"
                continue
        if mode == "inplace":
            ks = [rows_at(kc, b, L + s).copy() for s in src]
            vs = [rows_at(vc, b, L + s).copy() for s in src]
        else:
            ks = [kt[b, s].copy() for s in src]
            vs = [vt[b, s].copy() for s in src]
        for j in range(A + 1):
            put(kc, b, L + j, ks[j])
            put(vc, b, L + j, vs[j])
        pl[b] = L + A + 1
    return kc, vc, pl, st


# ----------------------------------------------------------------------------- whole step
def verify_step(inp: dict, rows=None):
    """One whole verify step on the CPU: structure, attention (all rows, or `rows`),
    acceptance (greedy or chain sampling, per the workload) and commit."""
    w = inp["workload"]
    B = inp["parent"].shape[0]
    for b in range(B):
        st = tree_structure(inp["parent"][b, :int(inp["num_nodes"][b])], int(inp["Dmax"]),
                            bool(getattr(w, "forest", False)))
        assert st["code"] == "ok"
    out = attention_rows(inp, rows)
    if w.accept == "greedy":
        acc = accept_greedy(inp)
        res = kv_commit(inp, acc["accept_len"], acc["path"], "path")
    else:
        acc = chain_sample(inp["z_p"], inp["z_q"], inp["x"], inp["u"], inp["T"])
        res = kv_commit(inp, acc["accept_len"], None, "length")
    return out, acc, res


from .draft_tree import DraftTree, draft_tree_build  # noqa: E402,F401
from . import ssd_cache  # noqa: E402,F401
from . import tree_sample  # noqa: E402,F401
