"""Python binding of libtsd, the tree speculative decoding verify library for B200 (sm_100a).

Argument marshalling only: every step of the verify path runs in the CUDA kernels behind the
C ABI declared in ``include/tsd.h``.  PyTorch supplies device memory and the current stream.
The functions carry the C names without the ``tsd_`` prefix and return the output tensors
(allocated here with torch when the caller passes none).  There is no CPU fallback: if the
library is missing or no GPU is present, every call raises.

Layouts (row-major, see include/tsd.h): q/out [B,N,Hq,d]; k_tree/v_tree [B,N,Hkv,d]; contiguous
cache [B,Hkv,Lmax,d]; paged cache [num_blocks,Hkv,block,d] + block_table [B,max_blocks]; logits
[B,N,V].  Node i's slot is i+1 (slot 0 is the dummy row that replaces the root's -1 parent).
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtsd.so")
_lib = None

TSD_F32, TSD_BF16 = 0, 1
COMMIT_MODES = {"path": 0, "length": 1, "inplace": 2}
STATUS = {0: "TSD_OK", 1: "TSD_ERR_INVALID_ARG", 2: "TSD_ERR_UNSUPPORTED_DTYPE", 3: "TSD_ERR_BAD_TREE",
          4: "TSD_ERR_TREE_DEPTH", 5: "TSD_ERR_TREE_ROOTS", 6: "TSD_ERR_CAPACITY", 7: "TSD_ERR_TIMEOUT",
          8: "TSD_ERR_CUDA", 9: "TSD_ERR_WORKSPACE"}
STATUS_CODE = {v: k for k, v in STATUS.items()}

# C signatures: name -> (restype, argtypes)
_P, _I, _F, _SZ = C.c_void_p, C.c_int, C.c_float, C.c_size_t
_SIGS = {
    "tsd_status_str": (C.c_char_p, [_I]),
    "tsd_abi_version": (_I, []),
    "tsd_tree_prepare": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "tsd_tree_verify_attn_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "tsd_tree_verify_attn": (_I, [_P, _P, _P, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P,
                                  _P, _SZ, _P, _P]),
    "tsd_tree_verify_attn_paged_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "tsd_tree_verify_attn_ticket_bytes": (_SZ, []),
    "tsd_tree_verify_attn_kernels": (_I, [_I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "tsd_tree_verify_attn_ctas": (C.c_longlong, [_I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "tsd_tree_verify_attn_paged": (_I, [_P, _P, _P, _I, _I, _P, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                        _I, _F, _P, _P, _P, _SZ, _P, _P]),
    "tsd_tree_accept_greedy_workspace_size": (_SZ, [_I, _I, _I]),
    "tsd_tree_accept_greedy": (_I, [_P, _I, _I, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _P, _SZ, _P, _P]),
    "tsd_tree_accept_threshold_workspace_size": (_SZ, [_I, _I, _I]),
    "tsd_tree_accept_threshold": (_I, [_P, _I, _I, _P, _P, _P, _P, _F, _F, _I, _I, _I, _P, _P, _P, _P, _SZ, _P, _P]),
    "tsd_tree_accept_greedy_noalloc": (_I, [_P, _I, _I, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _P, _P]),
    "tsd_tree_accept_greedy_noalloc_scratch_bytes": (_SZ, []),
    "tsd_chain_accept_sample_workspace_size": (_SZ, [_I, _I, _I]),
    "tsd_ssd_cache_build": (_I, [_P, _I, _I, _I, _I, _P, _F, _P, _F, _I, _P, _P, _P, _P, _P]),
    "tsd_tree_accept_sample": (_I, [_P, _P, _I, _I, _P, _P, _P, _P, _F, _I, _I, _I, _P, _P, _P, _P, _P]),
    "tsd_chain_accept_sample": (_I, [_P, _P, _I, _I, _P, _P, _F, _I, _I, _P, _P, _P, _SZ, _P]),
    "tsd_kv_commit": (_I, [_P, _P, _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P]),
    "tsd_kv_commit_paged": (_I, [_P, _P, _I, _I, _P, _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                 _P, _P]),
}


class KVCacheDesc(C.Structure):
    """tsd_kv_cache: the committed cache as the fused acceptance + commit call sees it."""
    _fields_ = [("k", _P), ("v", _P), ("prefix_len", _P), ("Lmax", _I), ("block_table", _P), ("max_blocks", _I),
                ("block_size", _I), ("num_blocks", _I)]


class DraftTreeDesc(C.Structure):
    """tsd_draft_tree: the device arrays of a draft tree under construction."""
    _fields_ = [("parent", _P), ("token", _P), ("score", _P), ("depth", _P), ("num_nodes", _P), ("frontier", _P),
                ("num_frontier", _P), ("max_nodes", _I), ("F", _I)]


_DT = C.POINTER(DraftTreeDesc)
_SIGS["tsd_draft_tree_init"] = (_I, [_DT, _P, _I, _P, _P])
_SIGS["tsd_draft_tree_expand_workspace_size"] = (_SZ, [_I, _I, _I, _I])
_SIGS["tsd_draft_tree_expand"] = (_I, [_DT, _P, _I, _I, _I, _I, _P, _SZ, _P, _P])
_SIGS["tsd_draft_tree_finalize"] = (_I, [_DT, _I, _I, _P, _P, _P, _P, _P])
_SIGS["tsd_tree_accept_commit"] = (_I, [_P, _I, _I, _P, _P, _P, _P, _I, _I, _I, C.POINTER(KVCacheDesc), _P, _P, _I,
                                        _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _SZ, _P, _P])


class TsdError(RuntimeError):
    pass


def lib() -> C.CDLL:
    """Load libtsd.so (built in-tree by ``__graft_entry__.build()``); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise TsdError(f"{LIB_PATH} is missing: build the CUDA library first "
                           "(python -m tree_speculative_decoding_06_b200._build)")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def status_str(code: int) -> str:
    return lib().tsd_status_str(int(code)).decode()


def _check(rc: int, name: str):
    if rc != 0:
        raise TsdError(f"{name} returned {status_str(rc)} ({rc})")


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return TSD_F32
    if t.dtype == torch.bfloat16:
        return TSD_BF16
    raise TsdError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise TsdError("tensor arguments must be CUDA tensors")
    if not t.is_contiguous():
        raise TsdError("tensor arguments must be contiguous")
    return C.c_void_p(t.data_ptr())


def _i32(t: Optional[torch.Tensor], name: str):
    if t is not None and t.dtype != torch.int32:
        raise TsdError(f"{name} must be int32")
    return _ptr(t)


def _stream(stream=None) -> C.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _empty(shape, dtype, like: torch.Tensor):
    return torch.empty(shape, dtype=dtype, device=like.device)


# ----------------------------------------------------------------------------- prepare
def tree_prepare(parent, num_nodes=None, Dmax: int = 8, forest: bool = False, parent_s=None, depth=None,
                 anc=None, anc_bits=None, status=None, want_bits: bool = False, stream=None):
    B, Nmax = parent.shape
    parent_s = _empty((B, Nmax + 1), torch.int32, parent) if parent_s is None else parent_s
    depth = _empty((B, Nmax + 1), torch.int32, parent) if depth is None else depth
    anc = _empty((B, Nmax + 1, Dmax + 1), torch.int32, parent) if anc is None else anc
    if anc_bits is None and want_bits:
        anc_bits = _empty((B, Nmax + 1, (Nmax + 1 + 31) // 32), torch.int32, parent)
    status = _empty((B,), torch.int32, parent) if status is None else status
    rc = lib().tsd_tree_prepare(_i32(parent, "parent"), _i32(num_nodes, "num_nodes"), B, Nmax, Dmax, int(forest),
                                _ptr(parent_s), _ptr(depth), _ptr(anc), _ptr(anc_bits), _ptr(status),
                                _stream(stream))
    _check(rc, "tsd_tree_prepare")
    return {"parent_s": parent_s, "depth": depth, "anc": anc, "anc_bits": anc_bits, "status": status}


# ----------------------------------------------------------------------------- attention
def tree_verify_attn_workspace_size(B, Nmax, Hq, Hkv, d, Lmax, dtype) -> int:
    return int(lib().tsd_tree_verify_attn_workspace_size(B, Nmax, Hq, Hkv, d, Lmax, dtype))


def tree_verify_attn_paged_workspace_size(B, Nmax, Hq, Hkv, d, max_blocks, block_size, dtype) -> int:
    return int(lib().tsd_tree_verify_attn_paged_workspace_size(B, Nmax, Hq, Hkv, d, max_blocks, block_size, dtype))


def tree_verify_attn_ticket_bytes() -> int:
    """Bytes of split-merge ticket words at the start of an attention workspace (kept zero)."""
    return int(lib().tsd_tree_verify_attn_ticket_bytes())


def tree_verify_attn_kernels(B, Nmax, Hq, Hkv, d, Lmax, dtype, block_size: int = 0, tree_in_cache: bool = False) -> int:
    """Kernels one attention call launches for these sizes (the split kernel, and the merge kernel
    when the keys are split and not merged inside it); Lmax = capacity, block_size 0 = contiguous."""
    return int(lib().tsd_tree_verify_attn_kernels(B, Nmax, Hq, Hkv, d, Lmax, block_size, int(tree_in_cache), dtype))


def tree_verify_attn_ctas(B, Nmax, Hq, Hkv, d, Lmax, dtype, block_size: int = 0, tree_in_cache: bool = False) -> int:
    """CTAs of the attention call's split kernel for these sizes (its grid)."""
    return int(lib().tsd_tree_verify_attn_ctas(B, Nmax, Hq, Hkv, d, Lmax, block_size, int(tree_in_cache), dtype))


def _nbytes(ws) -> int:
    """Bytes of a workspace tensor (0 for None): the size the C call is told it may use."""
    return 0 if ws is None else ws.numel() * ws.element_size()


def _ws(nbytes: int, like: torch.Tensor, ws):
    # a new workspace starts zeroed: the attention's ticket words must be zero before first use
    if nbytes == 0:
        return ws
    if ws is None or ws.numel() * ws.element_size() < nbytes:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=like.device)
    return ws


def tree_verify_attn(q, k_cache, v_cache, prefix_len, k_tree, v_tree, parent_s, num_nodes=None, Dmax: int = 8,
                     scale: Optional[float] = None, out=None, lse=None, workspace=None, status=None,
                     want_lse: bool = False, stream=None):
    """Contiguous cache [B,Hkv,Lmax,d]; k_tree=v_tree=None reads the tree K/V from the cache
    right after each prefix.  Returns (out, lse)."""
    B, Nmax, Hq, d = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    dt = _dt(q)
    scale = d ** -0.5 if scale is None else scale
    out = torch.empty_like(q) if out is None else out
    if lse is None and want_lse:
        lse = _empty((B, Nmax, Hq), torch.float32, q)
    if status is None:
        status = torch.zeros(B, dtype=torch.int32, device=q.device)
    nbytes = tree_verify_attn_workspace_size(B, Nmax, Hq, Hkv, d, Lmax, dt)
    workspace = _ws(nbytes, q, workspace)
    rc = lib().tsd_tree_verify_attn(_ptr(q), _ptr(k_cache), _ptr(v_cache), Lmax, _i32(prefix_len, "prefix_len"),
                                    _ptr(k_tree), _ptr(v_tree), _i32(parent_s, "parent_s"),
                                    _i32(num_nodes, "num_nodes"), B, Nmax, Hq, Hkv, d, Dmax, dt, float(scale),
                                    _ptr(out), _ptr(lse), _ptr(workspace), _nbytes(workspace), _ptr(status),
                                    _stream(stream))
    _check(rc, "tsd_tree_verify_attn")
    return out, lse


def tree_verify_attn_paged(q, k_pages, v_pages, block_table, prefix_len, k_tree, v_tree, parent_s, num_nodes=None,
                           Dmax: int = 8, scale: Optional[float] = None, out=None, lse=None, workspace=None,
                           status=None, want_lse: bool = False, stream=None):
    """Paged cache [num_blocks,Hkv,block,d] + block_table [B,max_blocks].  Returns (out, lse)."""
    B, Nmax, Hq, d = q.shape
    nblk, Hkv, bs = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    max_blocks = block_table.shape[1]
    dt = _dt(q)
    scale = d ** -0.5 if scale is None else scale
    out = torch.empty_like(q) if out is None else out
    if lse is None and want_lse:
        lse = _empty((B, Nmax, Hq), torch.float32, q)
    if status is None:
        status = torch.zeros(B, dtype=torch.int32, device=q.device)
    nbytes = tree_verify_attn_paged_workspace_size(B, Nmax, Hq, Hkv, d, max_blocks, bs, dt)
    workspace = _ws(nbytes, q, workspace)
    rc = lib().tsd_tree_verify_attn_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), nblk, bs,
                                          _i32(block_table, "block_table"), max_blocks,
                                          _i32(prefix_len, "prefix_len"), _ptr(k_tree), _ptr(v_tree),
                                          _i32(parent_s, "parent_s"), _i32(num_nodes, "num_nodes"), B, Nmax, Hq,
                                          Hkv, d, Dmax, dt, float(scale), _ptr(out), _ptr(lse), _ptr(workspace),
                                          _nbytes(workspace), _ptr(status), _stream(stream))
    _check(rc, "tsd_tree_verify_attn_paged")
    return out, lse


# ----------------------------------------------------------------------------- acceptance
def tree_accept_greedy_workspace_size(B, Nmax, V) -> int:
    return int(lib().tsd_tree_accept_greedy_workspace_size(B, Nmax, V))


def tree_accept_greedy(logits, tokens, parent_s, num_nodes=None, root_key=None, Dmax: int = 8, accept_len=None,
                       path=None, out_tokens=None, workspace=None, status=None, stream=None):
    B, Nmax, V = logits.shape
    accept_len = _empty((B,), torch.int32, logits) if accept_len is None else accept_len
    path = _empty((B, Dmax + 1), torch.int32, logits) if path is None else path
    out_tokens = _empty((B, Dmax + 1), torch.int32, logits) if out_tokens is None else out_tokens
    if status is None:
        status = torch.zeros(B, dtype=torch.int32, device=logits.device)
    nbytes = tree_accept_greedy_workspace_size(B, Nmax, V)
    workspace = _ws(nbytes, logits, workspace)
    rc = lib().tsd_tree_accept_greedy(_ptr(logits), _dt(logits), V, _i32(tokens, "tokens"),
                                      _i32(parent_s, "parent_s"), _i32(num_nodes, "num_nodes"),
                                      _i32(root_key, "root_key"), B, Nmax, Dmax, _ptr(accept_len), _ptr(path),
                                      _ptr(out_tokens), _ptr(workspace), nbytes, _ptr(status), _stream(stream))
    _check(rc, "tsd_tree_accept_greedy")
    return {"accept_len": accept_len, "path": path, "out_tokens": out_tokens}


def tree_accept_threshold_workspace_size(B, Nmax, V) -> int:
    return int(lib().tsd_tree_accept_threshold_workspace_size(B, Nmax, V))


def tree_accept_threshold(logits, tokens, parent_s, tau: float, temperature: float = 1.0, num_nodes=None,
                          root_key=None, Dmax: int = 8, accept_len=None, path=None, out_tokens=None, workspace=None,
                          status=None, stream=None):
    """Threshold acceptance over the tree (tsd_tree_accept_threshold): a node is accepted while its
    parent's target distribution gives its token probability >= tau."""
    B, Nmax, V = logits.shape
    accept_len = _empty((B,), torch.int32, logits) if accept_len is None else accept_len
    path = _empty((B, Dmax + 1), torch.int32, logits) if path is None else path
    out_tokens = _empty((B, Dmax + 1), torch.int32, logits) if out_tokens is None else out_tokens
    if status is None:
        status = torch.zeros(B, dtype=torch.int32, device=logits.device)
    nbytes = tree_accept_threshold_workspace_size(B, Nmax, V)
    workspace = _ws(nbytes, logits, workspace)
    rc = lib().tsd_tree_accept_threshold(_ptr(logits), _dt(logits), V, _i32(tokens, "tokens"),
                                         _i32(parent_s, "parent_s"), _i32(num_nodes, "num_nodes"),
                                         _i32(root_key, "root_key"), float(tau), float(temperature), B, Nmax, Dmax,
                                         _ptr(accept_len), _ptr(path), _ptr(out_tokens), _ptr(workspace), nbytes,
                                         _ptr(status), _stream(stream))
    _check(rc, "tsd_tree_accept_threshold")
    return {"accept_len": accept_len, "path": path, "out_tokens": out_tokens}


def accept_noalloc_scratch_bytes() -> int:
    """Size of the fixed scratch array tree_accept_greedy_noalloc uses, read from the library."""
    return int(lib().tsd_tree_accept_greedy_noalloc_scratch_bytes())


def tree_accept_greedy_noalloc(logits, tokens, parent_s, num_nodes=None, root_key=None, Dmax: int = 8,
                               accept_len=None, path=None, out_tokens=None, status=None, stream=None):
    """tree_accept_greedy for callers that may not allocate device scratch: the library's own
    fixed scratch array (accept_noalloc_scratch_bytes() per device) is used instead of a
    workspace.  Calls that overlap on the GPU share that array and race; the first call on a
    device should come before any stream capture."""
    B, Nmax, V = logits.shape
    accept_len = _empty((B,), torch.int32, logits) if accept_len is None else accept_len
    path = _empty((B, Dmax + 1), torch.int32, logits) if path is None else path
    out_tokens = _empty((B, Dmax + 1), torch.int32, logits) if out_tokens is None else out_tokens
    if status is None:
        status = torch.zeros(B, dtype=torch.int32, device=logits.device)
    rc = lib().tsd_tree_accept_greedy_noalloc(_ptr(logits), _dt(logits), V, _i32(tokens, "tokens"),
                                              _i32(parent_s, "parent_s"), _i32(num_nodes, "num_nodes"),
                                              _i32(root_key, "root_key"), B, Nmax, Dmax, _ptr(accept_len),
                                              _ptr(path), _ptr(out_tokens), _ptr(status), _stream(stream))
    _check(rc, "tsd_tree_accept_greedy_noalloc")
    return {"accept_len": accept_len, "path": path, "out_tokens": out_tokens}


def chain_accept_sample_workspace_size(B, K, V) -> int:
    return int(lib().tsd_chain_accept_sample_workspace_size(B, K, V))


def chain_accept_sample(target_logits, draft_logits, draft_tokens, uniforms, temperature: float,
                        accept_len=None, out_tokens=None, workspace=None, stream=None):
    B, K1, V = target_logits.shape
    K = K1 - 1
    accept_len = _empty((B,), torch.int32, target_logits) if accept_len is None else accept_len
    out_tokens = _empty((B, K + 1), torch.int32, target_logits) if out_tokens is None else out_tokens
    nbytes = chain_accept_sample_workspace_size(B, K, V)
    workspace = _ws(nbytes, target_logits, workspace)
    if uniforms.dtype != torch.float32:
        raise TsdError("uniforms must be float32")
    rc = lib().tsd_chain_accept_sample(_ptr(target_logits), _ptr(draft_logits), _dt(target_logits), V,
                                       _i32(draft_tokens, "draft_tokens"), _ptr(uniforms), float(temperature), B, K,
                                       _ptr(accept_len), _ptr(out_tokens), _ptr(workspace), nbytes,
                                       _stream(stream))
    _check(rc, "tsd_chain_accept_sample")
    return {"accept_len": accept_len, "out_tokens": out_tokens}


def tree_accept_sample(target_logits, draft_logits, tokens, parent_s, uniforms, temperature: float,
                       num_nodes=None, Dmax: int = 8, accept_len=None, path=None, out_tokens=None, status=None,
                       stream=None):
    """Stochastic acceptance of a draft tree (tsd_tree_accept_sample): target_logits / draft_logits
    [B, N, V] (row n = after node n), tokens [B, N], uniforms [B, N] fp32 (entry c tests node c,
    entry 0 is the final draw)."""
    B, Nmax, V = target_logits.shape
    if tuple(draft_logits.shape) != (B, Nmax, V) or draft_logits.dtype != target_logits.dtype:
        raise TsdError("draft_logits must match target_logits in shape and dtype")
    if uniforms.dtype != torch.float32 or tuple(uniforms.shape) != (B, Nmax):
        raise TsdError("uniforms must be float32 [B, Nmax]")
    accept_len = _empty((B,), torch.int32, target_logits) if accept_len is None else accept_len
    path = _empty((B, Dmax + 1), torch.int32, target_logits) if path is None else path
    out_tokens = _empty((B, Dmax + 1), torch.int32, target_logits) if out_tokens is None else out_tokens
    if status is None:
        status = torch.zeros(B, dtype=torch.int32, device=target_logits.device)
    rc = lib().tsd_tree_accept_sample(_ptr(target_logits), _ptr(draft_logits), _dt(target_logits), V,
                                      _i32(tokens, "tokens"), _i32(parent_s, "parent_s"),
                                      _i32(num_nodes, "num_nodes"), _ptr(uniforms), float(temperature), B, Nmax,
                                      Dmax, _ptr(accept_len), _ptr(path), _ptr(out_tokens), _ptr(status),
                                      _stream(stream))
    _check(rc, "tsd_tree_accept_sample")
    return {"accept_len": accept_len, "path": path, "out_tokens": out_tokens}


def ssd_cache_build(draft_logits, alpha, beta: float, uniforms, S: int, temperature: float = 1.0, slots=None,
                    key_len=None, key_tok=None, draft_tokens=None, stream=None):
    """SSD / Saguaro outcome cache (tsd_ssd_cache_build): draft_logits [B, K+1, V], alpha [B] fp32,
    uniforms [B, K] fp32.  Returns slots [B, K+1], key_len / key_tok [B, S], draft_tokens [B, K]."""
    B, K1, V = draft_logits.shape
    K = K1 - 1
    if alpha.dtype != torch.float32 or uniforms.dtype != torch.float32:
        raise TsdError("alpha and uniforms must be float32")
    slots = _empty((B, K + 1), torch.int32, draft_logits) if slots is None else slots
    key_len = _empty((B, S), torch.int32, draft_logits) if key_len is None else key_len
    key_tok = _empty((B, S), torch.int32, draft_logits) if key_tok is None else key_tok
    draft_tokens = _empty((B, max(K, 1)), torch.int32, draft_logits) if draft_tokens is None else draft_tokens
    rc = lib().tsd_ssd_cache_build(_ptr(draft_logits), _dt(draft_logits), V, K, S, _ptr(alpha), float(beta),
                                   _ptr(uniforms), float(temperature), B, _ptr(slots), _ptr(key_len), _ptr(key_tok),
                                   _ptr(draft_tokens), _stream(stream))
    _check(rc, "tsd_ssd_cache_build")
    return {"slots": slots, "key_len": key_len, "key_tok": key_tok, "draft_tokens": draft_tokens}


# ----------------------------------------------------------------------------- commit
def kv_commit(k_cache, v_cache, prefix_len, k_tree, v_tree, path, accept_len, num_nodes=None, Dmax: int = 8,
              mode: str = "path", status=None, Nmax: Optional[int] = None, stream=None):
    B, Hkv, Lmax, d = k_cache.shape
    Nmax = (k_tree.shape[1] if k_tree is not None else Nmax)
    if Nmax is None:
        raise TsdError("Nmax is needed when the tree K/V are not given")
    if status is None:
        status = torch.zeros(B, dtype=torch.int32, device=k_cache.device)
    rc = lib().tsd_kv_commit(_ptr(k_cache), _ptr(v_cache), Lmax, _i32(prefix_len, "prefix_len"), _ptr(k_tree),
                             _ptr(v_tree), _i32(path, "path"), _i32(accept_len, "accept_len"),
                             _i32(num_nodes, "num_nodes"), B, Nmax, Hkv, d, Dmax, _dt(k_cache), COMMIT_MODES[mode],
                             _ptr(status), _stream(stream))
    _check(rc, "tsd_kv_commit")
    return status


def kv_commit_paged(k_pages, v_pages, block_table, prefix_len, k_tree, v_tree, path, accept_len, num_nodes=None,
                    Dmax: int = 8, mode: str = "path", status=None, Nmax: Optional[int] = None, stream=None):
    nblk, Hkv, bs, d = k_pages.shape
    B, max_blocks = block_table.shape
    Nmax = (k_tree.shape[1] if k_tree is not None else Nmax)
    if Nmax is None:
        raise TsdError("Nmax is needed when the tree K/V are not given")
    if status is None:
        status = torch.zeros(B, dtype=torch.int32, device=k_pages.device)
    rc = lib().tsd_kv_commit_paged(_ptr(k_pages), _ptr(v_pages), nblk, bs, _i32(block_table, "block_table"),
                                   max_blocks, _i32(prefix_len, "prefix_len"), _ptr(k_tree), _ptr(v_tree),
                                   _i32(path, "path"), _i32(accept_len, "accept_len"), _i32(num_nodes, "num_nodes"),
                                   B, Nmax, Hkv, d, Dmax, _dt(k_pages), COMMIT_MODES[mode], _ptr(status),
                                   _stream(stream))
    _check(rc, "tsd_kv_commit_paged")
    return status


def tree_accept_commit(logits, tokens, parent_s, k_cache, v_cache, prefix_len, k_tree, v_tree, num_nodes=None,
                       root_key=None, Dmax: int = 8, mode: str = "path", block_table=None, history=None,
                       history_len=None, accept_len=None, path=None, out_tokens=None, workspace=None, status=None,
                       stream=None):
    """Greedy acceptance fused with the commit of the accepted path (tsd_tree_accept_commit).
    k_cache/v_cache are [B,Hkv,Lmax,d], or pages [num_blocks,Hkv,block,d] when block_table is
    given.  With history [B,cap] and history_len [B] the emitted tokens are appended on the
    device.  Returns the acceptance outputs; the cache, prefix_len and history change in place."""
    B, Nmax, V = logits.shape
    accept_len = _empty((B,), torch.int32, logits) if accept_len is None else accept_len
    path = _empty((B, Dmax + 1), torch.int32, logits) if path is None else path
    out_tokens = _empty((B, Dmax + 1), torch.int32, logits) if out_tokens is None else out_tokens
    if status is None:
        status = torch.zeros(B, dtype=torch.int32, device=logits.device)
    nbytes = tree_accept_greedy_workspace_size(B, Nmax, V)
    workspace = _ws(nbytes, logits, workspace)
    if block_table is not None:
        nblk, Hkv, bs, d = k_cache.shape
        desc = KVCacheDesc(_ptr(k_cache), _ptr(v_cache), _i32(prefix_len, "prefix_len"), 0,
                           _i32(block_table, "block_table"), block_table.shape[1], bs, nblk)
    else:
        _, Hkv, Lmax, d = k_cache.shape
        desc = KVCacheDesc(_ptr(k_cache), _ptr(v_cache), _i32(prefix_len, "prefix_len"), Lmax, None, 0, 0, 0)
    cap = history.shape[1] if history is not None else 0
    rc = lib().tsd_tree_accept_commit(_ptr(logits), _dt(logits), V, _i32(tokens, "tokens"),
                                      _i32(parent_s, "parent_s"), _i32(num_nodes, "num_nodes"),
                                      _i32(root_key, "root_key"), B, Nmax, Dmax, C.byref(desc), _ptr(k_tree),
                                      _ptr(v_tree), Hkv, d, _dt(k_cache), COMMIT_MODES[mode],
                                      _i32(history, "history"), cap, _i32(history_len, "history_len"),
                                      _ptr(accept_len), _ptr(path), _ptr(out_tokens), _ptr(workspace), nbytes,
                                      _ptr(status), _stream(stream))
    _check(rc, "tsd_tree_accept_commit")
    return {"accept_len": accept_len, "path": path, "out_tokens": out_tokens}


# ----------------------------------------------------------------------------- draft tree
class DraftTree:
    """A batch of EAGLE-2 draft trees built on the device (tsd_draft_tree_*).

    ``init(root_tokens)`` starts every tree at its root; ``expand(draft_logits, K)`` takes the
    [B, F, V] draft logits of the current frontier nodes (row f after frontier node f) and adds
    their top-K children; ``finalize(keep)`` returns the parent[] / tokens / num_nodes of the
    kept tree, ready for ``tree_prepare`` and the verify step."""

    def __init__(self, B: int, F: int, max_nodes: int, device="cuda"):
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        self.B, self.F, self.max_nodes = B, F, max_nodes
        self.parent = torch.zeros(B, max_nodes, **i32)
        self.token = torch.zeros(B, max_nodes, **i32)
        self.score = torch.zeros(B, max_nodes, dtype=torch.float64, device=dev)
        self.depth = torch.zeros(B, max_nodes, **i32)
        self.num_nodes = torch.zeros(B, **i32)
        self.frontier = torch.zeros(B, F, **i32)
        self.num_frontier = torch.zeros(B, **i32)
        self.status = torch.zeros(B, **i32)
        self._ws = None
        self.desc = DraftTreeDesc(_ptr(self.parent), _ptr(self.token), _ptr(self.score), _ptr(self.depth),
                                  _ptr(self.num_nodes), _ptr(self.frontier), _ptr(self.num_frontier), max_nodes, F)

    def init(self, root_tokens, stream=None):
        _check(lib().tsd_draft_tree_init(C.byref(self.desc), _i32(root_tokens, "root_tokens"), self.B,
                                         _ptr(self.status), _stream(stream)), "tsd_draft_tree_init")

    def expand(self, draft_logits, K: int, stream=None):
        B, F, V = draft_logits.shape
        if B != self.B or F != self.F:
            raise TsdError("draft_logits must be [B, F, V] of this tree")
        nbytes = int(lib().tsd_draft_tree_expand_workspace_size(B, F, K, V))
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=draft_logits.device)
        _check(lib().tsd_draft_tree_expand(C.byref(self.desc), _ptr(draft_logits), _dt(draft_logits), V, K, B,
                                           _ptr(self._ws), nbytes, _ptr(self.status), _stream(stream)),
               "tsd_draft_tree_expand")

    def finalize(self, keep: int, parent=None, tokens=None, num_nodes=None, stream=None):
        dev = self.parent.device
        parent = torch.empty(self.B, keep, dtype=torch.int32, device=dev) if parent is None else parent
        tokens = torch.empty(self.B, keep, dtype=torch.int32, device=dev) if tokens is None else tokens
        num_nodes = torch.empty(self.B, dtype=torch.int32, device=dev) if num_nodes is None else num_nodes
        _check(lib().tsd_draft_tree_finalize(C.byref(self.desc), self.B, keep, _ptr(parent), _ptr(tokens),
                                             _ptr(num_nodes), _ptr(self.status), _stream(stream)),
               "tsd_draft_tree_finalize")
        return {"parent": parent, "tokens": tokens, "num_nodes": num_nodes}


from .step import VerifyStep  # noqa: E402,F401
