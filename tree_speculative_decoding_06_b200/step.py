"""One whole verify step through the C ABI, with its buffers allocated once.

``VerifyStep(...)`` sizes every output and workspace for one batch shape; ``run(inputs)``
enqueues, on the current stream and without any host synchronisation,

    tsd_tree_prepare -> tsd_tree_verify_attn[_paged] -> acceptance -> tsd_kv_commit[_paged]

The acceptance (greedy, or the chain sampler) depends on the tree and the logits only, not on the
attention, so by default (schedule "overlap") it runs on a second stream forked after prepare --
the vocabulary scans and the decisions then use the SMs and memory cycles the attention leaves
idle -- and the commit (which must follow the attention: it advances prefix_len, which the
attention reads) joins both.  Schedule "fused"
runs tsd_tree_accept_commit after the attention on one stream (and can splice the emitted tokens
into a device token history); "serial" runs the acceptance then tsd_kv_commit on one stream.  A
linear draft takes tsd_chain_accept_sample -> tsd_kv_commit[_paged] (length mode).

In the overlap schedule the acceptance reads status[b] while the attention may still be flagging
that sequence (a bad block id, a capacity error, a timed-out wait): for a sequence whose status is
non-zero after the step, accept_len / path / out_tokens are unspecified (the other schedules give
the miss outputs).  The commit always reads the final status, so the status words, the caches and
prefix_len come out the same under every schedule.

run() returns the device tensors it wrote.  The cache and prefix_len in `inputs` are updated in
place by the commit, exactly as a decoding loop would carry them into the next step; with
history_cap > 0 the emitted tokens are also appended to a device token history.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import (tree_prepare, tree_verify_attn, tree_verify_attn_paged, tree_accept_greedy, chain_accept_sample,
               kv_commit, kv_commit_paged, tree_accept_commit, tree_verify_attn_workspace_size,
               tree_verify_attn_paged_workspace_size, tree_verify_attn_kernels, tree_verify_attn_ctas,
               tree_accept_greedy_workspace_size,
               chain_accept_sample_workspace_size, TSD_BF16, TSD_F32)


class VerifyStep:
    def __init__(self, *, B: int, Nmax: int, Hq: int, Hkv: int, d: int, Dmax: int, V: int, dtype: torch.dtype,
                 Lmax: Optional[int] = None, paged: bool = False, block_size: int = 16,
                 max_blocks: Optional[int] = None, forest: bool = False, accept: str = "greedy", K: int = 0,
                 schedule: Optional[str] = None, history_cap: int = 0, T: float = 0.0, device="cuda"):
        self.B, self.Nmax, self.Hq, self.Hkv, self.d, self.Dmax, self.V = B, Nmax, Hq, Hkv, d, Dmax, V
        self.dtype, self.paged, self.forest, self.accept, self.K = dtype, paged, forest, accept, K
        if schedule is None:
            schedule = "fused" if history_cap > 0 and accept == "greedy" else "overlap"
        if schedule not in ("overlap", "fused", "serial"):
            raise ValueError(f"unknown schedule {schedule!r}")
        if schedule == "fused" and accept != "greedy":
            raise ValueError("the fused schedule is greedy acceptance + commit")
        if history_cap > 0 and schedule != "fused":
            raise ValueError("a token history needs the fused schedule")
        self.schedule = schedule
        self.fused = schedule == "fused"
        self.T = T
        dt = TSD_BF16 if dtype == torch.bfloat16 else TSD_F32
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        self.parent_s = torch.zeros(B, Nmax + 1, **i32)
        self.depth = torch.zeros(B, Nmax + 1, **i32)
        self.anc = torch.zeros(B, Nmax + 1, Dmax + 1, **i32)
        self.status = torch.zeros(B, **i32)
        self.out = torch.empty(B, Nmax, Hq, d, dtype=dtype, device=dev)
        if paged:
            ws = tree_verify_attn_paged_workspace_size(B, Nmax, Hq, Hkv, d, max_blocks, block_size, dt)
        else:
            ws = tree_verify_attn_workspace_size(B, Nmax, Hq, Hkv, d, Lmax, dt)
        self.attn_ws = torch.zeros(max(ws, 1), dtype=torch.uint8, device=dev)   # ticket words start at zero
        if accept == "greedy":
            self.acc_ws = torch.empty(max(tree_accept_greedy_workspace_size(B, Nmax, V), 1), dtype=torch.uint8,
                                      device=dev)
            self.accept_len = torch.zeros(B, **i32)
            self.path = torch.zeros(B, Dmax + 1, **i32)
            self.out_tokens = torch.zeros(B, Dmax + 1, **i32)
        else:
            self.acc_ws = torch.empty(max(chain_accept_sample_workspace_size(B, K, V), 1), dtype=torch.uint8,
                                      device=dev)
            self.accept_len = torch.zeros(B, **i32)
            self.path = None
            self.out_tokens = torch.zeros(B, K + 1, **i32)
        self.history = torch.zeros(B, history_cap, **i32) if history_cap > 0 and self.fused else None
        self.history_len = torch.zeros(B, **i32) if self.history is not None else None
        # kernels of one attention call: the split kernel, and a merge kernel when the keys are split
        # and not merged inside it
        cap = max_blocks * block_size if paged else Lmax
        self.attn_kernels = tree_verify_attn_kernels(B, Nmax, Hq, Hkv, d, cap, dt, block_size if paged else 0)
        # Overlap schedule, launch order (measured on B200): an attention grid smaller than the GPU
        # (tree26: 72 CTAs) goes first and the acceptance's scan fills the idle SMs (step 29.1 ->
        # 26.2 us); a grid that fills the GPU (eagle60: 256 CTAs) goes after the scan, which then
        # runs alone at full bandwidth first (202.6 against 208.3 us the other way round).
        ctas = tree_verify_attn_ctas(B, Nmax, Hq, Hkv, d, cap, dt, block_size if paged else 0)
        self.attention_first = ctas < torch.cuda.get_device_properties(dev).multi_processor_count
        if schedule == "overlap":
            self.side = torch.cuda.Stream(device=dev)
            self.ev_fork, self.ev_join = torch.cuda.Event(), torch.cuda.Event()

    def launches_per_step(self) -> int:
        """Kernels one run() launches: prepare, attention (+ split merge), acceptance (scan +
        decide, or the chain sampler's three), commit (inside the fused acceptance)."""
        n = 1 + self.attn_kernels
        if self.accept == "greedy":
            return n + (2 if self.fused else 3)
        return n + (4 if self.T > 0 else 2) + 1

    def attn_launches(self) -> int:
        """Kernels one attention call launches (the split kernel, and its merge when split)."""
        return self.attn_kernels

    def _fork_accept(self, x: dict):
        """The acceptance on the side stream, after the prepare (the fork event), joined before the
        commit."""
        self.side.wait_event(self.ev_fork)
        with torch.cuda.stream(self.side):
            self._accept(x)
            self.ev_join.record(self.side)

    def _accept(self, x: dict):
        if self.accept == "greedy":
            tree_accept_greedy(x["logits"], x["tokens"], self.parent_s, x.get("num_nodes"), x.get("root_key"),
                               self.Dmax, accept_len=self.accept_len, path=self.path, out_tokens=self.out_tokens,
                               workspace=self.acc_ws, status=self.status)
        else:
            chain_accept_sample(x["z_p"], x["z_q"], x["x"], x["u"], x["T"], accept_len=self.accept_len,
                                out_tokens=self.out_tokens, workspace=self.acc_ws)

    def run(self, x: dict) -> dict:
        tree_prepare(x["parent"], x.get("num_nodes"), self.Dmax, self.forest, parent_s=self.parent_s,
                     depth=self.depth, anc=self.anc, status=self.status)
        overlap = self.schedule == "overlap"   # acceptance on the side stream, concurrently with the attention
        accept_first = not self.attention_first
        if overlap:
            main = torch.cuda.current_stream(self.parent_s.device)
            self.ev_fork.record(main)
            if accept_first:
                self._fork_accept(x)
        if self.paged:
            tree_verify_attn_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["prefix_len"],
                                   x.get("k_tree"), x.get("v_tree"), self.parent_s, x.get("num_nodes"), self.Dmax,
                                   out=self.out, workspace=self.attn_ws, status=self.status)
        else:
            tree_verify_attn(x["q"], x["k_cache"], x["v_cache"], x["prefix_len"], x.get("k_tree"), x.get("v_tree"),
                             self.parent_s, x.get("num_nodes"), self.Dmax, out=self.out, workspace=self.attn_ws,
                             status=self.status)
        if overlap and not accept_first:
            self._fork_accept(x)
        if self.fused:
            if self.paged:
                kc, vc, bt = x["k_pages"], x["v_pages"], x["block_table"]
            else:
                kc, vc, bt = x["k_cache"], x["v_cache"], None
            tree_accept_commit(x["logits"], x["tokens"], self.parent_s, kc, vc, x["prefix_len"], x["k_tree"],
                               x["v_tree"], x.get("num_nodes"), x.get("root_key"), self.Dmax, "path",
                               block_table=bt, history=self.history, history_len=self.history_len,
                               accept_len=self.accept_len, path=self.path, out_tokens=self.out_tokens,
                               workspace=self.acc_ws, status=self.status)
            return {"out": self.out, "accept_len": self.accept_len, "path": self.path,
                    "out_tokens": self.out_tokens, "status": self.status, "parent_s": self.parent_s}
        if self.schedule == "overlap":
            main.wait_event(self.ev_join)
        else:
            self._accept(x)
        mode = "path" if self.accept == "greedy" else "length"
        if self.paged:
            kv_commit_paged(x["k_pages"], x["v_pages"], x["block_table"], x["prefix_len"], x["k_tree"], x["v_tree"],
                            self.path, self.accept_len, x.get("num_nodes"), self.Dmax, mode, status=self.status)
        else:
            kv_commit(x["k_cache"], x["v_cache"], x["prefix_len"], x["k_tree"], x["v_tree"], self.path,
                      self.accept_len, x.get("num_nodes"), self.Dmax, mode, status=self.status)
        return {"out": self.out, "accept_len": self.accept_len, "path": self.path, "out_tokens": self.out_tokens,
                "status": self.status, "parent_s": self.parent_s}

    @staticmethod
    def for_inputs(x: dict, device="cuda", **kw) -> "VerifyStep":
        """Size a step for a device input dict as produced by ``to_device``."""
        B, Nmax, Hq, d = x["q"].shape
        Hkv = x["k_tree"].shape[2]
        paged = "k_pages" in x
        accept = "sample" if "z_p" in x else "greedy"
        V = x["z_p"].shape[2] if accept == "sample" else x["logits"].shape[2]
        return VerifyStep(B=B, Nmax=Nmax, Hq=Hq, Hkv=Hkv, d=d, Dmax=int(x["Dmax"]), V=V, dtype=x["q"].dtype,
                          Lmax=None if paged else x["k_cache"].shape[2], paged=paged,
                          block_size=x["k_pages"].shape[2] if paged else 16,
                          max_blocks=x["block_table"].shape[1] if paged else None, forest=bool(x.get("forest")),
                          accept=accept, K=(x["z_p"].shape[1] - 1) if accept == "sample" else 0, device=device,
                          T=float(x.get("T", 0.0)) if accept == "sample" else 0.0, **kw)


def to_device(inp: dict, device="cuda") -> dict:
    """Move a generated input dict (numpy; bf16 stored as uint16 bits) to device tensors."""
    import numpy as np
    w = inp.get("workload")
    bf16 = getattr(w, "dtype", "bf16") == "bf16"
    out = {}
    for k, v in inp.items():
        if isinstance(v, np.ndarray):
            if v.dtype == np.uint16:
                t = torch.from_numpy(v.view(np.int16)).to(device).view(torch.bfloat16)
            elif v.dtype == np.float32 and k in ("q", "k_tree", "v_tree", "k_cache", "v_cache", "k_pages", "v_pages",
                                                 "logits", "z_p", "z_q"):
                t = torch.from_numpy(v).to(device)
            elif v.dtype in (np.int32, np.int64) and k not in ("u",):
                t = torch.from_numpy(v.astype(np.int32)).to(device)
            else:
                t = torch.from_numpy(v).to(device)
            out[k] = t.contiguous()
        else:
            out[k] = v
    out["forest"] = bool(getattr(w, "forest", False))
    out["bf16"] = bf16
    return out
