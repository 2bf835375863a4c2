"""Benchmark of one tree-verify step on B200: prints ONE JSON line (rank 0).

A step is the whole hot path over one batch: tree_prepare -> tree_verify_attn (+ split merge)
-> acceptance (greedy tree, or chain rejection sampling) -> kv_commit.  Metric: verified tree
tokens per second (sum of tree nodes over the timed steps / device time), with the attention
call's achieved HBM bandwidth against the measured copy bandwidth as the roofline figure.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

The headline line is the chain5 workload (the largest: 2.16 GB of attention K/V per step).  With
no --workload at one GPU, the same measurement is also taken on the other four workloads and
reported under "per_workload" (value, ms per step, roofline, e2e of each); --workload NAME
measures that workload alone.

Multi-GPU (torchrun): every rank verifies its own batch (its own seeded sequences), no
collective on the data path; the timed region is bracketed by a barrier and a synchronize, the
time is the max over ranks, value = tokens of all ranks / that time ("weak" scaling).
`--impl reference` times the fp64 CPU oracle on host cores on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
DEFAULT_WORKLOAD = "chain5"
ALL_WORKLOADS = ("tiny", "tree26", "eagle60", "chain5", "forest")
DESCR = {
    "tiny": "B=1 Hq=8 Hkv=2 d=64 fp32, L=128, 8-node tree, V=256",
    "tree26": "Llama-3-8B-shaped verify: B=1 Hq=32 Hkv=8 d=128 bf16, L=2048, static EAGLE tree N=26 "
              "(4,3,2,1,1,1), V=128256, greedy, contiguous cache",
    "eagle60": "B=16 Hq=32 Hkv=8 d=128 bf16, ragged L in [1024,8192], EAGLE-2 trees N=60, V=128256, "
               "greedy, paged cache (block 16)",
    "chain5": "70B-shaped chain: B=64 Hq=64 Hkv=8 d=128 bf16, L=8192, K=5, T=1 rejection sampling, V=128256",
    "forest": "SSD forest: B=8 x 8 subtrees x 64 nodes, L=32768, Hq=32 Hkv=8 d=128 bf16, V=128256, greedy, "
              "paged cache (block 16)",
}


METRIC = "verified tree tokens/s (whole verify step: prepare + tree attention + acceptance + commit)"


def attn_algorithmic_bytes(inp) -> int:
    """Bytes a tree_verify_attn launch must move at minimum: prefix K+V once per (sequence, KV
    head), tree K+V, Q read and O written."""
    q = inp["q"]
    B, N, Hq, d = q.shape
    Hkv = inp["k_tree"].shape[2]
    es = 2 if q.dtype == np.uint16 else 4
    total = 0
    for b in range(B):
        L, n = int(inp["prefix_len"][b]), int(inp["num_nodes"][b])
        total += Hkv * (L + n) * d * es * 2 + n * Hq * d * es * 2
    return total


def attn_algorithmic_flops(inp) -> int:
    """Multiply-add flops a tree_verify_attn launch must do: every query row (node, head) takes a
    dot product with, and a weighted sum of, each key it sees -- the prefix plus its own root->node
    path -- at 2 flops per multiply-add and d per dot product: 4 d flops per (row, key)."""
    q = inp["q"]
    B, N, Hq, d = q.shape
    total = 0
    for b in range(B):
        L, n = int(inp["prefix_len"][b]), int(inp["num_nodes"][b])
        par = inp["parent"][b]
        depth = np.zeros(n, np.int64)
        for i in range(n):
            depth[i] = depth[par[i]] + 1 if par[i] >= 0 else 0
        total += 4 * d * Hq * int((L + depth + 1).sum())
    return total


def tokens_per_step(inp) -> int:
    return int(np.asarray(inp["num_nodes"]).sum())


def rank_workload(name: str, rank: int, batch: int = 0):
    """The workload one rank verifies: the named shape with its own seed (weak scaling: every rank
    owns a full batch of its own sequences; no data moves between ranks)."""
    w = W.WORKLOADS[name]
    if batch:
        w = w.scaled(B=batch)
    return w, w.seed + 1000 * rank


def reduce_over_ranks(values, world: int, device=None):
    """Max over ranks of per-rank device times (ms): the slowest rank bounds the step."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def aggregate_rate(tokens_per_rank_step: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the tokens every rank verified over the max-over-ranks time."""
    return world * tokens_per_rank_step * steps / (max_ms * 1e-3)


def _peaks_file():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f)
    return {}


def read_tensor_peak():
    """Dense bf16 TFLOP/s: the measured burst cuBLAS figure (the attention graph times one kernel
    back to back for well under a second), else the profiling recipe's fallback."""
    j = _peaks_file()
    if "bf16_tflops" in j:
        return float(j["bf16_tflops"]), "measured bf16_tflops (cuBLAS, burst)"
    return 1590.0, "fallback bf16 (burst)"


def read_tensor_peak_sustained():
    """Dense bf16 TFLOP/s sustained under the power cap (seconds-long cuBLAS loop)."""
    j = _peaks_file()
    if "bf16_tflops_sustained" in j:
        return float(j["bf16_tflops_sustained"]), "measured bf16_tflops_sustained"
    return 1400.0, "fallback bf16 (sustained)"


def read_peaks():
    j = _peaks_file()
    if "hbm_gbs" in j:
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def attn_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("attn.cu", "attn_umma.cu", "attn_common.cuh", "umma.cuh", "common.cuh", "kernels.h"):
        with open(os.path.join(ROOT, "tree_speculative_decoding_06_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """Per-launch DRAM bytes of the attention call from a committed ncu summary, if it was taken
    on the current attention source (profiles/attn_traffic.txt: workload source_hash bytes)."""
    p = os.path.join(ROOT, "profiles", "attn_traffic.txt")
    if not os.path.exists(p):
        return None
    cur = attn_source_hash()
    for ln in open(p):
        parts = ln.split()
        if len(parts) == 3 and not ln.startswith("#") and parts[0] == workload and parts[1] == cur:
            return float(parts[2])
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = "clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown," \
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown," \
             "clocks_event_reasons.sw_power_cap"

    def __init__(self, gpu_id: str):
        self.gpu_id, self.proc, self.lines = gpu_id, None, []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- our arm
def _roofline(inp, attn_ms, workload):
    """Roofline of the attention call: its bound is whichever floor is higher, the algorithmic
    bytes at the measured copy bandwidth or the algorithmic flops at the dense bf16 rate; both
    fractions are reported, the tensor one against the burst and the sustained bf16 figures."""
    peak, peak_kind = read_peaks()
    tpeak, tpeak_kind = read_tensor_peak()
    spk, spk_kind = read_tensor_peak_sustained()
    alg = attn_algorithmic_bytes(inp)
    flops = attn_algorithmic_flops(inp)
    sec = attn_ms * 1e-3
    tensor_bound = flops / (tpeak * 1e12) > alg / (peak * 1e9)
    if tensor_bound:
        roof = {"bound": "tensor", "achieved": round(flops / sec / 1e12, 1), "peak": tpeak, "unit": "TFLOP/s"}
        roof["frac"] = round(roof["achieved"] / tpeak, 4)
        roof["peak_kind"] = tpeak_kind + " (of measured)" if "measured" in tpeak_kind else tpeak_kind
    else:
        achieved = alg / sec / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_kind": f"{peak_kind} hbm_gbs (copy, burst)"}
    roof.update({"traffic": recorded_traffic(workload), "kernel": "tsd_tree_verify_attn",
                 "algorithmic_bytes_per_launch": alg, "algorithmic_flops_per_launch": flops,
                 "attn_us_per_launch": round(attn_ms * 1e3, 3),
                 "hbm_frac": round(alg / sec / 1e9 / peak, 4),
                 "tensor_frac": round(flops / sec / 1e12 / tpeak, 4),
                 "tensor_frac_sustained": round(flops / sec / 1e12 / spk, 4),
                 "tensor_peak_sustained": spk})
    return roof


def measure(name, args, rank, world, dev, gpu_id):
    """One workload: K whole steps captured into one CUDA graph and timed with CUDA events (max over
    ranks), the attention call alone the same way, and the e2e figure through the public API with
    host buffers.  Returns (fields of the JSON line, the generated inputs)."""
    import torch
    import torch.distributed as dist

    import tree_speculative_decoding_06_b200 as tsd
    from tree_speculative_decoding_06_b200.step import VerifyStep, to_device

    w, seed = rank_workload(name, rank, args.batch)
    inp = W.make_inputs(w, seed=seed, nan_guard=False)
    tok = tokens_per_step(inp)
    x0 = to_device(inp, dev)
    per_set = sum(v.numel() * v.element_size() for v in x0.values() if isinstance(v, torch.Tensor))
    nsets = 1 if per_set > 2 * L2_BYTES else max(2, math.ceil(2.5 * L2_BYTES / per_set))
    sets = [x0] + [{k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in x0.items()}
                   for _ in range(nsets - 1)]
    pl0 = [s["prefix_len"].clone() for s in sets]
    steps = [VerifyStep.for_inputs(s, dev) for s in sets]
    stream = torch.cuda.Stream(dev)

    def one_step(i):
        s = i % nsets
        sets[s]["prefix_len"].copy_(pl0[s], non_blocking=True)   # every step verifies the same batch
        steps[s].run(sets[s])

    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            one_step(i)
    torch.cuda.synchronize(dev)

    # The timed K steps are captured into ONE CUDA graph (step i on input set i % nsets), so the
    # device runs them back to back with no per-step host launch cost; likewise K attention calls.
    def attn_call(s):
        x, st = sets[s], steps[s]
        if st.paged:
            tsd.tree_verify_attn_paged(x["q"], x["k_pages"], x["v_pages"], x["block_table"], x["prefix_len"],
                                       x["k_tree"], x["v_tree"], st.parent_s, x["num_nodes"], st.Dmax,
                                       out=st.out, workspace=st.attn_ws, status=st.status)
        else:
            tsd.tree_verify_attn(x["q"], x["k_cache"], x["v_cache"], x["prefix_len"], x["k_tree"], x["v_tree"],
                                 st.parent_s, x["num_nodes"], st.Dmax, out=st.out, workspace=st.attn_ws,
                                 status=st.status)

    n_attn = args.steps
    g_steps, g_attn = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_steps, stream=stream):
        for i in range(args.steps):
            one_step(i)
    with torch.cuda.graph(g_attn, stream=stream):
        for i in range(n_attn):
            attn_call(i % nsets)
    with torch.cuda.stream(stream):       # untimed pass of both graphs
        g_steps.replay()
        g_attn.replay()
    torch.cuda.synchronize(dev)

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(gpu_id) as clocks:
        t_wall = time.perf_counter()
        with torch.cuda.stream(stream):
            ev0.record(stream)
            g_steps.replay()
            ev1.record(stream)
        torch.cuda.synchronize(dev)
        step_ms = ev0.elapsed_time(ev1)
        # the attention call alone over the same rotating inputs (its average launch duration)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a0.record(stream)
            g_attn.replay()
            a1.record(stream)
        torch.cuda.synchronize(dev)
        attn_ms = a0.elapsed_time(a1) / n_attn
        wall = time.perf_counter() - t_wall
    if world > 1:
        dist.barrier()
    step_ms, attn_ms = reduce_over_ranks([step_ms, attn_ms], world, dev)
    bad = sum(int((st.status != 0).sum()) for st in steps)   # every sequence of every set must be clean

    # end to end through the public API with host buffers: every step copies its inputs from pinned
    # host memory (H2D), runs, and reads back the accepted lengths / tokens / path (D2H).  Two
    # input buffers (the inputs only; the cache and prefix lengths are shared) and a copy stream
    # let step i+1's H2D run while step i computes, as a serving loop would.
    from tree_speculative_decoding_06_b200.step import VerifyStep as _VS
    keys_in = [k for k in ("q", "k_tree", "v_tree", "parent", "num_nodes", "tokens", "logits", "root_key", "z_p",
                           "z_q", "x", "u") if isinstance(x0.get(k), torch.Tensor)]
    host = {k: x0[k].cpu().pin_memory() for k in keys_in}
    bufs = [sets[0], {**sets[0], **{k: sets[0][k].clone() for k in keys_in}}]
    vsteps = [steps[0], _VS.for_inputs(bufs[1], dev)]
    outs = ["accept_len", "out_tokens"] + (["path"] if steps[0].path is not None else [])
    host_outs = [{k: getattr(vs, k).cpu().pin_memory() for k in outs} for vs in vsteps]
    h2d = sum(host[k].numel() * host[k].element_size() for k in keys_in)
    d2h = sum(host_outs[0][k].numel() * host_outs[0][k].element_size() for k in outs)
    e_steps = max(10, min(args.steps, 200))
    copy_stream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    done = [torch.cuda.Event(), torch.cuda.Event()]

    def e2e_step(i):
        j = i % 2
        copy_stream.wait_event(done[j])          # step i-2 has finished with buffer j
        with torch.cuda.stream(copy_stream):
            for k in keys_in:
                bufs[j][k].copy_(host[k], non_blocking=True)
            copied[j].record(copy_stream)
        stream.wait_event(copied[j])
        with torch.cuda.stream(stream):
            bufs[j]["prefix_len"].copy_(pl0[0], non_blocking=True)
            vsteps[j].run(bufs[j])
            for k in outs:
                host_outs[j][k].copy_(getattr(vsteps[j], k), non_blocking=True)
            done[j].record(stream)

    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_stream.wait_event(e0)
    for i in range(e_steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e_ms = reduce_over_ranks([e0.elapsed_time(e1) / e_steps], world, dev)[0]

    # launches of our kernels: per step (prepare, attention (+ merge), acceptance, commit), plus the
    # attention-only graph
    per_step = steps[0].launches_per_step()
    launches = per_step * args.steps + steps[0].attn_launches() * n_attn
    fields = {
        "value": round(aggregate_rate(tok, world, args.steps, step_ms), 1),
        "ms_per_step": round(step_ms / args.steps, 6),
        "dtype": "bf16" if inp["q"].dtype == np.uint16 else "f32",
        "config": {"workload": f"{name}: {DESCR[name]}" +
                               (f" [batch overridden to {args.batch}]" if args.batch else ""),
                   "tokens_per_step_per_gpu": tok,
                   "l2": (f"rotating {nsets} input sets ({nsets * per_set / 2**20:.0f} MiB > 2x L2)"
                          if nsets > 1 else f"inputs {per_set / 2**20:.0f} MiB > L2"),
                   "graphs": "the K timed steps replayed as one CUDA graph",
                   "parallelism": f"replicas over sequences x{world}"},
        "roofline": _roofline(inp, attn_ms, name) if rank == 0 else None,
        "e2e": {"value": round(aggregate_rate(tok, world, 1, e_ms), 1), "unit": "tokens/s",
                "copies": "every step: H2D of its inputs from pinned memory, D2H of its results; the next "
                          "step's H2D overlaps this step's compute (two input buffers)",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms, 4)},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
        "status_errors": bad,
        "wall_s_timed": round(wall, 3),
    }
    del g_steps, g_attn, sets, steps, x0, host, host_outs, bufs, vsteps
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return fields, inp


def measure_extras(args, dev):
    """The kernels beyond the verify step, each at its natural shape, timed as one CUDA graph of K
    calls (CUDA events on the launching stream; inputs seeded, drawn on the device): the EAGLE-2
    draft-tree expansion (B=16, F=K=10), stochastic multi-branch and threshold acceptance over the
    eagle60 trees (B=16, N=60), and the SSD outcome-cache build (B=8, K=7 drafts, S=8 slots); all
    over V=128256 bf16 logits.  Each reports microseconds per call and its algorithmic bytes
    (the logits rows the call must read) as a fraction of the copy bandwidth."""
    import torch

    import tree_speculative_decoding_06_b200 as tsd
    peak, peak_kind = read_peaks()
    V = 128256
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)

    def randn(*shape, sigma=1.0):
        return (torch.randn(*shape, generator=gen, device=dev) * sigma).to(torch.bfloat16)

    stream = torch.cuda.Stream(dev)

    def timed(fn, n):
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(n):
                fn()
        with torch.cuda.stream(stream):
            g.replay()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / n

    def entry(ms, nbytes, what):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"us_per_call": round(ms * 1e3, 3), "algorithmic_bytes": int(nbytes), "achieved_gbs": round(gbs, 1),
                "hbm_frac": round(gbs / peak, 4), "peak_kind": f"{peak_kind} hbm_gbs", "shape": what}

    n = max(args.steps, 10)
    out = {}
    # draft tree expansion: capacity for every expansion the timing runs, so none overflows
    B, F, K = 16, 10, 10
    dt = tsd.DraftTree(B, F, 1 + (n + 4) * F * K, device=dev)
    dlog = randn(B, F, V, sigma=3.0)
    dt.init(torch.randint(0, V, (B,), device=dev, dtype=torch.int32, generator=gen))
    ms = timed(lambda: dt.expand(dlog, K, stream=stream), n)
    out["draft_tree_expand"] = entry(ms, B * F * V * 2, "B=16 F=10 K=10 V=128256 bf16")
    # stochastic and threshold acceptance over the eagle60 trees
    w = W.WORKLOADS["eagle60"].scaled(L=16, L_lo=8, V=256)
    base = W.make_inputs(w, nan_guard=False)
    N = base["parent"].shape[1]
    parent = torch.from_numpy(base["parent"]).to(dev)
    nn = torch.from_numpy(base["num_nodes"]).to(dev)
    prep = tsd.tree_prepare(parent, nn, int(base["Dmax"]), False)
    zp, zq = randn(w.B, N, V, sigma=2.0), None
    zq = (zp.float() + torch.randn(w.B, N, V, generator=gen, device=dev) * 0.8).to(torch.bfloat16)
    toks = torch.randint(0, V, (w.B, N), device=dev, dtype=torch.int32, generator=gen)
    u = torch.rand(w.B, N, device=dev, generator=gen)
    res = {}

    def sample():
        res["s"] = tsd.tree_accept_sample(zp, zq, toks, prep["parent_s"], u, 1.0, num_nodes=nn, Dmax=int(base["Dmax"]),
                                          status=prep["status"], stream=stream)
    ms = timed(sample, n)
    A = res["s"]["accept_len"].cpu().numpy()
    out["tree_accept_sample"] = entry(ms, int((A + 1).sum()) * 2 * V * 2,
                                      "eagle60 trees B=16 N=60 V=128256 bf16 T=1 (bytes: the two rows of every "
                                      "visited node)")
    ms = timed(lambda: tsd.tree_accept_threshold(zp, toks, prep["parent_s"], 0.01, 1.0, num_nodes=nn,
                                                 Dmax=int(base["Dmax"]), status=prep["status"], stream=stream), n)
    out["tree_accept_threshold"] = entry(ms, w.B * N * V * 2, "eagle60 trees B=16 N=60 V=128256 bf16 tau=0.01")
    # SSD outcome cache
    Bs, Ks, S = 8, 7, 8
    sl = randn(Bs, Ks + 1, V, sigma=3.0)
    alpha = torch.rand(Bs, device=dev, generator=gen) * 0.5 + 0.4
    us = torch.rand(Bs, Ks, device=dev, generator=gen)
    ms = timed(lambda: tsd.ssd_cache_build(sl, alpha, 0.5, us, S, 1.0, stream=stream), n)
    out["ssd_cache_build"] = entry(ms, Bs * (Ks + 1) * V * 2, "B=8 K=7 S=8 V=128256 bf16")
    torch.cuda.synchronize(dev)
    return out


def run_ours(args, rank, world, local_rank):
    import torch

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    gpu_id = os.environ.get("CUDA_VISIBLE_DEVICES", str(local_rank)).split(",")[local_rank] \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else str(local_rank)
    head = args.workload or DEFAULT_WORKLOAD
    fields, inp = measure(head, args, rank, world, dev, gpu_id)
    res = None
    if rank == 0:
        res = {"metric": METRIC, "value": fields["value"], "unit": "tokens/s", "n_gpus": world,
               "steps": args.steps, "warmup": args.warmup, "ms_per_step": fields["ms_per_step"],
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": fields["dtype"],
               "data": "synthetic (seeded; workloads module)"}
        res.update({k: fields[k] for k in ("config", "roofline", "e2e", "gpu_launches", "clocks", "status_errors",
                                           "wall_s_timed")})
    # every other workload at one GPU when none was named: same measurement, reported per workload
    if args.workload is None and world == 1:
        per = {}
        for name in ALL_WORKLOADS:
            if name == head:
                continue
            f, _ = measure(name, args, rank, world, dev, gpu_id)
            per[name] = {k: f[k] for k in ("value", "ms_per_step", "dtype", "roofline", "e2e", "gpu_launches",
                                           "clocks", "status_errors")}
            per[name]["unit"] = "tokens/s"
            per[name]["workload"] = f["config"]["workload"]
            res["gpu_launches"] += f["gpu_launches"]
        res["per_workload"] = per
        res["next_kernels"] = measure_extras(args, dev)
    return res, inp


# ----------------------------------------------------------------------------- oracle arms
def oracle_sample(inp, budget_s: float, max_rows: int = 256, seed: int = 0):
    """Time the oracle on a bounded sample of the workload.  One sample = one sequence b: its
    acceptance and commit in full, and its attention on at most `max_rows` (node, head) rows drawn
    at random, the attention time scaled to all the sequence's rows (linear in rows).  Samples are
    taken until `budget_s` is spent.  Returns (tokens/s, description, seconds spent)."""
    import oracle
    w = inp["workload"]
    B = inp["parent"].shape[0]
    Hq = inp["q"].shape[2]
    rng = np.random.default_rng(seed)
    t_all, toks, nseq, rows_done, rows_total = 0.0, 0, 0, 0, 0
    t0 = time.perf_counter()
    while nseq == 0 or time.perf_counter() - t0 < budget_s:
        b = nseq % B
        sub = {k: (v[b:b + 1] if isinstance(v, np.ndarray) and v.ndim >= 1 and v.shape[0] == B and k not in
                   ("k_pages", "v_pages") else v) for k, v in inp.items()}
        N = int(inp["num_nodes"][b])
        rows = [(0, i, h) for i in range(N) for h in range(Hq)]
        if len(rows) > max_rows:
            rows = [rows[j] for j in sorted(rng.choice(len(rows), size=max_rows, replace=False))]
        ta = time.perf_counter()
        oracle.attention_rows(sub, rows)
        tb = time.perf_counter()
        if w.accept == "greedy":
            acc = oracle.accept_greedy(sub)
            oracle.kv_commit(sub, acc["accept_len"], acc["path"], "path")
        else:
            acc = oracle.chain_sample(sub["z_p"], sub["z_q"], sub["x"], sub["u"], sub["T"])
            oracle.kv_commit(sub, acc["accept_len"], None, "length")
        tc = time.perf_counter()
        t_all += (tb - ta) * (N * Hq / len(rows)) + (tc - tb)
        toks += N
        rows_done += len(rows)
        rows_total += N * Hq
        nseq += 1
        if nseq >= 200:
            break
    spent = time.perf_counter() - t0
    frac = rows_done / max(rows_total, 1)
    desc = (f"{nseq} sequence(s) of {w.name}: acceptance + commit in full, attention on "
            f"{rows_done} of {rows_total} rows" + (" (scaled to all rows)" if frac < 1 else ""))
    return toks / t_all, desc, spent


def run_reference(args, rank):
    if rank != 0:
        return None
    import oracle
    oracle.build()
    name = args.workload or DEFAULT_WORKLOAD
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, nan_guard=False)
    for _ in range(max(args.warmup, 0)):
        oracle_sample(inp, 0.0)
    rates, secs = [], 0.0
    for _ in range(args.steps):
        r, desc, dt = oracle_sample(inp, 0.0)
        rates.append(r)
        secs += dt
    value = float(np.mean(rates))
    step_tokens = tokens_per_step(inp)
    cb = {"value": round(value, 2), "unit": "tokens/s", "cores": 1, "kind": "oracle", "host_cores": os.cpu_count(),
          "sample": f"per step: {desc}; {args.steps} steps, {secs:.1f} s"}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 2),
            "unit": "tokens/s", "n_gpus": args.gpus, "ran_on": "one host core of rank 0 (the fp64 oracle)",
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(step_tokens / value * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; workloads module)",
            "config": {"workload": f"{name}: {DESCR[name]}", "tokens_per_step_per_gpu": step_tokens},
            "cpu_baseline": cb,
            "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=None, choices=sorted(W.WORKLOADS),
                    help="measure this workload alone (default: the chain5 headline plus, at one GPU, every "
                         "other workload under per_workload)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--next-only", action="store_true",
                    help="measure only the kernels beyond the verify step (draft tree, tree sampling, threshold, "
                         "SSD cache) and print them (profiling runs)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch size (small profiling captures only; the bench line "
                         "of a workload uses its own size)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank)
        if res is not None:
            print(json.dumps(res))
        return
    if args.next_only:
        import torch
        torch.cuda.set_device(local_rank)
        print(json.dumps({"next_kernels": measure_extras(args, torch.device("cuda", local_rank))}))
        return

    import datetime

    import torch.distributed as dist
    if world > 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=__import__("torch").device("cuda", local_rank))
    try:
        res, inp = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1:   # the oracle baseline is timed at one GPU only
                v, desc, dt = oracle_sample(inp, args.cpu_budget)
                res["cpu_baseline"] = {"value": round(v, 2), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                       "host_cores": os.cpu_count(),
                                       "sample": f"{desc}; {dt:.1f} s, single-threaded C fp64"}
                res["speedup_vs_cpu_baseline"] = round(res["value"] / v, 1)
            print(json.dumps(res))
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
