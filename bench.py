"""Benchmark of the tree-verification hot path on B200.

One step = one pass of the verification path over one batch of the
Llama-3-8B-shaped workload (batch 1, 32 query / 8 kv heads, d = 128, bf16,
4096-token prefix, 64-node tree, vocabulary 128256, temperature 0.8):
tree-masked attention of the 64 nodes (tree_verify_attn) followed by the
speculative-sampling acceptance walk (tree_accept).  `value` is verified
tree tokens per second per layer over all ranks.  Inputs are synthetic
(seeded Gaussian activations and logits of those shapes).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--config llama3_8b|specexec70b|serving|longctx|longctx_sparse|tiny]

Timing: the step's calls are captured once into one CUDA graph (and each
call into a graph of its own); W untimed warm-up steps, then K steps of the
one-graph step, each preceded (outside the timed region) by a 256 MiB write
that flushes the 126 MB L2 and bracketed by CUDA events on the launching
stream (`ms_per_step`, `value`); then K steps of the per-call graphs with an
event between calls give the per-call durations (`calls`); the max over
ranks is reported.  The e2e figure calls
the Python API directly (no graph), copying the step's inputs from pinned
host memory and reading the accepted tokens back.  --impl reference times
the fp64 CPU oracle on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


TRAFFIC_PATH = os.path.join(ROOT, "profiles", "traffic.txt")
KERNEL_SOURCES = {
    "accept_node_kernel": "tree_verification_verify_b200/csrc/accept.cu",
    "attn_tc_kernel": "tree_verification_verify_b200/csrc/attn_tc.cu",
    "expand_rows_kernel": "tree_verification_verify_b200/csrc/expand.cu",
}


def measured_traffic(kernel, workload):
    """DRAM bytes per launch (read + write) of `kernel` on `workload` from the
    committed ncu summary, or None when there is none or the kernel's source
    has changed since the counters were taken (the summary records the
    source's sha1)."""
    import hashlib
    try:
        src = os.path.join(ROOT, KERNEL_SOURCES[kernel])
        sha = hashlib.sha1(open(src, "rb").read()).hexdigest()
        for line in open(TRAFFIC_PATH):
            f = line.split()
            if len(f) < 4 or f[0].startswith("#"):
                continue
            kv = dict(x.split("=", 1) for x in f[2:] if "=" in x)
            if f[0] == kernel and f[1] == workload and kv.get("source_sha1") == sha:
                return float(kv["dram_bytes_per_launch"])
    except Exception:
        return None
    return None


def peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


# --------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        if torch.cuda.is_available():
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------
# clocks
# --------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": []}
        if self.proc is None:
            return out
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm.append(float(f[1]))
                    smax.append(float(f[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, f[5:9]):
                    if v.lower() in ("active", "1", "0x1"):
                        reasons.add(nm)
            os.unlink(self.path)
        except Exception:
            pass
        if sm:
            out["sm_mhz"] = statistics.median(sm)
            out["sm_max_mhz"] = max(smax)
            out["samples"] = len(sm)
        out["reasons"] = sorted(reasons)
        return out


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------

class Step:
    """Device-resident inputs of one workload and the calls of one step.

    The SpecExec-shaped workload builds its 2048-node tree on the device in
    every step (16 best-first rounds of 128 from N(0, 4^2) draft logits over
    32000 tokens), then verifies it (attention over that tree) and accepts
    with SpecExec's rule at temperature 0.6."""

    def __init__(self, name, seed, dev):
        import tree_verification_verify_b200 as tv
        from synth import CONFIGS, config_attn_case, config_accept_case, config_expand_case, tree_depths
        self.tv = tv
        self.name = name
        base = "longctx" if name == "longctx_sparse" else name
        self.c = c = CONFIGS[base]
        self.sparse = name == "longctx_sparse"
        self.dev = dev
        self.expand = None
        self.attn = config_attn_case(base, seed=seed, device=dev, sparse=self.sparse)
        temp = c.get("temperature", c.get("temperatures", (0.0,))[-1])
        if base == "specexec70b":
            ec = config_expand_case(base, seed=seed)
            self.ec = ec
            self.exp_state = tv.tree_expand_init(ec.budget, ec.V, ec.Bsel, device=dev)
            calls = ec.n_calls()
            self.exp_logits = [ec.round_logits(k, 1 if k == 0 else ec.Bsel, device=dev) for k in range(calls)]
            self.exp_root = torch.zeros(1, dtype=torch.int32, device=dev)
            self.run_expand()
            torch.cuda.synchronize()
            par = self.exp_state.parent.view(1, -1)
            tok = self.exp_state.token.view(1, -1)
            self.attn.parent = par
            self.acc = config_accept_case(base, temperature=temp, seed=seed, device=dev,
                                          parents=[par[0].cpu().numpy()], mode="specexec")
            self.acc.parent = par
            self.acc.draft_tokens = tok
            self.acc.mode = "specexec"
            self.expand = True
        else:
            self.acc = config_accept_case(base, temperature=temp, seed=seed, device=dev,
                                          parents=[p.cpu().numpy() for p in self.attn.parent])
        self.temperature = temp
        B, T, Hq, d = self.attn.q.shape
        self.B, self.T = B, T
        self.out = torch.empty_like(self.attn.q)
        self.lse = torch.empty(B, T, Hq, dtype=torch.float32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.acc_out = dict(n_accepted=torch.empty(B, dtype=torch.int32, device=dev),
                            accepted_nodes=torch.empty(B, T, dtype=torch.int32, device=dev),
                            out_tokens=torch.empty(B, T + 1, dtype=torch.int32, device=dev),
                            min_margin=torch.empty(B, dtype=torch.float64, device=dev))
        # algorithmic work
        Hkv = self.attn.k_cache.shape[2]
        L = self.attn.prefix_len.cpu().numpy()
        par = self.attn.parent.cpu().numpy()
        keys = 0
        for b in range(B):
            dep = tree_depths(par[b])
            Lb = int(L[b])
            if self.sparse:
                nblk = (Lb + 63) // 64
                Lb = min(Lb, 32 * 64) if nblk > 32 else Lb
            keys += T * Lb + int(np.sum(dep + 1))
        elt = self.attn.q.element_size()
        self.attn_flops = 4.0 * d * Hq * keys
        self.attn_bytes = float(sum(int(x) + T for x in L)) * Hkv * d * 2 * elt
        V = self.acc.target_logits.shape[2]
        internal = 0
        if self.acc.draft_probs is not None:
            for b in range(B):
                internal += len(set(par[b][1:].tolist()))
        self.accept_bytes = float(B * T * V * 4 + internal * V * 4)
        self.expand_bytes = 0.0
        if self.expand:
            self.expand_bytes = float(sum(x.numel() for x in self.exp_logits) * 4)

    def run_expand(self):
        tv, st, ec = self.tv, self.exp_state, self.ec
        tv.tree_expand_init(ec.budget, ec.V, ec.Bsel, state=st)
        for k, z in enumerate(self.exp_logits):
            rows = self.exp_root if k == 0 else st.frontier
            tv.tree_expand_topb(st, z, rows)

    def run_attn(self):
        a = self.attn
        self.tv.tree_verify_attn(a.q, a.k_cache, a.v_cache, a.prefix_len, a.k_tree, a.v_tree, a.parent,
                                 n_nodes=a.n_nodes, sparse_topk=a.sparse_topk, block_size=a.block_size,
                                 out=self.out, lse=self.lse, dev_status=self.status)

    def run_accept(self):
        c = self.acc
        self.tv.tree_accept(c.target_logits, c.draft_tokens, c.parent, draft_probs=c.draft_probs,
                            mode=c.mode, temperature=self.temperature, seed=c.seed, step=0,
                            dev_status=self.status, outputs=self.acc_out)

    def launches_per_step(self):
        attn = self.attn_launches
        exp = (1 + 2 * len(self.exp_logits)) if self.expand else 0
        return attn + 1 + exp


def capture_graphs(step):
    """CUDA graphs of the calls of a step (captured once, replayed in the
    timed region so that no host launch overhead sits between kernels)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):                       # warm the library's host-side setup
            if step.expand:
                step.run_expand()
            step.run_attn()
            step.run_accept()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    step.attn_path = step.tv.last_attn_path
    step.attn_launches = step.tv.last_attn_launches
    # capture on the warm-up stream: the binding's per-stream workspace then
    # already exists and nothing is allocated (or zero-filled) in the graph
    graphs = {}
    calls = [(name, fn) for name, fn in (("expand", step.run_expand if step.expand else None),
                                         ("attn", step.run_attn), ("accept", step.run_accept)) if fn]
    for name, fn in calls:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            fn()
        graphs[name] = g
    # the whole step as one graph (how a caller launches it)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _, fn in calls:
            fn()
    graphs["step"] = g
    torch.cuda.synchronize()
    return graphs


def time_steps(step, K, W, world, flush):
    """K timed steps, each the one-graph step (`step`), then K steps of the
    per-call graphs with an event between calls (the per-call breakdown).
    Every step is preceded by the L2 flush, outside the timed region."""
    graphs = capture_graphs(step)
    names = [nm for nm in graphs if nm != "step"]
    s = torch.cuda.current_stream()
    for _ in range(W):
        flush.zero_()
        graphs["step"].replay()
        for nm in names:
            graphs[nm].replay()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(K)]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    for k in range(K):
        flush.zero_()
        evs[k][0].record(s)
        graphs["step"].replay()
        evs[k][1].record(s)
    torch.cuda.synchronize()
    barrier(world)
    for k in range(K):
        flush.zero_()
        ev[k][0].record(s)
        for j, nm in enumerate(names):
            graphs[nm].replay()
            ev[k][j + 1].record(s)
    torch.cuda.synchronize()
    times = {nm: [ev[k][j].elapsed_time(ev[k][j + 1]) for k in range(K)] for j, nm in enumerate(names)}
    times["step"] = [evs[k][0].elapsed_time(evs[k][1]) for k in range(K)]
    del graphs
    return times


def time_e2e(step, K, W, flush):
    """The same step through the public API from pinned host buffers: the
    step's inputs are copied host->device and the accepted tokens read
    back inside the timed region."""
    a, c = step.attn, step.acc
    dev_in = [a.q, a.k_cache, a.v_cache, a.prefix_len, a.k_tree, a.v_tree, c.target_logits]
    if step.expand:
        dev_in += step.exp_logits          # the tree itself is built on the device
    else:
        dev_in += [a.parent, c.draft_tokens]
    if c.draft_probs is not None:
        dev_in.append(c.draft_probs)
    host_in = [t.cpu().pin_memory() for t in dev_in]
    host_out = [torch.empty(step.acc_out[k].shape, dtype=step.acc_out[k].dtype).pin_memory()
                for k in ("n_accepted", "out_tokens")]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    s = torch.cuda.current_stream()

    def one():
        for d, h in zip(dev_in, host_in):
            d.copy_(h, non_blocking=True)
        if step.expand:
            step.run_expand()
        step.run_attn()
        step.run_accept()
        host_out[0].copy_(step.acc_out["n_accepted"], non_blocking=True)
        host_out[1].copy_(step.acc_out["out_tokens"], non_blocking=True)

    for _ in range(W):
        flush.zero_()
        one()
    torch.cuda.synchronize()
    tot = 0.0
    for _ in range(K):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        one()
        e1.record(s)
        e1.synchronize()
        tot += e0.elapsed_time(e1)
    return tot / K, h2d, d2h


def time_commit(step, K, W, flush):
    """tree_commit_kv on the step's accepted paths (the acceptance outputs of
    the last step), timed alone from a CUDA graph of its own: the K and V rows
    of each root and its accepted nodes are appended to a scratch cache of T
    rows per sequence (prefix_len set to 0 before every call, outside the
    timed region: where the rows land does not change the work).  Returns
    (ms per call, bytes moved per call: rows read plus rows written)."""
    a = step.attn
    B, T, Hkv, d = a.k_tree.shape
    kc = torch.zeros(B, T, Hkv, d, dtype=a.k_tree.dtype, device=step.dev)
    vc = torch.zeros_like(kc)
    pl = torch.zeros(B, dtype=torch.int32, device=step.dev)
    n_acc, acc = step.acc_out["n_accepted"], step.acc_out["accepted_nodes"]

    def one():
        step.tv.tree_commit_kv(kc, vc, pl, a.k_tree, a.v_tree, n_acc, acc, dev_status=step.status)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        pl.zero_()
        one()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        one()
    cur = torch.cuda.current_stream()
    for _ in range(W):
        flush.zero_()
        pl.zero_()
        g.replay()
    torch.cuda.synchronize()
    tot = 0.0
    for _ in range(K):
        flush.zero_()
        pl.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        g.replay()
        e1.record(cur)
        e1.synchronize()
        tot += e0.elapsed_time(e1)
    rows = int((n_acc.clamp(min=0) + 1).sum().item())
    moved = 2.0 * 2.0 * rows * Hkv * d * a.k_tree.element_size()
    del g
    return tot / K, moved


# --------------------------------------------------------------------------
# CPU baseline (the oracle, bounded sample)
# --------------------------------------------------------------------------

def cpu_baseline(step, budget_s=15.0):
    """Time the fp64 oracle on a bounded sample of the step: attention of a
    subset of nodes (all heads) plus the full acceptance walk; scaled to
    tokens per second of the whole step."""
    from oracle.attention import tree_verify_attn as o_attn
    from oracle.accept import tree_accept as o_accept
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    a = step.attn
    c = step.acc
    host = {k: getattr(a, k).cpu() for k in ("q", "k_cache", "v_cache", "prefix_len", "k_tree", "v_tree", "parent")}
    ch = dict(z=c.target_logits.cpu(), q=None if c.draft_probs is None else c.draft_probs.cpu(),
              tok=c.draft_tokens.cpu(), par=c.parent.cpu())
    t0 = time.perf_counter()
    o_accept(ch["z"], ch["q"], ch["tok"], ch["par"], mode=c.mode, temperature=step.temperature, seed=c.seed)
    t_acc = time.perf_counter() - t0
    t_exp, exp_note = 0.0, ""
    if step.expand:
        # expansion: the first calls of the build (all 16 take about as long
        # as each other past the first), scaled to the whole build
        from oracle.expand import ExpandState as OState, expand_call
        ec = step.ec
        ost = OState(ec.budget, ec.root_token)
        frontier = [0]
        n_calls, done_calls, t_e = len(step.exp_logits), 0, 0.0
        while done_calls < min(3, n_calls):
            z = step.exp_logits[done_calls].cpu().double().numpy()
            t0 = time.perf_counter()
            frontier = list(expand_call(ost, z[:len(frontier)] if done_calls else z[:1],
                                        np.asarray(frontier, np.int64), ec.Bsel))
            t_e += time.perf_counter() - t0
            done_calls += 1
        t_exp = t_e / done_calls * n_calls
        exp_note = f", plus {done_calls} of {n_calls} expansion rounds scaled to the build"
    B, T = step.B, step.T
    done = 0
    t_attn = 0.0
    order = [(b, i) for i in range(T) for b in range(B)]
    while done < len(order) and t_attn < budget_s:
        rows = {order[done]}
        t0 = time.perf_counter()
        o_attn(host["q"], host["k_cache"], host["v_cache"], host["prefix_len"], host["k_tree"],
               host["v_tree"], host["parent"], sparse_topk=a.sparse_topk, block_size=a.block_size, rows=rows)
        t_attn += time.perf_counter() - t0
        done += 1
    per_node = t_attn / done
    t_step = per_node * B * T + t_acc + t_exp
    return {"value": (B * T) / t_step, "unit": "tokens/s", "cores": int(cores), "kind": "oracle",
            "sample": f"attention of {done} of {B * T} nodes (all heads, fp64) scaled to the step, "
                      f"plus the full acceptance walk ({t_acc:.2f} s){exp_note}",
            "seconds": round(t_attn + t_acc + t_exp, 2)}


# --------------------------------------------------------------------------
# main
# --------------------------------------------------------------------------

METRIC = "verified tree tokens/s per layer"


def config_block(step, world):
    c = step.c
    return {"workload": f"{step.name}: B={c['B']} Hq={c['Hq']} Hkv={c['Hkv']} d={c['d']} {c['dtype']} "
                        f"prefix={c['L']} T={c['T']} V={c['V']} temp={step.temperature}"
                        + (" sparse top-32 blocks of 64" if step.sparse else ""),
            "tree_nodes_per_rank": step.B * step.T, "l2": "256 MiB flush before every timed step (not timed)",
            "launch": "each call replayed from a CUDA graph",
            "parallelism": f"replicas x{world}"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    step = Step(args.config, 0, dev)
    vals = []
    for k in range(args.warmup + args.steps):
        cb = cpu_baseline(step, budget_s=max(2.0, 60.0 / max(1, args.steps + args.warmup)))
        if k >= args.warmup:
            vals.append(cb)
    v = statistics.median([x["value"] for x in vals])
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * step.B * step.T / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_block(step, 1),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": vals[0]["cores"], "kind": "oracle",
                             "sample": vals[0]["sample"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="llama3_8b",
                    choices=["llama3_8b", "specexec70b", "serving", "longctx", "longctx_sparse", "tiny"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_setup(args.gpus)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    from tree_verification_verify_b200 import build
    build.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    step = Step(args.config, seed=rank, dev=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    clk = ClockSampler(local)
    clk.start()
    times = time_steps(step, args.steps, args.warmup, world, flush)
    clocks = clk.stop()
    ms_step = max_over_ranks(statistics.fmean(times["step"]), world)
    ms_calls = max_over_ranks(statistics.fmean([sum(ts) for ts in zip(*[times[nm] for nm in times if nm != "step"])]),
                              world)
    ms_attn = max_over_ranks(statistics.fmean(times["attn"]), world)
    ms_acc = max_over_ranks(statistics.fmean(times["accept"]), world)
    ms_exp = max_over_ranks(statistics.fmean(times["expand"]), world) if "expand" in times else 0.0
    e2e_ms, h2d, d2h = time_e2e(step, max(3, args.steps // 5), 3, flush)
    e2e_ms = max_over_ranks(e2e_ms, world)
    commit_ms, commit_bytes = time_commit(step, max(3, args.steps), 3, flush)
    commit_ms = max_over_ranks(commit_ms, world)
    tokens = step.B * step.T * world
    hbm, bf16, bf16_sus, src = peaks()
    # dominant call and its roofline
    attn_t = max(step.attn_bytes / (hbm * 1e9), step.attn_flops / (bf16 * 1e12))
    if ms_exp >= max(ms_acc, ms_attn):
        achieved = step.expand_bytes / (ms_exp * 1e-3) / 1e9
        roof = {"kernel": "tree_expand_topb (16 rounds: row + merge launches)", "bound": "hbm",
                "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                "traffic": None, "peak_source": src, "algorithmic_bytes": step.expand_bytes}
        tk = "expand_rows_kernel"
    elif ms_acc >= ms_attn:
        achieved = step.accept_bytes / (ms_acc * 1e-3) / 1e9
        roof = {"kernel": "accept_node_kernel (tree_accept: one launch)", "bound": "hbm",
                "achieved": round(achieved, 1),
                "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": None,
                "peak_source": src, "algorithmic_bytes": step.accept_bytes}
        tk = "accept_node_kernel"
    else:
        if step.attn_bytes / (hbm * 1e9) >= step.attn_flops / (bf16 * 1e12):
            achieved = step.attn_bytes / (ms_attn * 1e-3) / 1e9
            roof = {"kernel": "tree_verify_attn (all launches)", "bound": "hbm", "achieved": round(achieved, 1),
                    "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": None,
                    "peak_source": src, "algorithmic_bytes": step.attn_bytes}
            tk = "attn_tc_kernel"
        else:
            achieved = step.attn_flops / (ms_attn * 1e-3) / 1e12
            roof = {"kernel": "tree_verify_attn (all launches)", "bound": "tensor", "achieved": round(achieved, 2),
                    "peak": bf16, "unit": "TFLOP/s", "frac": round(achieved / bf16, 4), "traffic": None,
                    "peak_source": src, "algorithmic_flops": step.attn_flops}
            tk = "attn_tc_kernel"
    if tk == "attn_tc_kernel" and step.attn_path == 1:
        roof["kernel"] = "attn_tc_kernel (tree_verify_attn: one launch)"
    if step.attn_path != 1 and tk == "attn_tc_kernel":
        roof["kernel"] = "tree_verify_attn (all launches)"
    else:
        roof["traffic"] = measured_traffic(tk, step.name)
        roof["traffic_source"] = "profiles/traffic.txt (ncu dram__bytes_read.sum + dram__bytes_write.sum)"
    line = {
        "metric": METRIC, "value": tokens / (ms_step * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_block(step, world),
        "roofline": roof,
        "calls": {"tree_verify_attn_us": round(ms_attn * 1e3, 2), "tree_accept_us": round(ms_acc * 1e3, 2),
                  "attn_roofline_frac": round(attn_t / (ms_attn * 1e-3), 4),
                  "attn_tflops": round(step.attn_flops / (ms_attn * 1e-3) / 1e12, 2),
                  "accept_gbs": round(step.accept_bytes / (ms_acc * 1e-3) / 1e9, 1),
                  "accept_nodes_per_s": step.B * step.T / (ms_acc * 1e-3)},
        "launches_per_step": step.launches_per_step(),
        "ms_per_step_call_by_call": round(ms_calls, 5),
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": step.launches_per_step() * args.steps,
        "clocks": clocks,
    }
    # the KV commit of the accepted paths (not part of the timed step)
    line["calls"]["tree_commit_kv_us"] = round(commit_ms * 1e3, 2)
    line["calls"]["commit_bytes"] = commit_bytes
    line["calls"]["commit_gbs"] = round(commit_bytes / (commit_ms * 1e-3) / 1e9, 1)
    if step.expand:
        line["calls"]["tree_expand_us"] = round(ms_exp * 1e3, 2)
        line["calls"]["expand_gbs"] = round(step.expand_bytes / (ms_exp * 1e-3) / 1e9, 1)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(step)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
