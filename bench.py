"""Benchmark of the tree-verification hot path on B200.

Default workload: the long-context configuration, the largest one that fits a
single GPU -- batch 4, 32 query / 8 kv heads, d = 128, bf16, a 131072-token
prefix per sequence, a 256-node draft tree, vocabulary 128256, temperature 0.
One step = tree-masked attention of the 4 x 256 nodes over prefix and
ancestors (tree_verify_attn, dense) followed by the greedy acceptance walk
(tree_accept).  `value` is verified tree tokens per second per layer over all
ranks.  Inputs are synthetic (seeded Gaussian activations and logits of those
shapes).

The same run then times the other named workloads, each as its own step, and
reports them under "configs" in the same JSON line: block top-k long context
(the sparse path), the SpecExec-shaped 2048-node tree (16 rounds of
tree_expand_topb build it on the device, then attention and SpecExec
acceptance), batched serving (32 sequences) and the Llama-3-8B layer.  Every
call carries its roofline fraction against the measured peaks and against
the 8 TB/s / 2.25 PFLOP/s denominators.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--config longctx|longctx_sparse|specexec70b|serving|llama3_8b|tiny]
                    [--only] [--no-cpu-baseline] [--split-prefix | --iteration]

--iteration replays one whole speculative iteration (tree expansion with a
random-weight drafter stand-in, a random-weight target layer and
tree_verify_attn, tree_accept, tree_commit_kv) from a single CUDA graph.

--split-prefix times the long-context attention with each sequence's prefix
split across the N ranks (prefix-only partials, NCCL all-gather, the
log-sum-exp merge kernel): strong scaling of one layer's verification.

Timing: the step's calls are captured once into one CUDA graph (and each
call into a graph of its own); W untimed warm-up steps, then K steps of the
one-graph step, each preceded (outside the timed region) by a 256 MiB write
that flushes the 126 MB L2 and bracketed by CUDA events on the launching
stream (`ms_per_step`, `value`); then K steps of the per-call graphs with an
event between calls give the per-call durations; the max over ranks is
reported.  The e2e figure calls the Python API directly (no graph), copying
the step's inputs from pinned host memory and reading the accepted tokens
back.  --impl reference times the fp64 CPU oracle on a bounded sample of the
same workload, spread over the host cores by a process pool.
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
# the denominators the targets are stated against: 8 TB/s HBM and the B200
# dense bf16 datasheet peak
TARGET_HBM_GBS = 8000.0
TARGET_BF16_TFLOPS = 2250.0

CONFIG_NAMES = ["longctx", "longctx_sparse", "specexec70b", "serving", "llama3_8b", "tiny"]
# the workloads a default run times after its main one
EXTRA_CONFIGS = ["longctx_sparse", "specexec70b", "serving", "llama3_8b"]

TRAFFIC_PATH = os.path.join(ROOT, "profiles", "traffic.txt")
KERNEL_SOURCES = {
    "accept_node_kernel": "tree_verification_verify_b200/csrc/accept.cu",
    "attn_tc_kernel": "tree_verification_verify_b200/csrc/attn_tc.cu",
    "attn_pair_kernel": "tree_verification_verify_b200/csrc/attn_pair.cu",
    "expand_round_kernel": "tree_verification_verify_b200/csrc/expand.cu",
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


def roofline_fracs(seconds, nbytes=0.0, flops=0.0):
    """Roofline fraction of one call: (the slower of bytes / HBM bandwidth and
    FLOPs / bf16 peak) / measured time, against the measured peaks and
    against the 8 TB/s / 2.25 PFLOP/s denominators."""
    hbm, bf16, _, _ = peaks()
    out = {}
    for key, bw, pk in (("frac_measured", hbm, bf16), ("frac_target", TARGET_HBM_GBS, TARGET_BF16_TFLOPS)):
        t = max(nbytes / (bw * 1e9), flops / (pk * 1e12))
        out[key] = round(t / seconds, 4) if seconds > 0 else None
    return out


def accept_work(parents, T, V, with_draft_probs):
    """Algorithmic bytes of one tree_accept call: every node's target row
    (V fp32 values) and, when draft probabilities are given, the draft row
    of every node that has children (the rows its children were drawn
    from)."""
    internal = 0
    if with_draft_probs:
        for par in parents:
            internal += len(set(int(x) for x in list(par)[1:T] if x >= 0))
    return float(len(parents) * T * V * 4 + internal * V * 4)


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
# algorithmic work
# --------------------------------------------------------------------------

def attn_work(parents, prefix_lens, T, Hq, Hkv, d, elt, kept_keys=None, union_blocks=None,
              block_size=64, means_in_call=False):
    """Algorithmic FLOPs and bytes of one tree_verify_attn call.

    FLOPs = 4 d Hq sum_i |K(i)| (QK^T and PV), |K(i)| = prefix keys (dense) or
    kept keys (block top-k, per kv head) plus the root path.  Bytes = every
    K/V element read once: the prefix (dense) or, for block top-k, the union
    over a sequence's nodes of the kept blocks per kv head, plus one K read
    for the block means when they are computed in the call; and the tree
    K/V rows."""
    from synth import tree_depths
    B = len(prefix_lens)
    G = Hq // Hkv
    path = 0
    for b in range(B):
        path += int(np.sum(tree_depths(np.asarray(parents[b])) + 1))
    tree_bytes = float(B * T) * Hkv * d * 2 * elt
    if kept_keys is None:
        keys = sum(T * int(L) for L in prefix_lens)
        flops = 4.0 * d * Hq * (keys + path)
        nbytes = float(sum(int(L) for L in prefix_lens)) * Hkv * d * 2 * elt + tree_bytes
    else:
        # kept_keys: total kept prefix keys over (b, node, kv head)
        flops = 4.0 * d * G * kept_keys + 4.0 * d * Hq * path
        nbytes = float(union_blocks) * block_size * d * 2 * elt + tree_bytes
        if means_in_call:
            nbytes += float(sum(int(L) for L in prefix_lens)) * Hkv * d * elt
    return flops, nbytes


# --------------------------------------------------------------------------
# workloads (device side: the library path)
# --------------------------------------------------------------------------

class Step:
    """Device-resident inputs of one workload and the calls of one step.

    The SpecExec-shaped workload builds its 2048-node tree on the device in
    every step (16 best-first rounds of 128 from N(0, 4^2) draft logits over
    32000 tokens), then verifies it (attention over that tree) and accepts
    with SpecExec's rule at temperature 0.6."""

    def __init__(self, name, seed, dev):
        import tree_verification_verify_b200 as tv
        from synth import CONFIGS, config_attn_case, config_accept_case, config_expand_case
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
        L = [int(x) for x in self.attn.prefix_len.cpu().numpy()]
        par = self.attn.parent.cpu().numpy()
        elt = self.attn.q.element_size()
        self.union_blocks = None
        if self.sparse:
            kept, union = self.measure_selection()
            self.union_blocks = union
            self.attn_flops, self.attn_bytes = attn_work(par, L, T, Hq, Hkv, d, elt, kept_keys=kept,
                                                         union_blocks=union, block_size=self.attn.block_size,
                                                         means_in_call=True)
        else:
            self.attn_flops, self.attn_bytes = attn_work(par, L, T, Hq, Hkv, d, elt)
        V = self.acc.target_logits.shape[2]
        self.accept_bytes = accept_work(par, T, V, self.acc.draft_probs is not None)
        self.expand_bytes = 0.0
        if self.expand:
            self.expand_bytes = float(sum(x.numel() for x in self.exp_logits) * 4)

    def measure_selection(self):
        """Kept prefix keys summed over (sequence, node, kv head) and the
        number of distinct kept blocks summed over (sequence, kv head), from
        the selection the library returns (one untimed call)."""
        a = self.attn
        _, _, sel = self.tv.tree_verify_attn(a.q, a.k_cache, a.v_cache, a.prefix_len, a.k_tree, a.v_tree,
                                             a.parent, sparse_topk=a.sparse_topk, block_size=a.block_size,
                                             want_sel=True)
        torch.cuda.synchronize()
        sel = sel.cpu().numpy()                     # [B][T][Hkv][k]
        L = a.prefix_len.cpu().numpy()
        bs = a.block_size
        kept, union = 0, 0
        for b in range(sel.shape[0]):
            for g in range(sel.shape[2]):
                s = sel[b, :, g, :]
                s = s[s >= 0]
                keys = np.minimum(bs, int(L[b]) - bs * s)
                kept += int(np.sum(keys))
                union += len(np.unique(s))
        return kept, union

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
        exp = (1 + len(self.exp_logits)) if self.expand else 0
        return attn + 1 + exp

    def near_threshold(self):
        """Sequences whose walk met a decision within 1e-6 of its threshold
        (min_margin of the last acceptance call)."""
        mm = self.acc_out["min_margin"].cpu().numpy()
        return int(np.sum(mm < 1e-6))

    def free(self):
        for k in list(self.__dict__):
            if k not in ("name", "c", "B", "T", "sparse", "expand", "temperature"):
                self.__dict__.pop(k)
        torch.cuda.empty_cache()


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
    del host_in
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


def expansion_ablation(step):
    """The SpecExec page's ablation on the synthetic rows: the same 16 calls
    of draft rows build one tree best-first and one by beam search; each
    tree's sum of path probabilities is the expected number of accepted
    tokens when the target distribution equals the draft's.  Also the beam
    build's time (one build, CUDA events)."""
    tv, ec = step.tv, step.ec
    out = {}
    for mode in ("bestfirst", "beam"):
        st = tv.tree_expand_init(ec.budget, ec.V, ec.Bsel, device=step.dev)
        def build():
            tv.tree_expand_init(ec.budget, ec.V, ec.Bsel, state=st)
            for k, z in enumerate(step.exp_logits):
                rows = step.exp_root if k == 0 else st.frontier
                tv.tree_expand_topb(st, z, rows, mode=mode)
        build()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        build()
        e1.record()
        torch.cuda.synchronize()
        n = int(st.n_nodes.item())
        out[mode] = {"nodes": n, "expected_accepted": round(float(torch.exp(st.logp[1:n]).sum().item()), 4),
                     "build_us": round(e0.elapsed_time(e1) * 1e3, 1)}
    return out


def call_summary(step, times, world):
    """Per-call mean times (max over ranks) with their work and roofline
    fractions."""
    ms = {nm: max_over_ranks(statistics.fmean(times[nm]), world) for nm in times}
    out = {"ms_per_step": round(ms["step"], 5),
           "tree_tokens_per_s": step.B * step.T * world / (ms["step"] * 1e-3)}
    t = ms["attn"] * 1e-3
    out["tree_verify_attn"] = {
        "us": round(ms["attn"] * 1e3, 2), "path": step.attn_path, "launches": step.attn_launches,
        "tflops": round(step.attn_flops / t / 1e12, 2), "gbs": round(step.attn_bytes / t / 1e9, 1),
        "algorithmic_flops": step.attn_flops, "algorithmic_bytes": step.attn_bytes,
        "tokens_per_s": step.B * step.T / t, **roofline_fracs(t, step.attn_bytes, step.attn_flops)}
    if step.union_blocks is not None:
        out["tree_verify_attn"]["kept_block_union"] = step.union_blocks
    t = ms["accept"] * 1e-3
    out["tree_accept"] = {
        "us": round(ms["accept"] * 1e3, 2), "mode": step.acc.mode if step.temperature > 0 else "greedy",
        "gbs": round(step.accept_bytes / t / 1e9, 1), "algorithmic_bytes": step.accept_bytes,
        "nodes_per_s": step.B * step.T / t, "near_threshold": step.near_threshold(),
        **roofline_fracs(t, step.accept_bytes)}
    if "expand" in ms:
        t = ms["expand"] * 1e-3
        n_new = step.ec.budget - 1
        out["tree_expand_topb"] = {
            "us": round(ms["expand"] * 1e3, 2), "rounds": len(step.exp_logits),
            "gbs": round(step.expand_bytes / t / 1e9, 1), "algorithmic_bytes": step.expand_bytes,
            "nodes_per_s": n_new / t, **roofline_fracs(t, step.expand_bytes)}
        out["tree_expand_topb"]["ablation_bestfirst_vs_beam"] = expansion_ablation(step)
    return ms, out


# --------------------------------------------------------------------------
# CPU baseline and reference arm: the fp64 oracle over the host cores
# --------------------------------------------------------------------------

_POOL = None


def _pool_init(files, meta):
    global _POOL
    import numpy
    _POOL = {"meta": meta, "arr": {k: numpy.load(v, mmap_mode="r") for k, v in files.items()}}
    import oracle.attention  # noqa: F401  (imported before any timing)
    import oracle.accept  # noqa: F401


def _pool_ping(_):
    return os.getpid()


def _as_tensor(a, bf16):
    x = torch.from_numpy(np.array(a))
    return x.view(torch.bfloat16) if bf16 else x


def _pool_attn(task):
    """Oracle attention of some nodes of one (sequence, kv head): the call
    gets that sequence's inputs restricted to the kv head and its G query
    heads (contiguous GQA groups make this the same arithmetic)."""
    from oracle.attention import tree_verify_attn
    b, g, nodes = task
    A, m = _POOL["arr"], _POOL["meta"]
    G, bf = m["G"], m["bf16"]
    q = _as_tensor(A["q"][b:b + 1, :, g * G:(g + 1) * G], bf)
    k = _as_tensor(A["k"][b, g][None, :, None, :], bf)
    v = _as_tensor(A["v"][b, g][None, :, None, :], bf)
    kt = _as_tensor(A["kt"][b, :, g][None, :, None, :], bf)
    vt = _as_tensor(A["vt"][b, :, g][None, :, None, :], bf)
    pl = np.asarray(A["pl"][b:b + 1])
    par = np.asarray(A["par"][b:b + 1])
    t0 = time.perf_counter()
    tree_verify_attn(q, k, v, pl, kt, vt, par, sparse_topk=m["topk"], block_size=m["bs"],
                     rows={(0, int(i)) for i in nodes})
    return time.perf_counter() - t0, len(nodes)


def _pool_accept(b):
    """Oracle acceptance walk of sequence b."""
    from oracle.accept import tree_accept
    A, m = _POOL["arr"], _POOL["meta"]
    z = A["z"][b:b + 1]
    qd = A["qd"][b:b + 1] if "qd" in A else None
    tok, par = np.asarray(A["tok"][b:b + 1]), np.asarray(A["par"][b:b + 1])
    t0 = time.perf_counter()
    tree_accept(z, qd, tok, par, mode=m["mode"], temperature=m["temp"], seed=m["seed"])
    return time.perf_counter() - t0


class OracleRunner:
    """Times the fp64 oracle on a workload, spread over the host cores.

    The workload's inputs are written once to temporary .npy files (K/V as
    [B][Hkv][L][d], bf16 kept as raw 16-bit words) that every worker maps.
    Attention work is split into tasks of (sequence, kv head, nodes); the
    acceptance walk into one task per sequence.  Workers are spawned (not
    forked) with one BLAS thread each; the pool size is the number of cores
    this process may run on, at most MAX_WORKERS (each worker holds a few
    hundred MB of fp64 copies of one sequence's K/V)."""

    MAX_WORKERS = 32

    def __init__(self, host, workers=None):
        self.h = host
        self.dir = tempfile.mkdtemp(prefix="tv_oracle_")
        bf = host["q"].dtype == torch.bfloat16

        def arr(t):
            if isinstance(t, torch.Tensor):
                t = t.contiguous()
                return t.view(torch.int16).numpy() if t.dtype == torch.bfloat16 else t.numpy()
            return np.asarray(t)

        files = {}
        for name, t in (("q", host["q"]), ("k", host["k_cache"].permute(0, 2, 1, 3)),
                        ("v", host["v_cache"].permute(0, 2, 1, 3)), ("kt", host["k_tree"]),
                        ("vt", host["v_tree"]), ("pl", host["prefix_len"]), ("par", host["parent"]),
                        ("z", host["z"]), ("tok", host["tok"]), ("qd", host["qd"])):
            if t is None:
                continue
            p = os.path.join(self.dir, name + ".npy")
            np.save(p, arr(t))
            files[name] = p
        B, T, Hq, d = host["q"].shape
        Hkv = host["k_cache"].shape[2]
        self.B, self.T, self.Hkv, self.G = B, T, Hkv, Hq // Hkv
        self.meta = dict(G=self.G, bf16=bf, topk=host["topk"], bs=host["bs"], mode=host["mode"],
                         temp=host["temp"], seed=host["seed"])
        self.files = files
        try:
            ncpu = len(os.sched_getaffinity(0))
        except Exception:
            ncpu = os.cpu_count() or 1
        self.workers = workers or min(ncpu, self.MAX_WORKERS)
        import multiprocessing as mp
        saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        for k in saved:
            os.environ[k] = "1"
        try:
            self.pool = mp.get_context("spawn").Pool(self.workers, initializer=_pool_init,
                                                     initargs=(files, self.meta))
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        self.pool.map(_pool_ping, range(self.workers))        # every worker is up

    def attn_tasks(self, chunk):
        """(sequence, kv head, node chunk) tasks, chunk-major so that a prefix
        of the list covers every (sequence, kv head)."""
        tasks = []
        for c0 in range(0, self.T, chunk):
            for b in range(self.B):
                for g in range(self.Hkv):
                    tasks.append((b, g, list(range(c0, min(self.T, c0 + chunk)))))
        return tasks

    def one_worker_node_seconds(self, nodes=2):
        """Seconds per (node, kv head) of one oracle call in this process on
        one thread (the 1-worker time; also sizes the tasks)."""
        global _POOL
        from threadpoolctl import threadpool_limits
        _pool_init(self.files, self.meta)
        nt = torch.get_num_threads()
        torch.set_num_threads(1)
        try:
            with threadpool_limits(1):
                dt, n = _pool_attn((0, 0, list(range(min(nodes, self.T)))))
        finally:
            torch.set_num_threads(nt)
            _POOL = None
        return dt / n

    def time_attention(self, budget_s, per_unit_s):
        """Wall seconds of the pool over a bounded sample of attention tasks,
        and the (node, kv head) units it covered."""
        work_per_worker = max(1, int(budget_s / max(per_unit_s, 1e-6)))
        chunk = max(1, min(self.T, work_per_worker // 2))
        tasks = self.attn_tasks(chunk)
        total_units_wanted = work_per_worker * self.workers
        sample, units = [], 0
        for t in tasks:
            if units >= total_units_wanted:
                break
            sample.append(t)
            units += len(t[2])
        t0 = time.perf_counter()
        res = self.pool.map(_pool_attn, sample, chunksize=1)
        wall = time.perf_counter() - t0
        return wall, sum(n for _, n in res), sample

    def time_accept(self, seqs):
        """(wall seconds of the pool, summed seconds of the tasks) for the
        acceptance walks of the given sequences."""
        t0 = time.perf_counter()
        res = self.pool.map(_pool_accept, seqs, chunksize=1)
        return time.perf_counter() - t0, float(sum(res))

    def close(self):
        import shutil
        try:
            self.pool.terminate()
            self.pool.join()
        finally:
            shutil.rmtree(self.dir, ignore_errors=True)


def host_inputs(name, seed=0, device_step=None):
    """Host copies of a workload's inputs for the oracle.  From the device
    step when one exists (our arm's CPU baseline), else built on the host
    from the same seeded generators (the reference arm, which imports
    nothing of the library: the SpecExec tree is then built by the oracle's
    own expansion)."""
    from synth import CONFIGS, config_attn_case, config_accept_case, config_expand_case
    base = "longctx" if name == "longctx_sparse" else name
    c = CONFIGS[base]
    sparse = name == "longctx_sparse"
    temp = c.get("temperature", c.get("temperatures", (0.0,))[-1])
    if device_step is not None:
        a, ac = device_step.attn, device_step.acc
        h = {k: getattr(a, k).cpu() for k in ("q", "k_cache", "v_cache", "prefix_len", "k_tree", "v_tree",
                                              "parent")}
        h.update(z=ac.target_logits.cpu(), tok=ac.draft_tokens.cpu(),
                 qd=None if ac.draft_probs is None else ac.draft_probs.cpu(), mode=ac.mode, seed=ac.seed,
                 temp=device_step.temperature, topk=a.sparse_topk, bs=a.block_size,
                 exp=(device_step.ec, [z.cpu() for z in device_step.exp_logits]) if device_step.expand else None)
        return h
    exp = None
    if base == "specexec70b":
        from oracle.expand import ExpandState as OState, expand_call
        ec = config_expand_case(base, seed=seed)
        ost = OState(ec.budget, ec.root_token)
        frontier = [0]
        zs = []
        for call in range(ec.n_calls()):
            z = ec.round_logits(call, 1 if call == 0 else ec.Bsel)
            zs.append(z)
            if not frontier:
                break
            frontier = list(expand_call(ost, z.double().numpy()[:len(frontier)],
                                        np.asarray(frontier, np.int64), ec.Bsel))
        par = np.asarray(ost.parent, np.int32)
        a = config_attn_case(base, seed=seed, parents=[par])
        ac = config_accept_case(base, temperature=temp, seed=seed, parents=[par], mode="specexec")
        ac.draft_tokens = torch.tensor(np.asarray(ost.token, np.int32)).view(1, -1)
        mode = "specexec"
        exp = (ec, zs)
    else:
        a = config_attn_case(base, seed=seed, sparse=sparse)
        ac = config_accept_case(base, temperature=temp, seed=seed, parents=[p.numpy() for p in a.parent])
        mode = ac.mode
    h = {k: getattr(a, k) for k in ("q", "k_cache", "v_cache", "prefix_len", "k_tree", "v_tree", "parent")}
    h.update(z=ac.target_logits, tok=ac.draft_tokens, qd=ac.draft_probs, mode=mode, seed=ac.seed, temp=temp,
             topk=a.sparse_topk, bs=a.block_size, exp=exp)
    return h


def time_expand_oracle(exp, rounds=3):
    """Oracle expansion: the first `rounds` calls of the build timed (each
    round's rows depend on the previous round), scaled to the whole build."""
    from oracle.expand import ExpandState as OState, expand_call
    ec, zs = exp
    ost = OState(ec.budget, ec.root_token)
    frontier = [0]
    t = 0.0
    done = 0
    for call in range(min(rounds, len(zs))):
        z = zs[call].double().numpy()
        t0 = time.perf_counter()
        frontier = list(expand_call(ost, z[:len(frontier)], np.asarray(frontier, np.int64), ec.Bsel))
        t += time.perf_counter() - t0
        done += 1
    return t / done * len(zs), done, len(zs)


def cpu_baseline(host, budget_s=15.0, runner=None):
    """The oracle's whole-step throughput on the host cores: a bounded
    sample of the attention (tasks of (sequence, kv head, nodes) on a spawned
    process pool, wall-timed and scaled to every (node, kv head)), the full
    acceptance walk (one task per sequence), and for the SpecExec workload
    the expansion build (its first rounds, scaled).  Also the 1-worker time
    of the same work, from one call on one thread."""
    own = runner is None
    r = runner or OracleRunner(host)
    try:
        per_unit = r.one_worker_node_seconds()
        wall, units, sample = r.time_attention(budget_s, per_unit)
        all_units = r.B * r.T * r.Hkv
        t_attn = wall / units * all_units
        t_acc, t_acc_1 = r.time_accept(list(range(r.B)))
        t_exp, exp_note = 0.0, ""
        if host["exp"] is not None:
            t_exp, done, n = time_expand_oracle(host["exp"])
            exp_note = f"; expansion: {done} of {n} rounds timed (sequential), scaled to the build"
        t_step = t_attn + t_acc + t_exp
        t_step_1 = per_unit * all_units + t_acc_1 + t_exp
        tokens = r.B * r.T
        return {"value": tokens / t_step, "unit": "tokens/s", "cores": r.workers, "kind": "oracle",
                "workers": r.workers, "value_1worker": tokens / t_step_1,
                "sample": f"attention of {units} of {all_units} (node, kv head) pairs (fp64, all heads of the "
                          f"group) on {r.workers} spawned workers of one BLAS thread, wall {wall:.1f} s, scaled to "
                          f"the step; acceptance of all {r.B} sequences ({t_acc:.2f} s){exp_note}; the 1-worker "
                          f"value scales one single-thread call ({per_unit:.3f} s per pair)",
                "seconds": round(wall + t_acc + t_exp, 2)}
    finally:
        if own:
            r.close()


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
    """The oracle as the reference arm: each step is a bounded sample of the
    workload on the host cores, scaled to tokens per second."""
    if rank != 0:
        return
    host = host_inputs(args.config, 0)
    runner = OracleRunner(host)
    try:
        per_unit = runner.one_worker_node_seconds()
        budget = max(2.0, 45.0 / max(1, args.steps + args.warmup))
        t_exp = 0.0
        if host["exp"] is not None:
            t_exp, _, _ = time_expand_oracle(host["exp"], rounds=1)
        all_units = runner.B * runner.T * runner.Hkv
        workers = runner.workers
        vals = []
        for k in range(args.warmup + args.steps):
            wall, units, _ = runner.time_attention(budget, per_unit)
            b = k % runner.B
            _, t_one = runner.time_accept([b])
            t_acc = t_one * -(-runner.B // workers)
            t_step = wall / units * all_units + t_acc + t_exp
            if k >= args.warmup:
                vals.append(runner.B * runner.T / t_step)
        v = statistics.median(vals)
    finally:
        runner.close()
    from synth import CONFIGS
    base = "longctx" if args.config == "longctx_sparse" else args.config
    shim = type("S", (), dict(c=CONFIGS[base], name=args.config, temperature=host["temp"],
                              sparse=args.config == "longctx_sparse", B=runner.B, T=runner.T))()
    sample = (f"per step: attention of a bounded sample of (sequence, kv head, node) tasks on {workers} "
              f"spawned workers (about {budget:.0f} s), one sequence's acceptance walk (the pool walks "
              f"{min(workers, runner.B)} sequences at once), scaled to the step"
              + ("; expansion: one round timed, scaled to the build" if host["exp"] is not None else ""))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * runner.B * runner.T / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_block(shim, 1),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": workers, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_split_prefix(args, rank, world, dev, flush):
    """Strong scaling of the long-context attention: rank r attends to its
    slice [r * Lmax / N, (r + 1) * Lmax / N) of every sequence's prefix
    (prefix-only partials; the last rank also takes the tree keys), the
    partials are all-gathered over NCCL and merged by log-sum-exp with
    tree_verify_attn_merge.  A step = partial + all-gather + merge, timed
    with CUDA events (max over ranks); `value` counts each tree token once."""
    from synth import config_attn_case
    from tree_verification_verify_b200.split import prefix_slice, split_tree_verify_attn
    a = config_attn_case("longctx", seed=0, device=dev)
    B, T, Hq, d = a.q.shape
    Lmax = a.k_cache.shape[1]
    lo, hi = prefix_slice(rank, world, Lmax)
    L = a.prefix_len.cpu().numpy()
    kc, vc = a.k_cache[:, lo:hi], a.v_cache[:, lo:hi]
    parts = (torch.empty_like(a.q), torch.empty(B, T, Hq, dtype=torch.float32, device=dev),
             torch.empty((world,) + tuple(a.q.shape), dtype=a.q.dtype, device=dev),
             torch.empty(world, B, T, Hq, dtype=torch.float32, device=dev))
    out = torch.empty_like(a.q)
    lse = torch.empty(B, T, Hq, dtype=torch.float32, device=dev)

    def one():
        split_tree_verify_attn(a.q, kc, vc, a.prefix_len, a.k_tree, a.v_tree, a.parent, rank, world, lo, hi,
                               parts=parts, out=out, lse=lse)

    for _ in range(args.warmup):
        flush.zero_()
        one()
    torch.cuda.synchronize()
    barrier(world)
    ts = []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        one()
        e1.record()
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    ms = max_over_ranks(statistics.fmean(ts), world)
    flops, nbytes = attn_work(a.parent.cpu().numpy(), [int(x) for x in L], T, Hq, a.k_cache.shape[2], d,
                              a.q.element_size())
    line = {"metric": METRIC, "value": B * T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "longctx attention, prefix split across ranks: B=4 Hq=32 Hkv=8 d=128 bf16 "
                                   "prefix=131072 T=256", "parallelism": f"prefix split x{world}",
                       "l2": "256 MiB flush before every timed step (not timed)",
                       "launch": "eager calls; NCCL all-gather of the partials"},
            "roofline": {"bound": "tensor", "achieved": round(flops / (ms * 1e-3) / 1e12, 2),
                         "peak": peaks()[1] * world, "unit": "TFLOP/s",
                         "frac": round(flops / (ms * 1e-3) / 1e12 / (peaks()[1] * world), 4)},
            "gpu_launches": (3 if world > 1 else 2) * args.steps}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_iteration(args, rank, world, dev, flush):
    """Whole-iteration throughput of the speculative loop (loop.Iteration)
    replayed from one CUDA graph: emitted tokens (accepted + bonus) per
    second, and the per-iteration time."""
    from tree_verification_verify_b200.loop import Iteration
    it = Iteration(dev, iters_room=args.steps + args.warmup + 8)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(3):
            it.step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        it.step()
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    it.emitted.zero_()
    pl0 = int(it.prefix_len.item())
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record()
    for _ in range(args.steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    emitted = int(it.emitted.item())
    grown = int(it.prefix_len.item()) - pl0
    line = {"metric": "emitted tokens/s of the whole speculative iteration (random-weight stand-in models)",
            "value": emitted * world / (ms * 1e-3 * args.steps), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "iteration: drafter bigram stand-in V=32000, tree budget 64 in 4 rounds of 16, "
                                   "one target layer (32/8 heads, d=128, bf16) over a 4096-token prefix, "
                                   "SpecExec acceptance at temperature 0.6, KV commit",
                       "launch": "one CUDA graph per iteration", "parallelism": f"replicas x{world}"},
            "tokens_per_iteration": emitted / args.steps, "prefix_growth": grown,
            "status": int(it.status.item()),
            "gpu_launches": it.launches_per_step() * args.steps}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g


def main_roofline(step, ms, hbm, bf16, src):
    """The roofline object of the step's dominant call."""
    attn_s, acc_s = ms["attn"] * 1e-3, ms["accept"] * 1e-3
    exp_s = ms.get("expand", 0.0) * 1e-3
    if exp_s >= max(acc_s, attn_s):
        achieved = step.expand_bytes / exp_s / 1e9
        roof = {"kernel": "tree_expand_topb (16 rounds, one launch each)", "bound": "hbm",
                "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                "algorithmic_bytes": step.expand_bytes, "units": "draft logit rows of all rounds x V x 4 B"}
        tk = "expand_round_kernel"
    elif acc_s >= attn_s:
        achieved = step.accept_bytes / acc_s / 1e9
        roof = {"kernel": "accept_node_kernel (tree_accept: one launch)", "bound": "hbm",
                "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                "algorithmic_bytes": step.accept_bytes, "units": "B x T x V x 4 B of target logits (+ draft rows)"}
        tk = "accept_node_kernel"
    elif step.attn_bytes / (hbm * 1e9) >= step.attn_flops / (bf16 * 1e12):
        achieved = step.attn_bytes / attn_s / 1e9
        roof = {"kernel": "tree_verify_attn", "bound": "hbm", "achieved": round(achieved, 1),
                "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                "algorithmic_bytes": step.attn_bytes, "units": "every prefix and tree K/V element once"}
        tk = "attn_tc_kernel"
    else:
        achieved = step.attn_flops / attn_s / 1e12
        roof = {"kernel": "tree_verify_attn", "bound": "tensor", "achieved": round(achieved, 2),
                "peak": bf16, "unit": "TFLOP/s", "frac": round(achieved / bf16, 4),
                "algorithmic_flops": step.attn_flops, "units": "4 d Hq x sum over nodes of |K(i)|"}
        tk = "attn_tc_kernel"
    roof["peak_source"] = src + " (MEASURED_PEAKS.json: burst figures, each call timed alone)" \
        if src == "measured" else src
    # against the 8 TB/s / 2.25 PFLOP/s denominators
    tpk = TARGET_HBM_GBS if roof["bound"] == "hbm" else TARGET_BF16_TFLOPS
    roof["frac_target"] = round(roof["achieved"] / tpk, 4)
    roof["traffic"] = None
    if tk == "attn_tc_kernel" and step.attn_path == 4:
        tk = "attn_pair_kernel"
    if tk in ("attn_tc_kernel", "attn_pair_kernel") and step.attn_path in (1, 4):
        roof["kernel"] = f"{tk} (tree_verify_attn: one launch)"
    if tk not in ("attn_tc_kernel", "attn_pair_kernel") or step.attn_path in (1, 4):
        roof["traffic"] = measured_traffic(tk, step.name)
        roof["traffic_source"] = "profiles/traffic.txt (ncu dram__bytes_read.sum + dram__bytes_write.sum)"
    return roof


def run_config(name, args, world, rank, dev, flush, K, W, with_e2e):
    """Build one workload, time its step, and summarise it."""
    step = Step(name, seed=rank, dev=dev)
    times = time_steps(step, K, W, world, flush)
    ms, summary = call_summary(step, times, world)
    res = {"step": step, "ms": ms, "summary": summary}
    if with_e2e:
        e2e_ms, h2d, d2h = time_e2e(step, max(3, K // 5), 3, flush)
        res["e2e"] = (max_over_ranks(e2e_ms, world), h2d, d2h)
        commit_ms, commit_bytes = time_commit(step, max(3, K), 3, flush)
        res["commit"] = (max_over_ranks(commit_ms, world), commit_bytes)
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="longctx", choices=CONFIG_NAMES)
    ap.add_argument("--only", action="store_true", help="time the main workload alone (no other configs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--split-prefix", action="store_true",
                    help="long-context attention with the prefix split across the ranks (strong scaling)")
    ap.add_argument("--iteration", action="store_true",
                    help="the whole speculative iteration (expand, verify, accept, commit) as one CUDA graph")
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
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    if args.split_prefix or args.iteration:
        (run_split_prefix if args.split_prefix else run_iteration)(args, rank, world, dev, flush)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    clk = ClockSampler(local)
    clk.start()
    main_res = run_config(args.config, args, world, rank, dev, flush, args.steps, args.warmup, True)
    clocks = clk.stop()
    step, ms, summary = main_res["step"], main_res["ms"], main_res["summary"]
    hbm, bf16, bf16_sus, src = peaks()
    e2e_ms, h2d, d2h = main_res["e2e"]
    commit_ms, commit_bytes = main_res["commit"]
    tokens = step.B * step.T * world
    line = {
        "metric": METRIC, "value": tokens / (ms["step"] * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms["step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_block(step, world),
        "roofline": main_roofline(step, ms, hbm, bf16, src),
        "calls": summary,
        "launches_per_step": step.launches_per_step(),
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": "every step copies all of its inputs (KV cache included) from pinned host memory"},
        "gpu_launches": step.launches_per_step() * args.steps,
        "clocks": clocks,
        "near_threshold": step.near_threshold(),
    }
    line["calls"]["tree_commit_kv"] = {"us": round(commit_ms * 1e3, 2), "bytes": commit_bytes,
                                       "gbs": round(commit_bytes / (commit_ms * 1e-3) / 1e9, 1)}
    host = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = host_inputs(args.config, device_step=step)
    step.free()
    del main_res
    if not args.only and args.config == "longctx":
        line["configs"] = {}
        clk2 = ClockSampler(local)
        clk2.start()
        for name in EXTRA_CONFIGS:
            r = run_config(name, args, world, rank, dev, flush, max(5, min(args.steps, 10)), 3, False)
            s = r["summary"]
            s["workload"] = config_block(r["step"], world)["workload"]
            s["near_threshold"] = r["step"].near_threshold()
            line["configs"][name] = s
            r["step"].free()
            del r
        line["configs_clocks"] = clk2.stop()
    if host is not None:
        line["cpu_baseline"] = cpu_baseline(host)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
