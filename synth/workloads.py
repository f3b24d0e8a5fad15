"""Seeded synthetic workloads for tree verification.

Every array here is random input: tree shapes (`parent[]`), post-RoPE query,
key and value tensors, target and draft logits, the draft distribution handed
to the acceptance step, and the draft tokens on the tree nodes.  Nothing in
this module computes attention, acceptance or expansion.

The five named configurations follow the workloads of the speculative
decoding pages (SpecExec: Massively Parallel Speculative Decoding..., "Key
results": Llama 2-70B target, budgets 256 and 2048; EasySpec, "Experimental
setup": Llama-3 / Qwen2 shaped targets; "Accelerate Speculative Decoding with
Sparse Computation in Verification", "Methodology" 3: block top-k attention on
long prefixes).  The pages run their experiments on text datasets that are not
available here; Gaussian logits and N(0,1) activations of the same shapes,
vocabulary sizes and tree budgets stand in for them.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np
import torch

# --------------------------------------------------------------------------
# named configurations
# --------------------------------------------------------------------------

CONFIGS = {
    # batch 1, 4 query heads on 1 kv head, d=64 in fp32, 128-token prefix,
    # full binary tree of depth 3 (15 nodes), vocabulary 256.
    "tiny": dict(B=1, Hq=4, Hkv=1, d=64, dtype="fp32", L=128, T=15,
                 tree="binary", V=256, sigma=3.0, temperatures=(0.0, 0.8),
                 Bsel=8, budget=64),
    # one Llama-3-8B shaped attention layer: 32 q heads, 8 kv heads, d=128,
    # 4096-token prefix, 64-node tree with per-depth fan-out 4,3,2,2,...
    "llama3_8b": dict(B=1, Hq=32, Hkv=8, d=128, dtype="bf16", L=4096, T=64,
                      tree="bfs", fanout=(4, 3, 2), V=128256, sigma=3.0,
                      temperature=0.8),
    # Llama-2-70B shaped SpecExec tree: 64 q heads, 8 kv heads, 2048-token
    # prefix, 2048-node tree built by best-first expansion (128 per round)
    # from N(0, 4^2) draft logits over a 32000-token vocabulary.
    "specexec70b": dict(B=1, Hq=64, Hkv=8, d=128, dtype="bf16", L=2048,
                        T=2048, tree="expand", V=32000, sigma=4.0, Bsel=128,
                        budget=2048, temperatures=(0.0, 0.6)),
    # batched serving, Qwen2-72B shaped: 32 sequences, prefixes uniform in
    # [512, 16384], 16-node random trees of depth <= 6, vocabulary 152064.
    "serving": dict(B=32, Hq=64, Hkv=8, d=128, dtype="bf16", L=(512, 16384),
                    T=16, tree="random_depth", max_depth=6, V=152064,
                    sigma=3.0, temperature=0.8),
    # long context: 4 sequences of 131072 prefix tokens, 256-node tree, 5% of
    # the 64-token key blocks carry a shared offset; dense and block top-k.
    "longctx": dict(B=4, Hq=32, Hkv=8, d=128, dtype="bf16", L=131072, T=256,
                    tree="bfs", fanout=(4, 3, 2), V=128256, sigma=3.0,
                    temperature=0.0, sparse_topk=32, block_size=64,
                    offset_frac=0.05),
}


def _gen(seed: int, stream: int, device="cpu") -> torch.Generator:
    """A torch generator for one named random stream of one seed."""
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + int(stream) * 7919 + 17) % (2**63 - 1))
    return g


def _dtype(name):
    return {"fp32": torch.float32, "bf16": torch.bfloat16}[name]


# --------------------------------------------------------------------------
# tree shapes (parent[] arrays, node 0 = root = last committed token,
# parent[0] = -1, parent[i] < i)
# --------------------------------------------------------------------------

def tree_binary(T: int) -> np.ndarray:
    """Full binary tree in heap order: parent[i] = (i-1)//2."""
    p = np.array([-1] + [(i - 1) // 2 for i in range(1, T)], dtype=np.int32)
    return p[:T]


def tree_chain(T: int) -> np.ndarray:
    """A single path: parent[i] = i-1."""
    return np.arange(-1, T - 1, dtype=np.int32)


def tree_star(T: int) -> np.ndarray:
    """Every draft node hangs off the root."""
    p = np.zeros(T, dtype=np.int32)
    p[0] = -1
    return p


def tree_bfs_fanout(T: int, fanout: Sequence[int]) -> np.ndarray:
    """Breadth-first tree: a node at depth k gets fanout[k] children (the
    last entry repeats for deeper levels), nodes numbered level by level and
    the fill stops at T nodes."""
    parent = [-1]
    depth = [0]
    frontier = [0]
    while len(parent) < T and frontier:
        nxt = []
        for n in frontier:
            k = fanout[min(depth[n], len(fanout) - 1)]
            for _ in range(k):
                if len(parent) >= T:
                    break
                parent.append(n)
                depth.append(depth[n] + 1)
                nxt.append(len(parent) - 1)
        frontier = nxt
    return np.array(parent, dtype=np.int32)


def tree_random_depth_limited(T: int, max_depth: int, g: torch.Generator) -> np.ndarray:
    """parent[i] uniform over the earlier nodes of depth < max_depth."""
    parent = np.full(T, -1, dtype=np.int32)
    depth = np.zeros(T, dtype=np.int64)
    for i in range(1, T):
        elig = np.nonzero(depth[:i] < max_depth)[0]
        j = int(torch.randint(len(elig), (1,), generator=g).item())
        parent[i] = elig[j]
        depth[i] = depth[elig[j]] + 1
    return parent


def tree_random_recursive(T: int, g: torch.Generator) -> np.ndarray:
    """Random recursive tree: parent[i] uniform over [0, i)."""
    parent = np.full(T, -1, dtype=np.int32)
    if T > 1:
        u = torch.rand(T - 1, generator=g, dtype=torch.float64).numpy()
        parent[1:] = np.floor(u * np.arange(1, T)).astype(np.int32)
    return parent


def tree_depths(parent: np.ndarray) -> np.ndarray:
    """Depth of every node of a well-formed parent[] (root depth 0)."""
    d = np.zeros(len(parent), dtype=np.int64)
    for i in range(1, len(parent)):
        d[i] = d[parent[i]] + 1
    return d


# --------------------------------------------------------------------------
# attention inputs
# --------------------------------------------------------------------------

@dataclass
class AttnCase:
    q: torch.Tensor            # [B][T][Hq][d]
    k_cache: torch.Tensor      # [B][Lmax][Hkv][d]
    v_cache: torch.Tensor      # [B][Lmax][Hkv][d]
    prefix_len: torch.Tensor   # [B] int32
    k_tree: torch.Tensor       # [B][T][Hkv][d]
    v_tree: torch.Tensor       # [B][T][Hkv][d]
    parent: torch.Tensor       # [B][T] int32
    n_nodes: Optional[torch.Tensor] = None   # [B] int32 or None (= T)
    scale: float = 0.0
    sparse_topk: int = 0
    block_size: int = 64
    offset_blocks: Optional[list] = None     # per (b, kvh) offset block ids (info)

    @property
    def dims(self):
        B, T, Hq, d = self.q.shape
        return dict(B=B, T=T, Hq=Hq, Hkv=self.k_cache.shape[2], d=d,
                    Lmax=self.k_cache.shape[1])


def attn_case(B: int, T: int, Hq: int, Hkv: int, d: int, L, dtype: str,
              parents, seed: int = 0, n_nodes=None, Lmax: Optional[int] = None,
              device="cpu", offset_frac: float = 0.0, block_size: int = 64,
              sparse_topk: int = 0, scale: float = 0.0) -> AttnCase:
    """Q/K/V ~ N(0,1) (rounded to `dtype`), one prefix length per sequence.

    `L` is an int (same for every sequence) or a sequence of B ints.
    `parents` is one parent[] array (shared) or a list of B arrays.
    With offset_frac > 0, round(offset_frac * n_blocks) key blocks of
    `block_size` tokens per (sequence, kv head), chosen by a seeded
    permutation, get the same N(0,1)^d offset vector of their kv head added
    to every key: the high-relevance blocks of the long-context workload.
    """
    Ls = [int(L)] * B if np.isscalar(L) else [int(x) for x in L]
    assert len(Ls) == B
    if Lmax is None:
        Lmax = max(Ls) if Ls else 0
    if isinstance(parents, np.ndarray) and parents.ndim == 1:
        parents = [parents] * B
    par = np.stack([np.asarray(p, dtype=np.int32) for p in parents]) if B else np.zeros((0, T), np.int32)
    assert par.shape == (B, T)
    dt = _dtype(dtype)
    gq = _gen(seed, 1, device)
    gk = _gen(seed, 2, device)
    gv = _gen(seed, 3, device)
    gt = _gen(seed, 4, device)
    go = _gen(seed, 5, "cpu")
    q = torch.randn(B, T, Hq, d, generator=gq, device=device).to(dt)
    k_cache = torch.empty(B, Lmax, Hkv, d, dtype=dt, device=device)
    v_cache = torch.empty(B, Lmax, Hkv, d, dtype=dt, device=device)
    offsets = None
    if offset_frac > 0:
        m = torch.randn(Hkv, d, generator=go)
        offsets = []
    for b in range(B):
        kb = torch.randn(Lmax, Hkv, d, generator=gk, device=device)
        if offset_frac > 0:
            nblk = (Ls[b] + block_size - 1) // block_size
            n_off = int(round(offset_frac * nblk))
            per_b = []
            for h in range(Hkv):
                perm = torch.randperm(nblk, generator=go)[:n_off].sort().values
                per_b.append(perm.numpy())
                for j in perm.tolist():
                    lo, hi = j * block_size, min((j + 1) * block_size, Ls[b])
                    kb[lo:hi, h, :] += m[h].to(device)
            offsets.append(per_b)
        k_cache[b] = kb.to(dt)
        v_cache[b] = torch.randn(Lmax, Hkv, d, generator=gv, device=device).to(dt)
    k_tree = torch.randn(B, T, Hkv, d, generator=gt, device=device).to(dt)
    v_tree = torch.randn(B, T, Hkv, d, generator=gt, device=device).to(dt)
    nn = None
    if n_nodes is not None:
        nn = torch.tensor(np.broadcast_to(np.asarray(n_nodes, np.int32), (B,)).copy(),
                          dtype=torch.int32, device=device)
    return AttnCase(q=q, k_cache=k_cache, v_cache=v_cache,
                    prefix_len=torch.tensor(Ls, dtype=torch.int32, device=device),
                    k_tree=k_tree, v_tree=v_tree,
                    parent=torch.tensor(par, dtype=torch.int32, device=device),
                    n_nodes=nn, scale=scale, sparse_topk=sparse_topk,
                    block_size=block_size, offset_blocks=offsets)


# --------------------------------------------------------------------------
# acceptance inputs
# --------------------------------------------------------------------------

@dataclass
class AcceptCase:
    target_logits: torch.Tensor            # [B][T][V] fp32
    draft_probs: Optional[torch.Tensor]    # [B][T][V] fp32 or None
    draft_tokens: torch.Tensor             # [B][T] int32
    parent: torch.Tensor                   # [B][T] int32
    n_nodes: Optional[torch.Tensor]        # [B] int32 or None
    temperature: float
    seed: int
    step: int
    mode: str                              # auto | greedy | specsample | specexec


def accept_case(B: int, T: int, V: int, parents, temperature: float,
                sigma: float = 3.0, seed: int = 0, mode: str = "auto",
                correlated: bool = False, child_rule: str = "sample",
                n_nodes=None, with_q: bool = True, device="cpu",
                step: int = 0, rng_seed: Optional[int] = None,
                noise: float = 0.5) -> AcceptCase:
    """Target and draft logits ~ N(0, sigma^2) over V tokens per node.

    The draft distribution handed to acceptance is q = softmax(zd / t) of the
    draft logits zd, formed in float64 and rounded to fp32 (t = temperature,
    or 1 at temperature 0).  child_rule "sample": the token of node i >= 1 is
    drawn from q of its parent, independently per node (children drawn with
    replacement, as in a sampled draft tree).  child_rule "top": the children
    of a node, in node order, take the distinct top tokens of its draft
    logits in rank order (a deterministic tree).  With correlated=True the
    target logits are zd + N(0, noise^2), so that acceptance walks go deep.
    `rng_seed` is the Philox seed of the acceptance call (defaults to seed).
    """
    if isinstance(parents, np.ndarray) and parents.ndim == 1:
        parents = [parents] * B
    par = np.stack([np.asarray(p, dtype=np.int32) for p in parents]) if B else np.zeros((0, T), np.int32)
    gd = _gen(seed, 11, device)
    gz = _gen(seed, 12, device)
    gs = _gen(seed, 13, device)
    zd = torch.randn(B, T, V, generator=gd, device=device) * sigma
    if correlated:
        z = zd + noise * torch.randn(B, T, V, generator=gz, device=device)
    else:
        z = torch.randn(B, T, V, generator=gz, device=device) * sigma
    tq = temperature if temperature > 0 else 1.0
    q = None
    need_q = with_q or child_rule == "sample"
    if need_q:
        q = torch.empty(B, T, V, dtype=torch.float32, device=device)
        for b in range(B):
            q[b] = torch.softmax(zd[b].double() / tq, dim=-1).float()
    tokens = torch.zeros(B, T, dtype=torch.int64, device=device)
    partorch = torch.tensor(par, dtype=torch.int64, device=device)
    if T > 1:
        if child_rule == "sample":
            for b in range(B):
                rows = q[b][partorch[b, 1:]].double()
                tokens[b, 1:] = torch.multinomial(rows, 1, replacement=True, generator=gs)[:, 0]
        elif child_rule == "top":
            for b in range(B):
                kids = {}
                for i in range(1, T):
                    kids.setdefault(int(par[b, i]), []).append(i)
                for c, ch in kids.items():
                    top = torch.topk(zd[b, c], len(ch)).indices
                    for r, i in enumerate(ch):
                        tokens[b, i] = top[r]
        else:
            raise ValueError(child_rule)
    if T > 0:
        tokens[:, 0] = torch.randint(V, (B,), generator=gs, device=device)
    nn = None
    if n_nodes is not None:
        nn = torch.tensor(np.broadcast_to(np.asarray(n_nodes, np.int32), (B,)).copy(),
                          dtype=torch.int32, device=device)
    return AcceptCase(target_logits=z.float().contiguous(),
                      draft_probs=(q if with_q else None),
                      draft_tokens=tokens.to(torch.int32),
                      parent=torch.tensor(par, dtype=torch.int32, device=device),
                      n_nodes=nn, temperature=float(temperature),
                      seed=int(seed if rng_seed is None else rng_seed),
                      step=int(step), mode=mode)


# --------------------------------------------------------------------------
# expansion inputs
# --------------------------------------------------------------------------

@dataclass
class ExpandCase:
    V: int
    Bsel: int
    budget: int
    sigma: float
    seed: int
    draft_temperature: float = 1.0
    root_token: int = 0

    def n_calls(self) -> int:
        """Calls until the tree holds `budget` nodes (each call appends
        min(Bsel, budget - n_nodes) nodes while candidates last)."""
        return int(math.ceil((self.budget - 1) / self.Bsel)) if self.budget > 1 else 0

    def round_logits(self, call: int, R: int, device="cpu") -> torch.Tensor:
        """Draft logits [R][V] ~ N(0, sigma^2) for the rows of call `call`."""
        g = _gen(self.seed, 1000 + call, device)
        return (torch.randn(max(R, 0), self.V, generator=g, device=device) * self.sigma).contiguous()


def expand_case(V: int, Bsel: int, budget: int, sigma: float, seed: int = 0,
                draft_temperature: float = 1.0, root_token: int = 0) -> ExpandCase:
    return ExpandCase(V=V, Bsel=Bsel, budget=budget, sigma=sigma, seed=seed,
                      draft_temperature=draft_temperature, root_token=root_token)


# --------------------------------------------------------------------------
# named-configuration helpers
# --------------------------------------------------------------------------

def config_tree(name: str, seed: int = 0, b: int = 0) -> np.ndarray:
    """parent[] of one sequence of a named configuration (the SpecExec
    configuration's tree is built by expansion; a random recursive tree of
    the same size stands in where an attention-only case is wanted)."""
    c = CONFIGS[name]
    if c["tree"] == "binary":
        return tree_binary(c["T"])
    if c["tree"] == "bfs":
        return tree_bfs_fanout(c["T"], c["fanout"])
    if c["tree"] == "random_depth":
        return tree_random_depth_limited(c["T"], c["max_depth"], _gen(seed, 100 + b))
    if c["tree"] == "expand":
        return tree_random_recursive(c["T"], _gen(seed, 200 + b))
    raise ValueError(c["tree"])


def config_prefix_lens(name: str, seed: int = 0) -> list:
    c = CONFIGS[name]
    if isinstance(c["L"], tuple):
        lo, hi = c["L"]
        u = torch.rand(c["B"], generator=_gen(seed, 300), dtype=torch.float64).numpy()
        return [int(lo + math.floor(x * (hi - lo + 1))) for x in u]
    return [c["L"]] * c["B"]


def config_attn_case(name: str, seed: int = 0, device="cpu", parents=None,
                     sparse: bool = False) -> AttnCase:
    c = CONFIGS[name]
    B = c["B"]
    if parents is None:
        parents = [config_tree(name, seed, b) for b in range(B)]
    return attn_case(B, c["T"], c["Hq"], c["Hkv"], c["d"], config_prefix_lens(name, seed),
                     c["dtype"], parents, seed=seed, device=device,
                     offset_frac=c.get("offset_frac", 0.0),
                     block_size=c.get("block_size", 64),
                     sparse_topk=(c.get("sparse_topk", 0) if sparse else 0))


def config_accept_case(name: str, temperature: Optional[float] = None, seed: int = 0,
                       device="cpu", parents=None, correlated: bool = False,
                       mode: str = "auto") -> AcceptCase:
    c = CONFIGS[name]
    t = c.get("temperature", 0.0) if temperature is None else temperature
    B = c["B"]
    if parents is None:
        parents = [config_tree(name, seed, b) for b in range(B)]
    child_rule = "sample" if t > 0 else "top"
    if mode == "specexec":
        child_rule = "top"
    need_q = (mode in ("specsample",)) or (mode == "auto" and t > 0)
    return accept_case(B, c["T"], c["V"], parents, t, sigma=c["sigma"], seed=seed,
                       mode=mode, correlated=correlated, child_rule=child_rule,
                       with_q=need_q, device=device)


def config_expand_case(name: str, seed: int = 0) -> ExpandCase:
    c = CONFIGS[name]
    return expand_case(c["V"], c["Bsel"], c["budget"], c["sigma"], seed=seed)
