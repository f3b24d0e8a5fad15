"""SpecExec's batched best-first tree expansion, fp64 oracle.

SpecExec page, "Approach": build the draft tree from the highest
cumulative-probability continuations with a parallel (batched) Dijkstra-style
search using the draft model; "Builds on": Dijkstra's algorithm; the
ablation table shows standard beam search is a worse constructor.

State: the tree (node 0 = root, logp 0) and a pool of candidates not yet
taken.  One call (one round of the batched search):

1. For every expanded row r (the draft logits zd_r of tree node n_r; each
   node is expanded at most once) and every token t, the child candidate
   (n_r, t) gets the cumulative draft log-probability

       score = (logp(n_r) + zd_r[t] / tau) - lse_r,
       lse_r = logsumexp_t(zd_r[t] / tau)          (float64, two-pass)

   i.e. logp(parent) + log softmax(zd_r / tau)[t].
2. Pool and new candidates are merged and sorted by the total order
   (score desc, parent asc, token asc).
3. The first sel = min(Bsel, budget - n_nodes, #candidates) become nodes
   n_nodes, n_nodes + 1, ... in that order; they are the next frontier.
4. The pool keeps the next budget - n_nodes(after) candidates.  Candidates
   ranked beyond the remaining budget are never taken: every later
   candidate descends from a taken node and scores no higher than it
   (log-probabilities only decrease along a path), and the kept ones all
   rank above them.

Reading of "top-B": Bsel nodes are appended per round (batched Dijkstra with
a carried pool), not the top-B children of the current depth (beam search).
The budget counts the root.

Beam mode (the page's ablation "Replace parallel SSSP tree search with
standard beam search"): a call ranks only the children of its own rows (the
current depth's beam) by the same scores and order, appends the best
min(Bsel, budget - n_nodes) of them, and carries nothing to later calls.

Status bits: BAD_ROW (8) for a row whose node is not in the tree or was
already expanded (the row is skipped); NONFINITE (4) for a row holding a
non-finite logit (skipped; the node still counts as expanded).
"""

from __future__ import annotations

import numpy as np

from .attention import _f64, _i64, ST_NONFINITE, ST_BAD_ROW



class ExpandState:
    def __init__(self, budget: int, root_token: int = 0):
        self.budget = int(budget)
        self.parent = [-1]
        self.token = [int(root_token)]
        self.logp = [0.0]
        self.pool_score = np.zeros(0)
        self.pool_parent = np.zeros(0, dtype=np.int64)
        self.pool_token = np.zeros(0, dtype=np.int64)
        self.expanded = set()
        self.status = 0
        self.gaps = []          # per call: min score gap among ranks 1..sel+1

    @property
    def n_nodes(self):
        return len(self.parent)


def row_scores(logp_n: float, z, tau: float):
    """Cumulative log-probabilities of the V children of one node."""
    x = _f64(z) / float(np.float32(tau))     # the call takes an fp32 temperature
    m = np.max(x)
    lse = m + np.log(np.sum(np.exp(x - m)))
    return (logp_n + x) - lse


def expand_call(st: ExpandState, draft_logits, row_node, Bsel: int, tau: float = 1.0,
                mode: str = "bestfirst"):
    """One round.  draft_logits [R][V], row_node [R] (-1 = no row); mode
    "bestfirst" (carried pool) or "beam" (this call's rows only).
    Returns the appended node indices (the next frontier)."""
    if mode not in ("bestfirst", "beam"):
        raise ValueError(mode)
    Zd = draft_logits
    rows = [int(x) for x in _i64(row_node)]
    rem = st.budget - st.n_nodes
    if mode == "beam":
        sc, pa, tk = [np.zeros(0)], [np.zeros(0, dtype=np.int64)], [np.zeros(0, dtype=np.int64)]
    else:
        sc = [st.pool_score]
        pa = [st.pool_parent]
        tk = [st.pool_token]
    for r, n in enumerate(rows):
        if n < 0:
            continue
        if n >= st.n_nodes or n in st.expanded:
            st.status |= ST_BAD_ROW
            continue
        st.expanded.add(n)                      # a row is consumed once given
        z = _f64(Zd[r])
        if not np.all(np.isfinite(z)):
            st.status |= ST_NONFINITE
            continue
        V = len(z)
        sc.append(row_scores(st.logp[n], z, tau))
        pa.append(np.full(V, n, dtype=np.int64))
        tk.append(np.arange(V, dtype=np.int64))
    score = np.concatenate(sc)
    par = np.concatenate(pa)
    tok = np.concatenate(tk)
    if rem <= 0 or len(score) == 0:
        st.gaps.append(np.inf)
        return []
    order = np.lexsort((tok, par, -score))      # primary key last
    score, par, tok = score[order], par[order], tok[order]
    sel = min(int(Bsel), rem, len(score))
    k = min(sel + 1, len(score))
    st.gaps.append(float(np.min(score[:k - 1] - score[1:k])) if k > 1 else np.inf)
    new = []
    for r in range(sel):
        st.parent.append(int(par[r]))
        st.token.append(int(tok[r]))
        st.logp.append(float(score[r]))
        new.append(st.n_nodes - 1)
    keep = st.budget - st.n_nodes if mode == "bestfirst" else 0
    st.pool_score = score[sel:sel + keep]
    st.pool_parent = par[sel:sel + keep]
    st.pool_token = tok[sel:sel + keep]
    return new


def expand_build(budget: int, Bsel: int, logits_for_call, tau: float = 1.0,
                 root_token: int = 0, max_calls: int = 1 << 30):
    """Run rounds from the root until the tree holds `budget` nodes.
    logits_for_call(call, frontier) returns the [len(frontier)][V] draft
    logits of the frontier nodes."""
    st = ExpandState(budget, root_token)
    frontier = [0]
    call = 0
    while st.n_nodes < budget and frontier and call < max_calls:
        z = logits_for_call(call, frontier)
        frontier = expand_call(st, z, frontier, Bsel, tau)
        call += 1
    return st
