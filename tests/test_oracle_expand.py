"""Pins of the expansion oracle.

* Bsel = 1 is exact Dijkstra: the tree equals the brute-force global top-N
  of the (path-keyed, hence order-independent) infinite draft tree
  enumerated to a depth that contains it.
* Bsel > 1 equals an independent heap-based simulation of the rounds that
  keeps every candidate (so pool truncation loses nothing).
* Ties: with every logit of a row equal, all candidates of one depth tie
  exactly and the order rests on the tie-breaks alone (parent ascending,
  then token ascending): the oracle equals the heap simulation (which
  orders by the tuple (-score, parent, token)), and at Bsel = 1 the tree is
  the breadth-first numbering (node k: parent (k-1) // V, token (k-1) % V).
* Best-first differs from beam search (the SpecExec page's ablation) and,
  at Bsel = 1, keeps at least as much draft probability mass.
* A closed-form worked example with exact probabilities (golden file).
* Structural invariants on the SpecExec-sized workload.
"""

import heapq
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
from scipy.special import logsumexp

from oracle.expand import ExpandState, expand_call, expand_build, ST_BAD_ROW

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "expand_worked_example.txt")


def _row(path, V, sigma, seed):
    ss = np.random.SeedSequence([seed, 77, len(path)] + [t + 1 for t in path])
    return np.random.default_rng(ss).normal(0.0, sigma, size=V)


def _paths(st):
    paths = [()]
    for i in range(1, st.n_nodes):
        paths.append(paths[st.parent[i]] + (st.token[i],))
    return paths


def _run(V, Bsel, budget, sigma, seed, tau=1.0):
    st = ExpandState(budget)
    frontier = [0]
    while st.n_nodes < budget and frontier:
        paths = _paths(st)
        z = np.stack([_row(paths[n], V, sigma, seed) for n in frontier])
        frontier = expand_call(st, z, frontier, Bsel, tau)
    return st


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_bsel1_is_global_top_n(seed):
    V, budget, sigma, D = 4, 40, 1.0, 8
    st = _run(V, 1, budget, sigma, seed)
    # brute force: every token path up to depth D with its log-probability
    allp = {(): 0.0}
    frontier = [()]
    for _ in range(D):
        nxt = []
        for p in frontier:
            z = _row(p, V, sigma, seed)
            ls = z - logsumexp(z)
            for t in range(V):
                allp[p + (t,)] = allp[p] + ls[t]
                nxt.append(p + (t,))
        frontier = nxt
    ranked = sorted((k for k in allp if k), key=lambda k: -allp[k])
    top = set(ranked[:budget - 1])
    got = set(_paths(st)[1:])
    assert max(len(p) for p in got) < D
    assert got == top
    for i, p in enumerate(_paths(st)):
        assert abs(st.logp[i] - allp[p]) < 1e-12


def _heap_rounds(V, Bsel, budget, sigma, seed, rows=None):
    """Independent round simulation: a binary heap over every candidate
    ever generated (no truncation).  rows(path) gives a node's draft
    logits (default: the seeded Gaussian rows)."""
    paths, logp, par, tok = [()], [0.0], [-1], [0]
    heap = []
    frontier = [0]
    while len(paths) < budget and frontier:
        for n in frontier:
            z = rows(paths[n]) if rows else _row(paths[n], V, sigma, seed)
            lz = z - logsumexp(z)
            for t in range(V):
                heapq.heappush(heap, (-(logp[n] + lz[t]), n, t))
        frontier = []
        for _ in range(min(Bsel, budget - len(paths))):
            if not heap:
                break
            s, n, t = heapq.heappop(heap)
            paths.append(paths[n] + (t,))
            logp.append(-s)
            par.append(n)
            tok.append(t)
            frontier.append(len(paths) - 1)
    return par, tok, logp


@pytest.mark.parametrize("V,Bsel,budget,seed", [(5, 3, 40, 0), (8, 4, 61, 1), (3, 7, 50, 2), (16, 8, 64, 3)])
def test_batched_rounds_match_heap_simulation(V, Bsel, budget, seed):
    st = _run(V, Bsel, budget, 1.5, seed)
    par, tok, logp = _heap_rounds(V, Bsel, budget, 1.5, seed)
    assert st.parent == par and st.token == tok
    np.testing.assert_allclose(st.logp, logp, rtol=0, atol=1e-12)
    assert min(st.gaps) > 1e-9     # no near-ties decided these seeds


@pytest.mark.parametrize("V,Bsel,budget", [(2, 3, 40), (3, 1, 30), (4, 5, 50), (5, 2, 33), (7, 16, 64)])
def test_ties_order_by_parent_then_token(V, Bsel, budget):
    def flat(path):
        return np.full(V, 0.25 * len(path))
    st = ExpandState(budget)
    frontier = [0]
    while st.n_nodes < budget and frontier:
        paths = _paths(st)
        frontier = expand_call(st, np.stack([flat(paths[n]) for n in frontier]), frontier, Bsel)
    par, tok, _ = _heap_rounds(V, Bsel, budget, 0.0, 0, rows=flat)
    assert st.parent == par and st.token == tok
    if Bsel == 1:
        k = np.arange(1, budget)
        assert st.parent[1:] == list((k - 1) // V) and st.token[1:] == list((k - 1) % V)


def _beam(V, Bsel, budget, rows):
    """Beam search: each depth keeps the top-Bsel children of the previous
    depth's beam only."""
    paths, logp = [()], [0.0]
    beam = [0]
    while len(paths) < budget and beam:
        cand = []
        for n in beam:
            z = rows(paths[n])
            lz = z - logsumexp(z)
            cand += [(-(logp[n] + lz[t]), n, t) for t in range(V)]
        cand.sort()
        beam = []
        for s, n, t in cand[:min(Bsel, budget - len(paths))]:
            paths.append(paths[n] + (t,))
            logp.append(-s)
            beam.append(len(paths) - 1)
    return paths, logp


def test_differs_from_beam_search():
    V, Bsel, budget = 32, 2, 7
    # root: token 0 has probability ~0.9; every other row is flat, so the
    # root's runners-up beat the grandchildren through token 0
    def rows(path):
        z = np.zeros(V)
        if path == ():
            z[0] = math.log(0.9 * (V - 1) / 0.1)
        return z
    st = ExpandState(budget)
    frontier = [0]
    while st.n_nodes < budget and frontier:
        paths = _paths(st)
        frontier = expand_call(st, np.stack([rows(paths[n]) for n in frontier]), frontier, Bsel)
    bf = set(_paths(st))
    bpaths, blogp = _beam(V, Bsel, budget, rows)
    assert bf != set(bpaths)
    # at Bsel = 1 best-first is the exact top-N, so its mass is maximal
    st1 = ExpandState(budget)
    frontier = [0]
    while st1.n_nodes < budget and frontier:
        paths = _paths(st1)
        frontier = expand_call(st1, np.stack([rows(paths[n]) for n in frontier]), frontier, 1)
    b1paths, b1logp = _beam(V, 1, budget, rows)
    assert sum(np.exp(st1.logp[1:])) > sum(np.exp(b1logp[1:])) + 1e-3


def _golden():
    out = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        case, node, parent, token, prob = line.split()
        out.setdefault(case, []).append((int(node), int(parent), int(token), Fraction(prob)))
    return out


def test_worked_example():
    ln3 = math.log(3.0)
    rows = {(): [0.0, ln3], (1,): [ln3, 0.0], (0,): [0.0, ln3], (1, 0): [0.0, 0.0]}
    g = _golden()
    for case, Bsel, budget in (("A", 1, 4), ("B", 2, 5)):
        st = ExpandState(budget)
        frontier = [0]
        while st.n_nodes < budget and frontier:
            paths = _paths(st)
            frontier = expand_call(st, np.array([rows[paths[n]] for n in frontier]), frontier, Bsel)
        assert st.n_nodes == budget
        for node, parent, token, prob in g[case]:
            assert st.parent[node] == parent and st.token[node] == token
            assert abs(st.logp[node] - math.log(float(prob))) < 1e-15 * 8


def test_bad_rows_and_budget():
    st = ExpandState(4)
    expand_call(st, np.zeros((2, 3)), [0, 5], 2)         # node 5 does not exist
    assert st.status & ST_BAD_ROW and st.n_nodes == 3
    expand_call(st, np.zeros((1, 3)), [0], 2)            # root already expanded
    assert st.n_nodes == 4                               # pool still serves
    assert expand_call(st, np.zeros((1, 3)), [1], 2) == []   # tree full


def test_specexec_sized_invariants():
    V, Bsel, budget = 32000, 128, 2048
    rng_rows = {}

    def logits(call, frontier):
        g = np.random.default_rng(1000 + call)
        return g.normal(0, 4.0, size=(len(frontier), V))
    st = expand_build(budget, Bsel, logits)
    assert st.n_nodes == budget
    par = np.array(st.parent)
    assert par[0] == -1 and np.all(par[1:] < np.arange(1, budget)) and np.all(par[1:] >= 0)
    pairs = set(zip(st.parent[1:], st.token[1:]))
    assert len(pairs) == budget - 1
    lp = np.array(st.logp)
    assert np.all(lp[1:] <= lp[par[1:]] + 1e-12)          # scores only decrease down a path
    # rounds append in non-increasing score order within a round
    for r in range(16):
        lo, hi = 1 + r * Bsel, min(1 + (r + 1) * Bsel, budget)
        assert np.all(np.diff(lp[lo:hi]) <= 0)


def test_nonfinite_row_consumes_its_node():
    """A row holding a non-finite logit adds no candidates, sets the
    NONFINITE bit, and still counts as the node's expansion: the same node
    given again is a bad row.  Rows given alongside it expand normally."""
    from oracle.attention import ST_NONFINITE, ST_BAD_ROW
    st = ExpandState(16)
    z = np.zeros((1, 4))
    z[0, 2] = np.inf
    new = expand_call(st, z, [0], 2)
    assert new == [] and st.n_nodes == 1
    assert st.status & ST_NONFINITE and not st.status & ST_BAD_ROW
    assert 0 in st.expanded
    new = expand_call(st, np.zeros((1, 4)), [0], 2)
    assert new == [] and st.status & ST_BAD_ROW
    # a NaN row next to a finite one: the NaN row's node gets no children
    # (the pool still holds the root's third child), the finite one does
    st = ExpandState(16)
    new = expand_call(st, np.array([[0.0, 1.0, 2.0]]), [0], 2)          # nodes 1, 2 (tokens 2, 1)
    z = np.array([[np.nan, 0.0, 0.0], [5.0, 0.0, 0.0]])
    new = expand_call(st, z, new, 3)
    assert st.status & ST_NONFINITE
    parents = [st.parent[i] for i in new]
    assert 1 not in parents and 2 in parents
    assert 1 in st.expanded and 2 in st.expanded


def _path_rows(V, seed):
    """Draft logits keyed by the node's token path (order-independent)."""
    def rows(path):
        h = (seed * 1_000_003 + hash(path)) % (2 ** 32)
        return np.random.default_rng(h).normal(0.0, 2.0, V)
    return rows


@pytest.mark.parametrize("V,Bsel,budget,seed", [(4, 3, 30, 0), (7, 5, 60, 1), (3, 9, 40, 2), (16, 6, 50, 3)])
def test_beam_mode_matches_beam_search(V, Bsel, budget, seed):
    """Beam mode, round by round with the frontier as the rows, builds the
    tree that an independent path-level beam search builds (each depth keeps
    the best Bsel children of the previous depth)."""
    rows = _path_rows(V, seed)
    st = ExpandState(budget)
    frontier = [0]
    while st.n_nodes < budget and frontier:
        paths = _paths(st)
        frontier = expand_call(st, np.stack([rows(paths[n]) for n in frontier]), frontier, Bsel, mode="beam")
        assert len(st.pool_score) == 0
    bpaths, blogp = _beam(V, Bsel, budget, rows)
    got = _paths(st)
    assert got == bpaths
    np.testing.assert_allclose(st.logp, blogp, rtol=0, atol=1e-12)


def test_beam_mode_with_one_beam_is_greedy_decoding():
    """Bsel = 1: every call appends the single best child of the one
    frontier node, so the tree is the chain of row argmaxes."""
    V, budget = 9, 12
    rows = _path_rows(V, 7)
    st = ExpandState(budget)
    frontier = [0]
    while st.n_nodes < budget and frontier:
        paths = _paths(st)
        frontier = expand_call(st, np.stack([rows(paths[n]) for n in frontier]), frontier, 1, mode="beam")
    path = ()
    for i in range(1, budget):
        assert st.parent[i] == i - 1
        assert st.token[i] == int(np.argmax(rows(path)))
        path = path + (st.token[i],)


def test_beam_mode_never_revisits_an_earlier_depth():
    """With the root's runners-up far better than every grandchild, best
    first takes them in the second round while beam mode does not."""
    V, Bsel, budget = 6, 2, 6

    def rows(path):
        z = np.full(V, -8.0)
        if path == ():
            z[:4] = [3.0, 2.9, 2.8, 2.7]
        return z
    for mode, want_root_children in (("bestfirst", 4), ("beam", 2)):
        st = ExpandState(budget)
        frontier = [0]
        while st.n_nodes < budget and frontier:
            paths = _paths(st)
            frontier = expand_call(st, np.stack([rows(paths[n]) for n in frontier]), frontier, Bsel, mode=mode)
        assert sum(1 for q in st.parent[1:] if q == 0) == want_root_children
