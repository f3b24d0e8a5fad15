"""Pins of the acceptance oracle.

* Temperature 0 on a chain tree accepts the longest prefix of draft tokens
  equal to the successive target argmaxes; on random tiny trees without
  duplicate sibling tokens the walk equals the unique maximal matching path
  found by enumerating every root-to-node path.
* Stochastic acceptance reproduces sequential sampling from the target:
  the walk is enumerated exactly over its uniforms (the decision at each
  draw is a monotone step function of u; its breakpoints are located by
  bisection on the oracle itself) and over all draft-token assignments
  (children drawn i.i.d. from q), and the resulting distribution of the
  first two emitted tokens must equal p(t1) * p(t2 | t1) to 1e-10.
* A Monte-Carlo check of the Philox-driven walk over many seeds.
* Malformed inputs set status bits and keep outputs defined.
"""

import itertools

import numpy as np
import pytest
import torch

from oracle.accept import tree_accept, softmax_t, inverse_cdf, GREEDY, SPECSAMPLE, SPECEXEC
from oracle.attention import ST_BAD_PARENT, ST_BAD_TOKEN, ST_NONFINITE, ST_BAD_LEN
from oracle.philox import TAG_CHILD, TAG_RESIDUAL, TAG_SPECEXEC
from synth import tree_chain, accept_case, tree_random_recursive


# ---------------------------------------------------------------- greedy

def test_greedy_chain_is_longest_matching_prefix():
    rng = np.random.default_rng(0)
    for trial in range(30):
        T, V = 8, 5
        z = rng.normal(size=(1, T, V)).astype(np.float32)
        am = z[0].argmax(-1)
        tok = rng.integers(0, V, size=(1, T))
        m = int(rng.integers(0, T))       # force a matching run of length m
        for i in range(1, m + 1):
            tok[0, i] = am[i - 1]
        o = tree_accept(z, None, tok, tree_chain(T)[None], mode=GREEDY)
        # longest prefix with tok[i+1] == argmax(z[i])
        n = 0
        while n + 1 < T and tok[0, n + 1] == am[n]:
            n += 1
        assert o["n_accepted"][0] == n
        assert list(o["accepted_nodes"][0, :n]) == list(range(1, n + 1))
        assert list(o["out_tokens"][0, :n + 1]) == [int(tok[0, i]) for i in range(1, n + 1)] + [int(am[n])]
        assert np.all(o["out_tokens"][0, n + 1:] == -1)


def test_greedy_matches_path_enumeration_on_random_trees():
    rng = np.random.default_rng(1)
    g = torch.Generator().manual_seed(1)
    done = 0
    while done < 40:
        T, V = 12, 6
        par = tree_random_recursive(T, g)
        kids = {}
        for j in range(1, T):
            kids.setdefault(int(par[j]), []).append(j)
        if max(len(c) for c in kids.values()) > V:
            continue
        done += 1
        # distinct sibling tokens: a random permutation per parent
        tok = np.zeros(T, dtype=np.int64)
        for c, ch in kids.items():
            perm = rng.permutation(V)
            for r, j in enumerate(ch):
                tok[j] = perm[r]
        z = rng.normal(size=(1, T, V)).astype(np.float32)
        # bias rows so that matches happen often
        for j in range(1, T):
            z[0, par[j], tok[j]] += rng.uniform(0, 2.0)
        am = z[0].argmax(-1)
        o = tree_accept(z, None, tok[None], par[None], mode=GREEDY)
        # enumerate all root-to-node paths; a path matches if each node's
        # token is the argmax of its parent's row
        best = []
        for j in range(T):
            path, c = [], j
            while c != 0:
                path.append(c)
                c = int(par[c])
            path = path[::-1]
            if all(tok[x] == am[int(par[x])] for x in path) and len(path) > len(best):
                best = path
        assert list(o["accepted_nodes"][0, :len(best)]) == best
        assert o["n_accepted"][0] == len(best)
        last = best[-1] if best else 0
        assert o["out_tokens"][0, len(best)] == am[last]


def test_greedy_ties_take_lowest_index_and_first_child():
    z = np.zeros((1, 3, 4), np.float32)
    z[0, 0, 1] = z[0, 0, 3] = 2.0          # tie: argmax = 1
    tok = np.array([[0, 1, 1]])
    par = np.array([[-1, 0, 0]])
    o = tree_accept(z, None, tok, par, mode=GREEDY)
    assert o["accepted_nodes"][0, 0] == 1 and o["n_accepted"][0] == 1
    assert o["out_tokens"][0, 1] == 0       # row of node 1 is all zeros: argmax 0


# ------------------------------------------------ exact enumeration (stochastic)

class _Need(Exception):
    pass


def _path_row(path, kind, V, sigma, seed):
    ss = np.random.SeedSequence([seed, kind, len(path)] + [t + 1 for t in path])
    return np.random.default_rng(ss).normal(0.0, sigma, size=V)


def _segments(f, lo=0.0, hi=1.0, eps=1e-14):
    """Maximal intervals of [lo, hi) on which the monotone step function f is
    constant, breakpoints located by bisection."""
    a = f(lo)
    b = f(np.nextafter(hi, 0.0))
    if a == b:
        return [(lo, hi, a)]
    if hi - lo < eps:
        return [(lo, hi, a)]
    mid = 0.5 * (lo + hi)
    left = _segments(f, lo, mid, eps)
    right = _segments(f, mid, hi, eps)
    if left[-1][2] == right[0][2]:
        return left[:-1] + [(left[-1][0], right[0][1], left[-1][2])] + right[1:]
    return left + right


def _decision(res, key):
    node, draw, tag = key
    for e in res["trace"][0]:
        if tag == TAG_CHILD and e[0] == "test" and e[1] == node and e[3] == draw:
            return 0 if e[6] else 1
        if tag == TAG_RESIDUAL and e[0] == "residual" and e[1] == node:
            return e[2]
        if tag == TAG_SPECEXEC and e[0] == "sample" and e[1] == node:
            return e[2]
    raise AssertionError("decision not found")


def _walk_distribution(z, q, tok, par, mode, tau):
    """Exact distribution of the emitted sequence of one tree."""
    out = {}

    def run(fixed, strict):
        def ufn(b, node, draw, tag):
            key = (node, draw, tag)
            if key in fixed:
                return fixed[key]
            if strict:
                raise _Need(key)
            return 0.5
        return tree_accept(z, q, tok, par, mode=mode, temperature=tau, uniform_fn=ufn)

    def explore(fixed, w):
        try:
            res = run(fixed, True)
        except _Need as e:
            key = e.args[0]

            def f(u):
                return _decision(run({**fixed, key: u}, False), key)
            for lo, hi, _ in _segments(f):
                explore({**fixed, key: 0.5 * (lo + hi)}, w * (hi - lo))
            return
        n = int(res["n_accepted"][0])
        seq = tuple(int(t) for t in res["out_tokens"][0, :n + 1])
        out[seq] = out.get(seq, 0.0) + w

    explore({}, 1.0)
    return out


def _check_lossless(par, V, tau, mode, seed=0, sigma=1.0):
    """Sum the exact walk distribution over all i.i.d. draft assignments
    and compare the first two emitted tokens with sequential sampling from
    the path-keyed target."""
    T = len(par)
    kids_order = list(range(1, T))
    tau = float(np.float32(tau))        # the walk takes an fp32 temperature

    def target_p(path):
        return softmax_t(_path_row(path, 1, V, sigma, seed), tau)

    def draft_q(path):
        return softmax_t(_path_row(path, 2, V, sigma, seed), tau)

    P1 = np.zeros(V)
    P2 = np.zeros((V, V))
    assignments = itertools.product(range(V), repeat=T - 1)
    for assign in assignments:
        tok = np.zeros(T, dtype=np.int64)
        tok[1:] = assign
        paths = [()]
        for j in range(1, T):
            paths.append(paths[par[j]] + (int(tok[j]),))
        w = 1.0
        if mode == SPECSAMPLE:
            for j in kids_order:
                w *= draft_q(paths[par[j]])[tok[j]]
        z = np.stack([_path_row(paths[c], 1, V, sigma, seed) for c in range(T)])[None].astype(np.float64)
        q = np.stack([draft_q(paths[c]) for c in range(T)])[None]
        dist = _walk_distribution(z, q, tok[None], np.asarray(par)[None], mode, tau)
        for seq, pw in dist.items():
            P1[seq[0]] += w * pw
            if len(seq) >= 2:
                P2[seq[0], seq[1]] += w * pw
            else:
                P2[seq[0]] += w * pw * target_p((seq[0],))
        if mode == SPECEXEC:
            break                      # deterministic tree: one assignment
    p0 = target_p(())
    np.testing.assert_allclose(P1, p0, rtol=0, atol=1e-10)
    ref2 = np.stack([p0[a] * target_p((a,)) for a in range(V)])
    np.testing.assert_allclose(P2, ref2, rtol=0, atol=1e-10)


@pytest.mark.parametrize("par,V,tau", [
    ([-1, 0, 0], 3, 0.8),           # two i.i.d. children of the root
    ([-1, 0, 0, 1], 3, 1.3),        # plus a grandchild
    ([-1, 0, 0, 0], 3, 0.7),        # three children (two residual updates)
    ([-1, 0, 1], 4, 1.0),           # chain of two
])
def test_specsample_reproduces_sequential_sampling(par, V, tau):
    _check_lossless(par, V, tau, SPECSAMPLE, seed=len(par) * 10 + V)


@pytest.mark.parametrize("par,V,tau", [([-1, 0, 0, 1], 3, 0.6), ([-1, 0, 1, 0], 4, 1.0)])
def test_specexec_reproduces_sequential_sampling(par, V, tau):
    _check_lossless(par, V, tau, SPECEXEC, seed=3)


def test_monte_carlo_first_token_distribution():
    """The Philox-driven walk: first emitted token over 4000 seeds versus the
    target distribution of the root (chi-square)."""
    V, T = 6, 5
    par = np.array([-1, 0, 0, 1, 1])
    case = accept_case(1, T, V, par, 0.9, sigma=1.0, seed=5, correlated=True, noise=0.7)
    z, q = case.target_logits, case.draft_probs
    qn = q[0].double().numpy()
    rng = np.random.default_rng(0)
    counts = np.zeros(V)
    n = 4000
    for s in range(n):
        # a fresh sampled tree per trial: children i.i.d. from q of the parent
        tok = np.zeros((1, T), dtype=np.int64)
        for j in range(1, T):
            tok[0, j] = rng.choice(V, p=qn[par[j]] / qn[par[j]].sum())
        o = tree_accept(z, q, tok, par[None], mode=SPECSAMPLE, temperature=0.9, seed=s)
        counts[o["out_tokens"][0, 0]] += 1
    p = softmax_t(z[0, 0].double().numpy(), 0.9)
    chi2 = np.sum((counts - n * p) ** 2 / (n * p))
    assert chi2 < 25.7       # 5 dof, p ~ 1e-4


# ---------------------------------------------------------------- helpers

def test_inverse_cdf_definition():
    p = np.array([0.1, 0.0, 0.3, 0.6])
    assert inverse_cdf(p, 0.0)[0] == 0
    assert inverse_cdf(p, 0.0999)[0] == 0
    assert inverse_cdf(p, 0.1)[0] == 2          # strict ">" skips the zero token
    assert inverse_cdf(p, 0.3999)[0] == 2
    assert inverse_cdf(p, 0.4001)[0] == 3
    assert inverse_cdf(p, 1 - 2**-53)[0] == 3


def test_temperature_zero_is_greedy_in_every_mode():
    case = accept_case(2, 7, 9, tree_random_recursive(7, torch.Generator().manual_seed(3)), 0.0,
                       seed=2, correlated=True, child_rule="top")
    ref = tree_accept(case.target_logits, None, case.draft_tokens, case.parent, mode=GREEDY)
    for mode in (SPECSAMPLE, SPECEXEC, "auto"):
        o = tree_accept(case.target_logits, case.draft_probs, case.draft_tokens, case.parent,
                        mode=mode, temperature=0.0)
        np.testing.assert_array_equal(o["out_tokens"], ref["out_tokens"])


def test_malformed_inputs_set_status():
    V = 4
    z = np.zeros((1, 4, V), np.float32)
    z[0, 0, 2] = 1.0
    tok = np.array([[0, 7, 2, 1]])             # node 1 carries token 7 >= V
    par = np.array([[-1, 0, 0, 3]])            # parent[3] = 3 is invalid
    o = tree_accept(z, None, tok, par, mode=GREEDY)
    assert o["status"] & ST_BAD_TOKEN and o["status"] & ST_BAD_PARENT
    assert o["accepted_nodes"][0, 0] == 2
    z2 = z.copy()
    z2[0, 2, 1] = np.nan
    o = tree_accept(z2, None, tok, par, mode=GREEDY)
    assert o["status"] & ST_NONFINITE and o["out_tokens"][0, 1] == -1
    o = tree_accept(z, None, tok, par, n_nodes=np.array([5]), mode=GREEDY)
    assert o["status"] & ST_BAD_LEN and o["n_accepted"][0] == 0
    o = tree_accept(z, None, tok, par, n_nodes=np.array([0]), mode=GREEDY)
    assert o["status"] == 0 and np.all(o["out_tokens"] == -1)
