"""GPU parity of tree_accept against the fp64 oracle (through the C ABI).

Paths, accepted node lists and emitted tokens must be identical; a sequence
whose oracle walk met a decision within 1e-6 of its threshold is counted as
near-threshold and only checked for validity.  Sizes run from a few nodes
(ties, ragged vocabularies, malformed input) to the full workloads of the
named configurations."""

import numpy as np
import pytest
import torch

from oracle.accept import tree_accept as oracle_accept
from oracle.attention import ST_BAD_PARENT, ST_BAD_TOKEN, ST_NONFINITE, ST_BAD_LEN
from synth import (accept_case, config_accept_case, tree_binary, tree_random_recursive,
                   tree_star, tree_chain, tree_bfs_fanout, CONFIGS)
from parity_util import check_accept, cuda, near_allowed

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tree_verification_verify_b200 import build
    build.build()


def _run(case, mode=None, n_nodes=None):
    import tree_verification_verify_b200 as tv
    mode = mode or case.mode
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nn = n_nodes if n_nodes is not None else case.n_nodes
    g = tv.tree_accept(cuda(case.target_logits), cuda(case.draft_tokens), cuda(case.parent),
                       draft_probs=cuda(case.draft_probs), n_nodes=cuda(nn), mode=mode,
                       temperature=case.temperature, seed=case.seed, step=case.step, dev_status=st)
    torch.cuda.synchronize()
    o = oracle_accept(case.target_logits, case.draft_probs, case.draft_tokens, case.parent, nn,
                      mode=mode, temperature=case.temperature, seed=case.seed, step=case.step)
    return g, o, int(st.item())


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("temperature", [0.0, 0.8])
@pytest.mark.parametrize("correlated", [False, True])
def test_tiny(seed, temperature, correlated):
    case = config_accept_case("tiny", temperature=temperature, seed=seed, correlated=correlated)
    g, o, st = _run(case)
    exact, near = check_accept(g, o, case.parent, case.target_logits.shape[1], V=case.target_logits.shape[2],
                               draft_tokens=case.draft_tokens, what="tiny")
    assert st == o["status"] == 0
    assert near <= near_allowed(1) and exact == 1


@pytest.mark.parametrize("V", [1, 3, 5, 257, 1000])
@pytest.mark.parametrize("mode,temperature", [("greedy", 0.0), ("specsample", 0.9), ("specexec", 1.1)])
def test_ragged_vocab_and_random_trees(V, mode, temperature):
    gen = torch.Generator().manual_seed(V)
    T, B = 19, 5
    parents = [tree_random_recursive(T, gen) for _ in range(B)]
    rule = "top" if mode == "specexec" else "sample"
    if rule == "top":
        # deterministic trees need enough distinct tokens per parent
        parents = [tree_chain(T) for _ in range(B)] if V < 8 else parents
    case = accept_case(B, T, V, parents, temperature, sigma=2.0, seed=V + 7, correlated=True,
                       child_rule=rule, mode=mode, with_q=(mode == "specsample"), noise=0.3)
    g, o, st = _run(case)
    exact, near = check_accept(g, o, case.parent, T, V=V, draft_tokens=case.draft_tokens, what=f"V={V} {mode}")
    assert st == o["status"]
    assert near <= near_allowed(B) and exact == B - near


def test_greedy_ties_pick_lowest_index():
    B, T, V = 3, 9, 16
    par = tree_binary(T)
    z = torch.zeros(B, T, V)
    z[:, :, 3] = 1.0
    z[:, :, 11] = 1.0            # tie with token 3
    z[1] = torch.round(torch.randn(T, V, generator=torch.Generator().manual_seed(1)))
    tok = torch.full((B, T), 3, dtype=torch.int32)
    case = accept_case(B, T, V, par, 0.0, seed=0)
    case.target_logits = z
    case.draft_tokens = tok
    g, o, st = _run(case, mode="greedy")
    check_accept(g, o, case.parent, T)
    assert g["n_accepted"][0].item() == 3     # always the first child (node 1, 3, 7)


def test_node_counts_and_empty_trees():
    T, V = 12, 40
    par = tree_random_recursive(T, torch.Generator().manual_seed(4))
    case = accept_case(4, T, V, par, 0.7, seed=3, correlated=True, noise=0.2)
    nn = torch.tensor([12, 5, 1, 0], dtype=torch.int32)
    g, o, st = _run(case, mode="specsample", n_nodes=nn)
    check_accept(g, o, case.parent, T)
    assert st == o["status"] == 0
    assert g["n_accepted"][3].item() == 0 and torch.all(g["out_tokens"][3] == -1)
    bad = torch.tensor([12, 13, 5, -1], dtype=torch.int32)
    g, o, st = _run(case, mode="specsample", n_nodes=bad)
    assert st & ST_BAD_LEN and o["status"] & ST_BAD_LEN
    assert g["n_accepted"][1].item() == 0 and torch.all(g["out_tokens"][1] == -1)


def test_malformed_input_status():
    T, V = 8, 10
    par = np.array([-1, 0, 0, 1, 3, 7, 2, 2], np.int32)      # parent[5] = 7 >= 5
    case = accept_case(2, T, V, par, 0.0, seed=5, correlated=True, child_rule="top")
    case.draft_tokens[0, 6] = V + 3                          # bad token
    g, o, st = _run(case, mode="greedy")
    check_accept(g, o, case.parent, T)
    assert st == o["status"] and st & ST_BAD_PARENT and st & ST_BAD_TOKEN
    # NaN on a row the walk visits vs a row it does not
    case2 = accept_case(1, T, V, tree_chain(T), 0.0, seed=6, correlated=True, child_rule="top", noise=0.0)
    case2.target_logits[0, 6, 2] = float("nan")
    g, o, st = _run(case2, mode="greedy")
    check_accept(g, o, case2.parent, T)
    assert (st & ST_NONFINITE) == (o["status"] & ST_NONFINITE)
    case2.target_logits[0, 0, 1] = float("nan")             # the root row
    g, o, st = _run(case2, mode="greedy")
    assert st & ST_NONFINITE and g["out_tokens"][0, 0].item() == -1 and o["out_tokens"][0, 0] == -1


def test_many_children_residual_chain():
    """A root with 300 sampled children: up to 300 residual passes."""
    T, V = 301, 64
    case = accept_case(1, T, V, tree_star(T), 1.0, sigma=1.0, seed=8, correlated=False)
    g, o, st = _run(case, mode="specsample")
    exact, near = check_accept(g, o, case.parent, T, V=V, draft_tokens=case.draft_tokens, what="star 300")
    assert near <= near_allowed(1) and exact == 1


def test_specexec_on_expansion_shaped_tree():
    """Deterministic tree (distinct top tokens per parent), temperature 0.6,
    V = 32000, 600 nodes of a random recursive tree."""
    T, V = 600, 32000
    par = tree_random_recursive(T, torch.Generator().manual_seed(9))
    case = accept_case(1, T, V, par, 0.6, sigma=4.0, seed=10, correlated=True, child_rule="top",
                       mode="specexec", with_q=False, noise=0.5)
    g, o, st = _run(case)
    exact, near = check_accept(g, o, case.parent, T, V=V, draft_tokens=case.draft_tokens, what="specexec 600")
    assert near <= near_allowed(1) and exact == 1


@pytest.mark.parametrize("name,temperature,correlated", [
    ("llama3_8b", 0.8, False), ("llama3_8b", 0.8, True),
    ("serving", 0.8, False), ("serving", 0.8, True),
    ("longctx", 0.0, True),
])
def test_full_size_configs(name, temperature, correlated):
    c = CONFIGS[name]
    case = config_accept_case(name, temperature=temperature, seed=0, correlated=correlated)
    g, o, st = _run(case)
    exact, near = check_accept(g, o, case.parent, c["T"], V=c["V"], draft_tokens=case.draft_tokens, what=name)
    assert near <= near_allowed(c["B"]) and exact == c["B"] - near
    assert st == o["status"] == 0
    if correlated:
        assert int(g["n_accepted"].sum()) > 0


@pytest.mark.parametrize("temperature,mode", [(0.0, "greedy"), (0.6, "specexec")])
def test_specexec70b_accept(temperature, mode):
    c = CONFIGS["specexec70b"]
    par = tree_random_recursive(c["T"], torch.Generator().manual_seed(11))
    case = accept_case(1, c["T"], c["V"], par, temperature, sigma=4.0, seed=1, correlated=True,
                       child_rule="top", mode=mode, with_q=False)
    g, o, st = _run(case)
    exact, near = check_accept(g, o, case.parent, c["T"], V=c["V"], draft_tokens=case.draft_tokens,
                               what=f"specexec70b {mode}")
    assert near <= near_allowed(1) and exact == 1


@pytest.mark.parametrize("V,noise", [(6, 0.7), (600, 1.5)])
def test_first_token_distribution_over_many_sequences(V, noise):
    """Speculative sampling is lossless: over sequences whose children are
    drawn i.i.d. from q, the first emitted token (the accepted child's token,
    else the residual sample) follows softmax(z_root / tau) exactly (SpecExec
    page, "Builds on": speculative sampling reproduces the target's
    distribution).  One call carries 16384 sequences, each with its own
    Philox stream; 8 seeds give 131072 samples, compared with the closed form
    by a chi-square test (bins with an expected count below 40 pooled).  V =
    600 runs two-CTA clusters and residual passes over two segments."""
    import scipy.stats
    import tree_verification_verify_b200 as tv
    tau, T, B = 0.9, 5, 16384
    par = np.array([-1, 0, 0, 0, 1], dtype=np.int32)
    base = accept_case(1, T, V, par, tau, sigma=1.0, seed=21, correlated=True, noise=noise)
    z = base.target_logits.expand(B, T, V).contiguous().cuda()
    q = base.draft_probs.expand(B, T, V).contiguous().cuda()
    parent = torch.from_numpy(np.broadcast_to(par, (B, T)).copy()).cuda()
    qd = base.draft_probs[0].double()
    gen = torch.Generator().manual_seed(22)
    p = torch.softmax(base.target_logits[0, 0].double() / float(np.float32(tau)), -1).numpy()
    counts = np.zeros(V)
    rounds = 8
    for s in range(rounds):
        tok = torch.zeros(B, T, dtype=torch.int32)
        for j in range(1, T):
            tok[:, j] = torch.multinomial(qd[par[j]], B, replacement=True, generator=gen).to(torch.int32)
        g = tv.tree_accept(z, tok.cuda(), parent, draft_probs=q, mode="specsample", temperature=tau,
                           seed=1000 + s, step=0)
        first = g["out_tokens"][:, 0].cpu().numpy()
        assert first.min() >= 0 and first.max() < V
        counts += np.bincount(first, minlength=V)
    n = rounds * B
    expect = n * p
    big = expect >= 40.0
    obs = np.append(counts[big], counts[~big].sum())
    exp = np.append(expect[big], expect[~big].sum())
    if exp[-1] == 0.0:
        obs, exp = obs[:-1], exp[:-1]
    chi2 = float(np.sum((obs - exp) ** 2 / exp))
    dof = len(obs) - 1
    assert chi2 < scipy.stats.chi2.isf(1e-4, dof), (chi2, dof)
