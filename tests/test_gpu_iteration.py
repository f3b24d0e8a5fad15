"""The whole speculative iteration (tree_verification_verify_b200.loop):
expansion from a random-weight drafter stand-in, a target attention layer
through tree_verify_attn, tree_accept and tree_commit_kv chained on the
device and replayed from one CUDA graph.

Checked against the oracle per step on the step's own inputs (the stand-in
models' rows, which torch computes, are inputs here, not outputs of this
library): the tree against oracle expansion of the recorded drafter rows,
the walk against the oracle walk on the target rows, the commit against the
oracle commit; then that graph replays reproduce eager iterations exactly
(every call is deterministic)."""

import numpy as np
import pytest
import torch

from oracle.accept import tree_accept as o_accept, SPECEXEC
from oracle.commit import tree_commit_kv as o_commit
from oracle.expand import ExpandState as OState, expand_call

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tree_verification_verify_b200 import build
    build.build()


def _make(seed=0, **kw):
    from tree_verification_verify_b200.loop import Iteration
    return Iteration(torch.device("cuda", 0), prefix=1000, budget=64, Bsel=16, V=4096, hidden=512,
                     iters_room=16, seed=seed, **kw)


def test_one_iteration_matches_oracle():
    it = _make()
    for i in range(3):
        it.record = []
        root = int(it.root.item())
        L0 = int(it.prefix_len.item())
        kc0, vc0 = it.kc.clone(), it.vc.clone()
        it.step()
        torch.cuda.synchronize()
        assert int(it.status.item()) == 0

        # the tree: oracle expansion of the same drafter rows
        os_ = OState(it.budget, root)
        for rows, z in it.record:
            nap = len(os_.parent)
            expand_call(os_, z.cpu(), rows.cpu(), it.Bsel)
            assert os_.gaps[-1] > 1e-10, "near-tie in the draft ranking"
        n = int(it.st.n_nodes.item())
        assert n == it.budget == len(os_.parent)
        assert it.st.parent.cpu().tolist() == os_.parent
        assert it.st.token.cpu().tolist() == os_.token

        # the walk: oracle SpecExec walk on the target rows
        T = it.budget
        par = torch.tensor(os_.parent, dtype=torch.int32).view(1, T)
        tok = torch.tensor(os_.token, dtype=torch.int32).view(1, T)
        ref = o_accept(it.target_logits.cpu(), None, tok, par, mode=SPECEXEC, temperature=it.temperature,
                       seed=1234, step=0)
        o = it.acc_out
        if ref["min_margin"][0] >= 1e-6:
            assert o["n_accepted"].cpu().tolist() == ref["n_accepted"].tolist()
            assert o["out_tokens"].cpu().numpy()[0].tolist() == ref["out_tokens"][0].tolist()
        na = int(o["n_accepted"].item())
        path = o["accepted_nodes"].cpu().numpy()[0][:na].tolist()
        prev = 0
        for j in path:                       # a root-to-node chain of the tree
            assert os_.parent[j] == prev
            prev = j

        # the commit: root then the accepted nodes appended, prefix advanced
        rc = o_commit(kc0.cpu(), vc0.cpu(), torch.tensor([L0], dtype=torch.int32), it.kt.cpu(), it.vt.cpu(),
                      o["n_accepted"].cpu(), o["accepted_nodes"].cpu())
        assert int(it.prefix_len.item()) == int(rc["prefix_len"][0]) == L0 + na + 1
        rows = slice(L0, L0 + na + 1)
        assert np.array_equal(it.kc[0, rows].double().cpu().numpy(), rc["k_cache"][0, rows])
        assert np.array_equal(it.vc[0, rows].double().cpu().numpy(), rc["v_cache"][0, rows])
        assert int(it.root.item()) == int(o["out_tokens"][0, na].item())
    print(f"emitted {int(it.emitted.item())} tokens in 3 iterations")


def test_graph_replay_equals_eager():
    a, b = _make(seed=3), _make(seed=3)
    for _ in range(4):
        a.step()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        b.step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        b.step()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert int(a.status.item()) == int(b.status.item()) == 0
    assert int(a.prefix_len.item()) == int(b.prefix_len.item())
    assert int(a.root.item()) == int(b.root.item())
    assert int(a.emitted.item()) == int(b.emitted.item())
    assert torch.equal(a.kc, b.kc) and torch.equal(a.vc, b.vc)
    assert torch.equal(a.st.parent, b.st.parent) and torch.equal(a.st.token, b.st.token)
    del g
