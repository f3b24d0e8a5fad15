"""tree_accept_noalloc, the acceptance entry point for callers that cannot
allocate device memory (their memory belongs to a runtime that reserved it
up front, or cudaMalloc's device-wide synchronisation is not allowed where
they run).  It must give exactly what tree_accept gives on the same inputs,
call after call: its scratch is a fixed array inside the library that every
call reuses.  Collected last so that a failure here leaves every other test
already run."""

import ctypes

import numpy as np
import pytest
import torch

from synth import accept_case, config_accept_case, tree_random_recursive

pytestmark = pytest.mark.gpu


def _cases():
    yield config_accept_case("tiny", temperature=0.8, seed=1, correlated=True, device="cuda")
    par = tree_random_recursive(40, torch.Generator().manual_seed(7))
    yield accept_case(3, 40, 5000, par, 0.7, sigma=2.0, seed=4, correlated=True, noise=0.3, device="cuda")
    yield config_accept_case("tiny", temperature=0.0, seed=2, correlated=True, device="cuda")


def _via_c_abi(case):
    """Call tree_accept_noalloc through the C ABI directly."""
    import tree_verification_verify_b200 as tv
    z, q, tok, par = case.target_logits, case.draft_probs, case.draft_tokens, case.parent
    B, T, V = z.shape
    out = dict(n_accepted=torch.full((B,), -7, dtype=torch.int32, device="cuda"),
               accepted_nodes=torch.full((B, T), -7, dtype=torch.int32, device="cuda"),
               out_tokens=torch.full((B, T + 1), -7, dtype=torch.int32, device="cuda"),
               min_margin=torch.zeros(B, dtype=torch.float64, device="cuda"))
    a = tv.AcceptArgs(B, T, V, z.data_ptr(), z.stride(0), z.stride(1),
                      q.data_ptr() if q is not None else None, q.stride(0) if q is not None else 0,
                      q.stride(1) if q is not None else 0,
                      tok.data_ptr(), tok.stride(0), par.data_ptr(), par.stride(0), None,
                      tv.MODES[case.mode], float(case.temperature), case.seed, case.step,
                      out["n_accepted"].data_ptr(), out["accepted_nodes"].data_ptr(),
                      out["out_tokens"].data_ptr(), out["min_margin"].data_ptr(), None)
    rc = tv.lib().tree_accept_noalloc(ctypes.byref(a), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, tv.status_string(rc)
    return out


def test_noalloc_matches_tree_accept_on_consecutive_calls():
    import tree_verification_verify_b200 as tv
    from tree_verification_verify_b200 import build
    build.build()
    for case in _cases():
        ref = tv.tree_accept(case.target_logits, case.draft_tokens, case.parent, draft_probs=case.draft_probs,
                             mode=case.mode, temperature=case.temperature, seed=case.seed, step=case.step)
        for _ in range(2):                        # two calls in a row on the shared scratch
            got = _via_c_abi(case)
            torch.cuda.synchronize()
            for k in ("n_accepted", "accepted_nodes", "out_tokens"):
                assert torch.equal(got[k].cpu(), ref[k].cpu()), k
            np.testing.assert_allclose(got["min_margin"].cpu().numpy(), ref["min_margin"].cpu().numpy(),
                                       rtol=0, atol=1e-12)


def test_noalloc_rejects_sizes_past_its_scratch():
    import tree_verification_verify_b200 as tv
    a = tv.AcceptArgs()
    a.B, a.T, a.V, a.mode = 200, 200, 4, 1               # 40000 rows > 32768
    a.target_logits = a.draft_tokens = a.parent = a.n_accepted = a.accepted_nodes = a.out_tokens = 16
    a.tl_st = 4
    assert tv.lib().tree_accept_noalloc(ctypes.byref(a), None) == 2
