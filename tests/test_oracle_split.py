"""Splitting a long prefix into slices (one per GPU), attending to each slice
alone (prefix-only partials, the tree keys counted in one slice) and merging
the partials by log-sum-exp gives the tree attention over the whole prefix.
Host only: the oracle's partials and merge against its full attention (which
is pinned elsewhere against causal attention and the explicit ancestor
mask), and the exchange across two gloo ranks."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle.attention import tree_verify_attn, merge_partials
from synth import attn_case, tree_random_recursive, tree_bfs_fanout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _slice_case(case, lo, hi):
    """The inputs a rank holding prefix rows [lo, hi) passes: its cache
    slice and the slice's length per sequence."""
    L = case.prefix_len.numpy()
    pl = np.clip(L - lo, 0, hi - lo).astype(np.int32)
    return case.k_cache[:, lo:hi], case.v_cache[:, lo:hi], torch.from_numpy(pl)


def _split_attention(case, bounds):
    outs, lses = [], []
    for r in range(len(bounds) - 1):
        kc, vc, pl = _slice_case(case, bounds[r], bounds[r + 1])
        last = r == len(bounds) - 2
        o = tree_verify_attn(case.q, kc, vc, pl, case.k_tree, case.v_tree, case.parent, n_nodes=case.n_nodes,
                             prefix_only=not last)
        outs.append(o["out"])
        lses.append(o["lse"])
    return merge_partials(outs, lses)


@pytest.mark.parametrize("bounds", [[0, 40, 200], [0, 7, 90, 91, 200], [0, 200, 200], [0, 1, 2, 3, 200]])
def test_merged_slices_equal_tree_attention(bounds):
    T = 9
    case = attn_case(3, T, 8, 2, 32, [150, 0, 200], "fp32", tree_random_recursive(T, torch.Generator().manual_seed(3)),
                     seed=2)
    full = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len, case.k_tree, case.v_tree,
                            case.parent)
    out, lse = _split_attention(case, bounds)
    np.testing.assert_allclose(out, full["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, full["lse"], rtol=0, atol=1e-12)


def test_prefix_only_of_an_empty_slice():
    T = 5
    case = attn_case(2, T, 4, 1, 32, [0, 10], "fp32", tree_bfs_fanout(T, (2,)), seed=4)
    o = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len, case.k_tree, case.v_tree,
                         case.parent, prefix_only=True)
    assert np.all(o["out"][0] == 0.0) and np.all(o["lse"][0] == -np.inf)
    assert np.all(np.isfinite(o["out"][1]))
    # parent[] is not read: a malformed tree changes nothing
    bad = case.parent.clone()
    bad[:, 3] = 4
    o2 = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len, case.k_tree, case.v_tree, bad,
                          prefix_only=True)
    assert o2["status"] == 0
    np.testing.assert_array_equal(o2["out"], o["out"])


def test_merge_partials_identities():
    rng = np.random.default_rng(0)
    o = rng.normal(size=(2, 3, 4))
    lse = rng.normal(size=(2, 3))
    out, l = merge_partials([o[0]], [lse[0]])
    np.testing.assert_allclose(out, o[0], atol=1e-15)
    np.testing.assert_allclose(l, lse[0], atol=1e-15)
    ninf = np.full((2, 3), -np.inf)
    out, l = merge_partials([o[0], np.zeros_like(o[0])], [lse[0], ninf[0]])
    np.testing.assert_allclose(out, o[0], atol=1e-15)
    out, l = merge_partials([np.zeros_like(o[0])], [ninf[0]])
    assert np.all(out == 0.0) and np.all(l == -np.inf)
    nan = lse[0].copy()
    nan[1] = np.nan
    out, l = merge_partials([o[0], o[1]], [nan, lse[1]])
    assert np.all(np.isnan(out[1])) and np.isnan(l[1]) and np.all(np.isfinite(out[0]))
    # two partials: the weights are their softmax masses
    out, l = merge_partials([o[0], o[1]], [lse[0], lse[1]])
    w0 = np.exp(lse[0]) / (np.exp(lse[0]) + np.exp(lse[1]))
    np.testing.assert_allclose(out, w0[:, None] * o[0] + (1 - w0)[:, None] * o[1], atol=1e-12)
    np.testing.assert_allclose(l, np.logaddexp(lse[0], lse[1]), atol=1e-12)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    import sys
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    from oracle.attention import tree_verify_attn as attn, merge_partials as merge
    from synth import attn_case, tree_bfs_fanout
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    T = 13
    case = attn_case(2, T, 8, 2, 32, [333, 120], "fp32", tree_bfs_fanout(T, (3, 2)), seed=7)
    from tree_verification_verify_b200.split import prefix_slice, slice_prefix_len
    Lmax = case.k_cache.shape[1]
    lo, hi = prefix_slice(rank, world, Lmax)       # the partition the GPU split uses
    pl = slice_prefix_len(case.prefix_len, lo, hi)
    part = attn(case.q, case.k_cache[:, lo:hi], case.v_cache[:, lo:hi], pl, case.k_tree, case.v_tree, case.parent,
                prefix_only=(rank != world - 1))
    o = torch.from_numpy(np.nan_to_num(part["out"], nan=0.0))
    lse = torch.from_numpy(part["lse"])
    go = [torch.empty_like(o) for _ in range(world)]
    gl = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(go, o)
    dist.all_gather(gl, lse)
    out, l = merge([x.numpy() for x in go], [x.numpy() for x in gl])
    full = attn(case.q, case.k_cache, case.v_cache, case.prefix_len, case.k_tree, case.v_tree, case.parent)
    err = max(float(np.max(np.abs(out - full["out"]))), float(np.max(np.abs(l - full["lse"]))))
    q.put((rank, err))
    dist.destroy_process_group()


def test_two_ranks_gather_and_merge():
    """Each of two gloo ranks attends to its slice of the prefix (the
    partition of tree_verification_verify_b200.split; the last rank with the
    tree keys), the partials are all-gathered, and every rank merges them
    into the full tree attention."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _ in res] == [0, 1]
    assert all(e < 1e-12 for _, e in res), res


def test_prefix_slices_partition_the_cache():
    """The split's slices cover [0, Lmax) in rank order without overlap,
    sizes within one row; each sequence's keys are counted once."""
    from tree_verification_verify_b200.split import prefix_slice, slice_prefix_len
    for Lmax in (0, 1, 7, 333, 131072):
        for world in (1, 2, 3, 8):
            sl = [prefix_slice(r, world, Lmax) for r in range(world)]
            assert sl[0][0] == 0 and sl[-1][1] == Lmax
            assert all(sl[r][1] == sl[r + 1][0] for r in range(world - 1))
            sizes = [hi - lo for lo, hi in sl]
            assert max(sizes) - min(sizes) <= 1
            L = torch.tensor([0, min(1, Lmax), Lmax // 2, Lmax], dtype=torch.int32)
            tot = sum(slice_prefix_len(L, lo, hi).to(torch.int64) for lo, hi in sl)
            assert torch.equal(tot, L.to(torch.int64))

