"""Pins of the KV-commit oracle against what the method fixes.

* Commit, then decode: after the accepted path is appended to the cache, the
  next token's single-node attention over the new prefix equals the tree
  attention of that token placed as a child of the last accepted node over
  the old prefix (both through the attention oracle, which never sees the
  commit): the appended rows are the path's rows, for K and V.  Attention
  does not see the order of its keys; positions do: the tree pass places
  node i at prefix_len + depth(i), so cache row L + r must hold the path
  node of depth r.
* A chain tree accepted whole appends the tree rows 0 .. T-1 in order.
* A tree stored in the cache right after the prefix is compacted in place:
  the same result as with the tree in its own arrays.
* Malformed paths and lengths leave the sequence untouched and set the
  status bits.
"""

import numpy as np
import pytest
import torch

from oracle.attention import tree_verify_attn
from oracle.commit import tree_commit_kv, ST_BAD_LEN, ST_BAD_ROW
from synth import tree_chain, tree_depths, tree_random_recursive


def _root_path(parent_row, x):
    """Nodes root .. x, root included."""
    p = [x]
    while p[-1] != 0:
        p.append(int(parent_row[p[-1]]))
    return p[::-1]


def _rand(shape, rng):
    return rng.standard_normal(shape)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_commit_then_decode_equals_tree_attention(seed):
    rng = np.random.default_rng(seed)
    B, T, Hq, Hkv, d, Lmax = 3, 12, 4, 2, 16, 40
    L = np.array([20, 7, 0])
    par = np.stack([tree_random_recursive(T, torch.Generator().manual_seed(seed * 10 + b)) for b in range(B)])
    kc, vc = _rand((B, Lmax, Hkv, d), rng), _rand((B, Lmax, Hkv, d), rng)
    kt, vt = _rand((B, T, Hkv, d), rng), _rand((B, T, Hkv, d), rng)
    # accepted paths: to a random node (b = 0, 2), the root alone (b = 1)
    acc = np.full((B, T), -1)
    n = np.zeros(B, dtype=np.int64)
    last = np.zeros(B, dtype=np.int64)
    for b in range(B):
        if b == 1:
            continue
        x = int(rng.integers(1, T))
        path = _root_path(par[b], x)[1:]
        n[b] = len(path)
        acc[b, :len(path)] = path
        last[b] = path[-1]
    com = tree_commit_kv(kc, vc, L, kt, vt, n, acc)
    assert com["status"] == 0
    assert list(com["prefix_len"]) == list(L + n + 1)
    # positions: row L + r holds the path node whose depth is r
    for b in range(B):
        dep = tree_depths(par[b])
        on_path = [0] + list(acc[b, :n[b]])
        for r in range(n[b] + 1):
            (x,) = [j for j in on_path if dep[j] == r]
            np.testing.assert_array_equal(com["k_cache"][b, L[b] + r], kt[b, x])
            np.testing.assert_array_equal(com["v_cache"][b, L[b] + r], vt[b, x])
    # the next token: its query, key and value
    qn, kn, vn = _rand((B, 1, Hq, d), rng), _rand((B, 1, Hkv, d), rng), _rand((B, 1, Hkv, d), rng)
    # route 1: a child of the last accepted node in the old tree, old prefix
    par2 = np.concatenate([par, last[:, None]], axis=1)
    q2 = np.zeros((B, T + 1, Hq, d))
    q2[:, T] = qn[:, 0]
    kt2, vt2 = np.concatenate([kt, kn], axis=1), np.concatenate([vt, vn], axis=1)
    r1 = tree_verify_attn(q2, kc, vc, L, kt2, vt2, par2, rows={(b, T) for b in range(B)})
    # route 2: a one-node tree over the committed cache
    r2 = tree_verify_attn(qn, com["k_cache"], com["v_cache"], com["prefix_len"], kn, vn,
                          np.full((B, 1), -1))
    np.testing.assert_allclose(r2["out"][:, 0], r1["out"][:, T], rtol=0, atol=1e-12)
    np.testing.assert_allclose(r2["lse"][:, 0], r1["lse"][:, T], rtol=0, atol=1e-12)


def test_chain_accepted_whole_appends_the_tree_in_order():
    rng = np.random.default_rng(3)
    B, T, Hkv, d, Lmax = 2, 9, 3, 8, 30
    L = np.array([5, 21])
    kc, vc = _rand((B, Lmax, Hkv, d), rng), _rand((B, Lmax, Hkv, d), rng)
    kt, vt = _rand((B, T, Hkv, d), rng), _rand((B, T, Hkv, d), rng)
    acc = np.tile(np.arange(1, T + 1), (B, 1))
    acc[:, -1] = -1
    n = np.full(B, T - 1)
    com = tree_commit_kv(kc, vc, L, kt, vt, n, acc)
    assert com["status"] == 0
    for b in range(B):
        np.testing.assert_array_equal(com["k_cache"][b, L[b]:L[b] + T], kt[b])
        np.testing.assert_array_equal(com["v_cache"][b, L[b]:L[b] + T], vt[b])
        np.testing.assert_array_equal(com["k_cache"][b, :L[b]], kc[b, :L[b]])
        np.testing.assert_array_equal(com["k_cache"][b, L[b] + T:], kc[b, L[b] + T:])
    assert list(com["prefix_len"]) == [5 + T, 21 + T]


def test_tree_inside_the_cache_is_compacted_in_place():
    rng = np.random.default_rng(4)
    B, T, Hkv, d, Lmax = 3, 10, 2, 4, 40
    L = np.array([6, 0, 13])
    par = tree_random_recursive(T, torch.Generator().manual_seed(4))
    kc, vc = _rand((B, Lmax, Hkv, d), rng), _rand((B, Lmax, Hkv, d), rng)
    acc = np.full((B, T), -1)
    n = np.zeros(B, dtype=np.int64)
    for b in range(B):
        path = _root_path(par, int(rng.integers(1, T)))[1:]
        n[b] = len(path)
        acc[b, :len(path)] = path
    # the tree's K/V are the cache rows L .. L + T - 1
    kt = np.stack([kc[b, L[b]:L[b] + T] for b in range(B)])
    vt = np.stack([vc[b, L[b]:L[b] + T] for b in range(B)])
    sep = tree_commit_kv(kc, vc, L, kt, vt, n, acc)
    inp = tree_commit_kv(kc, vc, L, None, None, n, acc, tree_in_cache_at=L)
    assert sep["status"] == inp["status"] == 0
    for b in range(B):
        e = L[b] + n[b] + 1
        np.testing.assert_array_equal(inp["k_cache"][b, :e], sep["k_cache"][b, :e])
        np.testing.assert_array_equal(inp["v_cache"][b, :e], sep["v_cache"][b, :e])
        rows = [0] + list(acc[b, :n[b]])
        np.testing.assert_array_equal(inp["k_cache"][b, L[b]:e], kt[b, rows])


def test_empty_path_appends_the_root():
    rng = np.random.default_rng(5)
    kc, vc = _rand((1, 8, 1, 4), rng), _rand((1, 8, 1, 4), rng)
    kt, vt = _rand((1, 3, 1, 4), rng), _rand((1, 3, 1, 4), rng)
    com = tree_commit_kv(kc, vc, [2], kt, vt, [0], np.full((1, 3), -1))
    np.testing.assert_array_equal(com["k_cache"][0, 2], kt[0, 0])
    np.testing.assert_array_equal(com["v_cache"][0, 2], vt[0, 0])
    assert com["prefix_len"][0] == 3 and com["status"] == 0


@pytest.mark.parametrize("L,n,path,bit", [
    (5, 3, [1, 2, 3], ST_BAD_LEN),       # 5 + 3 + 1 > Lmax = 8
    (-1, 0, [], ST_BAD_LEN),
    (9, 0, [], ST_BAD_LEN),              # L > Lmax
    (0, 5, [1, 2, 3, 4, 5], ST_BAD_LEN),  # n > T - 1 = 4
    (0, 2, [2, 2], ST_BAD_ROW),          # not increasing
    (0, 2, [0, 2], ST_BAD_ROW),          # the root is not a path node
    (0, 1, [5], ST_BAD_ROW),             # outside [1, T)
])
def test_malformed_input_leaves_the_sequence_untouched(L, n, path, bit):
    rng = np.random.default_rng(6)
    B, T, Lmax = 2, 5, 8
    kc, vc = _rand((B, Lmax, 2, 4), rng), _rand((B, Lmax, 2, 4), rng)
    kt, vt = _rand((B, T, 2, 4), rng), _rand((B, T, 2, 4), rng)
    acc = np.full((B, T), -1)
    acc[0, :len(path)] = path
    acc[1, :2] = [1, 3]
    com = tree_commit_kv(kc, vc, [L, 2], kt, vt, [n, 2], acc)
    assert com["status"] == bit
    np.testing.assert_array_equal(com["k_cache"][0], kc[0])
    np.testing.assert_array_equal(com["v_cache"][0], vc[0])
    assert com["prefix_len"][0] == L
    # the well-formed sequence next to it is committed
    assert com["prefix_len"][1] == 5
    np.testing.assert_array_equal(com["k_cache"][1, 2:5], kt[1, [0, 1, 3]])
