"""Pins of the attention oracle against what the mathematics fixes.

* a chain-shaped tree is causal attention over [prefix; tree]
  (torch scaled_dot_product_attention in float64 with an explicit mask);
* every node equals attention under an ancestor mask obtained a different
  way (transitive closure of the parent relation by boolean matrix
  products) through the same library routine;
* one node (T = 1) is single-token decode attention;
* a star tree sees prefix + root + itself;
* Hkv = Hq with repeated K/V equals the grouped (GQA) result;
* block top-k with k * block >= L equals dense; the kept blocks equal a
  brute-force count of the blocks ranked above each block;
* malformed trees give NaN rows and the status bit; rows past n_nodes are
  not written.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle.attention import (tree_verify_attn, block_means, ST_BAD_PARENT, ST_BAD_LEN)
from synth import (attn_case, tree_chain, tree_star, tree_binary, tree_bfs_fanout,
                   tree_random_recursive, tree_random_depth_limited)


def _sdpa(q, k, v, mask, scale):
    """q [Hq][Tq][d], k/v [Hq][Tk][d], mask [Tq][Tk] bool -> ([Hq][Tq][d])."""
    return F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)


def _closure_mask(parent_row, n):
    """anc[i][j] = j is node i or an ancestor of i, by repeated squaring of
    the parent adjacency (boolean matrix products)."""
    A = torch.zeros(n, n, dtype=torch.float64)
    for i in range(1, n):
        A[i, int(parent_row[i])] = 1.0
    R = torch.eye(n, dtype=torch.float64) + A
    for _ in range(int(np.ceil(np.log2(max(n, 2)))) + 1):
        R = ((R @ R) > 0).to(torch.float64)
    return R > 0


def _reference_by_mask(case, b):
    """Attention of every node of sequence b from the closure mask and SDPA."""
    q = case.q[b].to(torch.float64)                 # [T][Hq][d]
    T, Hq, d = q.shape
    Hkv = case.k_cache.shape[2]
    G = Hq // Hkv
    L = int(case.prefix_len[b])
    k = torch.cat([case.k_cache[b, :L], case.k_tree[b]], 0).to(torch.float64)  # [L+T][Hkv][d]
    v = torch.cat([case.v_cache[b, :L], case.v_tree[b]], 0).to(torch.float64)
    k = k.repeat_interleave(G, dim=1).permute(1, 0, 2)   # [Hq][L+T][d]
    v = v.repeat_interleave(G, dim=1).permute(1, 0, 2)
    mask = torch.cat([torch.ones(T, L, dtype=torch.bool), _closure_mask(case.parent[b].numpy(), T)], 1)
    return _sdpa(q.permute(1, 0, 2), k, v, mask, 1.0 / np.sqrt(d)).permute(1, 0, 2)


@pytest.mark.parametrize("T,L", [(1, 5), (7, 0), (9, 33)])
def test_chain_tree_is_causal_attention(T, L):
    case = attn_case(1, T, 4, 2, 16, L, "fp32", tree_chain(T), seed=3)
    o = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len,
                         case.k_tree, case.v_tree, case.parent)
    q = case.q[0].to(torch.float64).permute(1, 0, 2)
    k = torch.cat([case.k_cache[0, :L], case.k_tree[0]], 0).to(torch.float64)
    v = torch.cat([case.v_cache[0, :L], case.v_tree[0]], 0).to(torch.float64)
    k = k.repeat_interleave(2, dim=1).permute(1, 0, 2)
    v = v.repeat_interleave(2, dim=1).permute(1, 0, 2)
    # query i sits at position L + i: causal = keys 0 .. L + i
    pos_q = torch.arange(T)[:, None] + L
    mask = torch.arange(L + T)[None, :] <= pos_q
    ref = _sdpa(q, k, v, mask, 0.25).permute(1, 0, 2)
    np.testing.assert_allclose(o["out"][0], ref.numpy(), rtol=0, atol=1e-12)
    assert o["status"] == 0


@pytest.mark.parametrize("shape", ["binary", "bfs", "recursive", "depth6"])
def test_every_node_matches_closure_mask(shape):
    T = 23
    g = torch.Generator().manual_seed(5)
    par = {"binary": tree_binary(T), "bfs": tree_bfs_fanout(T, (4, 3, 2)),
           "recursive": tree_random_recursive(T, g),
           "depth6": tree_random_depth_limited(T, 6, g)}[shape]
    case = attn_case(2, T, 8, 2, 32, [40, 17], "fp32", par, seed=7)
    o = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len,
                         case.k_tree, case.v_tree, case.parent)
    for b in range(2):
        ref = _reference_by_mask(case, b)
        np.testing.assert_allclose(o["out"][b], ref.numpy(), rtol=0, atol=1e-12)


def test_single_node_is_decode_attention():
    case = attn_case(1, 1, 8, 8, 64, 100, "fp32", np.array([-1], np.int32), seed=11)
    o = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len,
                         case.k_tree, case.v_tree, case.parent)
    q = case.q[0].to(torch.float64).permute(1, 0, 2)       # [H][1][d]
    k = torch.cat([case.k_cache[0], case.k_tree[0]], 0).to(torch.float64).permute(1, 0, 2)
    v = torch.cat([case.v_cache[0], case.v_tree[0]], 0).to(torch.float64).permute(1, 0, 2)
    ref = F.scaled_dot_product_attention(q, k, v, scale=1 / 8.0).permute(1, 0, 2)
    np.testing.assert_allclose(o["out"][0], ref.numpy(), rtol=0, atol=1e-12)
    # lse from the definition log sum exp
    s = torch.einsum("hd,hkd->hk", q[:, 0], k) / 8.0
    np.testing.assert_allclose(o["lse"][0, 0], torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-12)


def test_star_tree_sees_prefix_root_and_self():
    T, L = 6, 10
    case = attn_case(1, T, 2, 1, 8, L, "fp32", tree_star(T), seed=2)
    o = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len,
                         case.k_tree, case.v_tree, case.parent)
    for i in range(T):
        keys = [case.k_cache[0, :L, 0], case.k_tree[0, [0] + ([i] if i else []), 0]]
        vals = [case.v_cache[0, :L, 0], case.v_tree[0, [0] + ([i] if i else []), 0]]
        k = torch.cat(keys, 0).double()
        v = torch.cat(vals, 0).double()
        for h in range(2):
            s = (k @ case.q[0, i, h].double()) / np.sqrt(8)
            ref = torch.softmax(s, 0) @ v
            np.testing.assert_allclose(o["out"][0, i, h], ref.numpy(), rtol=0, atol=1e-12)


def test_gqa_equals_repeated_kv():
    T = 9
    par = tree_binary(T)
    case = attn_case(1, T, 8, 2, 16, 21, "fp32", par, seed=4)
    o = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len,
                         case.k_tree, case.v_tree, case.parent)
    rep = lambda x: x.repeat_interleave(4, dim=2)
    o2 = tree_verify_attn(case.q, rep(case.k_cache), rep(case.v_cache), case.prefix_len,
                          rep(case.k_tree), rep(case.v_tree), case.parent)
    np.testing.assert_allclose(o["out"], o2["out"], rtol=0, atol=1e-13)


def test_bf16_inputs_are_widened_exactly():
    case = attn_case(1, 3, 2, 1, 8, 4, "bf16", tree_chain(3), seed=1)
    o = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len,
                         case.k_tree, case.v_tree, case.parent)
    o2 = tree_verify_attn(case.q.float(), case.k_cache.float(), case.v_cache.float(), case.prefix_len,
                          case.k_tree.float(), case.v_tree.float(), case.parent)
    np.testing.assert_array_equal(o["out"], o2["out"])


def test_empty_prefix_root_returns_its_own_value():
    case = attn_case(1, 4, 2, 1, 8, 0, "fp32", tree_chain(4), seed=9)
    o = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len,
                         case.k_tree, case.v_tree, case.parent)
    np.testing.assert_allclose(o["out"][0, 0, :], case.v_tree[0, 0, 0].double().expand(2, 8).numpy(),
                               rtol=0, atol=1e-15)


def test_sparse_with_all_blocks_equals_dense():
    T = 7
    case = attn_case(1, T, 4, 2, 16, 300, "fp32", tree_binary(T), seed=12)
    dense = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len,
                             case.k_tree, case.v_tree, case.parent)
    sp = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len,
                          case.k_tree, case.v_tree, case.parent, sparse_topk=5, block_size=64)
    np.testing.assert_allclose(sp["out"], dense["out"], rtol=0, atol=1e-13)
    assert np.all(sp["sel"][0, :, :, :5] == np.arange(5))


def test_block_selection_matches_brute_force_rank_count():
    T, L, bs, k = 5, 1000, 64, 4
    case = attn_case(2, T, 4, 2, 16, [L, 700], "fp32", tree_binary(T), seed=13,
                     offset_frac=0.2, block_size=bs)
    o = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len,
                         case.k_tree, case.v_tree, case.parent, sparse_topk=k, block_size=bs)
    Kf = case.k_cache.double().numpy()
    for b in range(2):
        Lb = int(case.prefix_len[b])
        nblk = (Lb + bs - 1) // bs
        for g in range(2):
            # block means by an explicit per-position sum
            kbar = np.zeros((nblk, 16))
            cnt = np.zeros(nblk)
            for p in range(Lb):
                kbar[p // bs] += Kf[b, p, g]
                cnt[p // bs] += 1
            kbar /= cnt[:, None]
            for i in range(T):
                qg = case.q[b, i, 2 * g:2 * g + 2].double().numpy()
                sc = np.array([qg[0] @ kbar[j] + qg[1] @ kbar[j] for j in range(nblk)])
                kept = [j for j in range(nblk)
                        if sum(1 for m in range(nblk)
                               if sc[m] > sc[j] or (sc[m] == sc[j] and m < j)) < k]
                assert list(o["sel"][b, i, g]) == kept
                # and the node's output is attention over those blocks + path
                pos = [p for j in kept for p in range(j * bs, min((j + 1) * bs, Lb))]
                path = [0] if i == 0 else ([0, (i - 1) // 2, i] if i > 2 else [0, i])
                kk = np.concatenate([Kf[b, pos, g], case.k_tree[b, path, g].double().numpy()])
                vv = np.concatenate([case.v_cache[b, pos, g].double().numpy(),
                                     case.v_tree[b, path, g].double().numpy()])
                for hh in range(2):
                    s = kk @ case.q[b, i, 2 * g + hh].double().numpy() / 4.0
                    w = np.exp(s - s.max())
                    ref = (w / w.sum()) @ vv
                    np.testing.assert_allclose(o["out"][b, i, 2 * g + hh], ref, rtol=0, atol=1e-12)


def test_offset_blocks_are_preferred_when_aligned():
    """With a strong shared offset m_g on 20% of the blocks, a query whose
    group sum is aligned with m_g keeps offset blocks."""
    T, L, bs = 3, 64 * 40, 64
    case = attn_case(1, T, 4, 1, 32, L, "fp32", tree_chain(T), seed=21, offset_frac=0.2, block_size=bs)
    kbar = block_means(case.k_cache, case.prefix_len, bs)[0, :, 0]
    off = set(case.offset_blocks[0][0].tolist())
    m = kbar[sorted(off)].mean(0) - kbar[[j for j in range(40) if j not in off]].mean(0)
    q = case.q.clone()
    q[0, 0, :, :] = torch.tensor(m, dtype=torch.float32)[None, :] * 3
    o = tree_verify_attn(q, case.k_cache, case.v_cache, case.prefix_len,
                         case.k_tree, case.v_tree, case.parent, sparse_topk=4, block_size=bs)
    assert set(o["sel"][0, 0, 0].tolist()) <= off


def test_malformed_parent_and_partial_rows():
    T = 6
    par = np.array([-1, 0, 0, 5, 1, 2], np.int32)        # parent[3] = 5 >= 3
    case = attn_case(1, T, 2, 1, 8, 5, "fp32", par, seed=1, n_nodes=5)
    o = tree_verify_attn(case.q, case.k_cache, case.v_cache, case.prefix_len,
                         case.k_tree, case.v_tree, case.parent, n_nodes=case.n_nodes)
    assert o["status"] & ST_BAD_PARENT
    assert not o["valid"][0, 3] and o["written"][0, 3] and np.all(np.isnan(o["out"][0, 3]))
    assert o["valid"][0, 4] and np.all(np.isfinite(o["out"][0, 4]))
    assert not o["written"][0, 5]
    bad = tree_verify_attn(case.q, case.k_cache, case.v_cache, torch.tensor([9], dtype=torch.int32),
                           case.k_tree, case.v_tree, case.parent)
    assert bad["status"] & ST_BAD_LEN and np.all(np.isnan(bad["out"]))
