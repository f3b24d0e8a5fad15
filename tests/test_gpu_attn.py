"""GPU parity of tree_verify_attn against the fp64 oracle (through the C ABI).

bf16: max-abs <= 2e-2 and relative L2 <= 5e-3; fp32: max-abs <= 2e-5 and
relative L2 <= 2e-6.  Small cases compare every row (several tiles, ragged
tails, malformed trees, rows past n_nodes left untouched); the full-size
workloads compare sampled nodes, computed one by one by the oracle."""

import numpy as np
import pytest
import torch

from oracle.attention import tree_verify_attn as oracle_attn, ST_BAD_PARENT, ST_BAD_LEN
from synth import (attn_case, config_attn_case, tree_binary, tree_chain, tree_star,
                   tree_bfs_fanout, tree_random_recursive, tree_random_depth_limited, CONFIGS)
from parity_util import check_attn, cuda, BF16_MAX_ABS, BF16_REL_L2, FP32_MAX_ABS, FP32_REL_L2

pytestmark = pytest.mark.gpu
POISON = 512.0          # exactly representable in bf16 and fp32


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tree_verification_verify_b200 import build
    build.build()


def _gpu(case, n_nodes=None, prefix_len=None, sparse_topk=None, want_sel=False, q=None):
    import tree_verification_verify_b200 as tv
    qd = cuda(case.q if q is None else q)
    B, T, Hq, d = qd.shape
    out = torch.full((B, T, Hq, d), POISON, dtype=qd.dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nn = n_nodes if n_nodes is not None else case.n_nodes
    pl = prefix_len if prefix_len is not None else case.prefix_len
    k = case.sparse_topk if sparse_topk is None else sparse_topk
    o, lse, sel = tv.tree_verify_attn(qd, cuda(case.k_cache), cuda(case.v_cache), cuda(pl),
                                      cuda(case.k_tree), cuda(case.v_tree), cuda(case.parent),
                                      n_nodes=cuda(nn), scale=case.scale, sparse_topk=k,
                                      block_size=case.block_size, out=out, want_sel=want_sel,
                                      dev_status=st)
    torch.cuda.synchronize()
    return o, lse, sel, int(st.item())


def _oracle(case, n_nodes=None, prefix_len=None, rows=None, sparse_topk=None):
    return oracle_attn(case.q, case.k_cache, case.v_cache,
                       case.prefix_len if prefix_len is None else prefix_len,
                       case.k_tree, case.v_tree, case.parent,
                       n_nodes=case.n_nodes if n_nodes is None else n_nodes, scale=case.scale,
                       sparse_topk=case.sparse_topk if sparse_topk is None else sparse_topk,
                       block_size=case.block_size, rows=rows)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_config_fp32(seed):
    case = config_attn_case("tiny", seed=seed)
    o, lse, _, st = _gpu(case)
    ref = _oracle(case)
    check_attn(o, ref, torch.float32, lse_gpu=lse, poison=POISON)
    assert st == 0


SHAPES = [
    # B, T, Hq, Hkv, d, L, dtype, tree
    (2, 23, 8, 2, 64, [300, 0], "bf16", "recursive"),
    (1, 40, 32, 8, 128, [1000], "bf16", "bfs"),
    (3, 17, 4, 4, 128, [129, 64, 1], "bf16", "depth6"),
    (1, 9, 16, 1, 64, [513], "bf16", "chain"),
    (2, 33, 8, 1, 32, [77, 200], "fp32", "star"),
    (1, 15, 64, 8, 128, [2048], "bf16", "binary"),
    (2, 70, 16, 2, 128, [0, 700], "bf16", "recursive"),
    (1, 300, 32, 8, 128, [200], "bf16", "chain"),        # deep: 3 gathered tree tiles
    (2, 129, 8, 1, 128, [333, 1], "bf16", "binary"),
    (1, 600, 64, 8, 128, [5000], "bf16", "recursive"),   # split prefix + cluster merge
    (1, 300, 32, 8, 128, [2000], "bf16", "chain"),       # ragged last row tile after 3 tree tiles
    (1, 1000, 64, 8, 128, [300], "bf16", "chain"),       # 8 tree tiles per row tile
    (1, 256, 32, 8, 128, [20000], "bf16", "bfs"),        # long prefix (two-tile CTAs where the plan picks them)
    (2, 100, 16, 2, 128, [9000, 3000], "bf16", "recursive"),  # odd tile count: a last pair with one tile
    (1, 200, 8, 8, 128, [12000], "bf16", "chain"),       # G = 1: 128 nodes per tile, deep tree tiles
]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"{s[6]}-T{s[1]}-G{s[2]//s[3]}-d{s[4]}" for s in SHAPES])
def test_shapes(shape):
    B, T, Hq, Hkv, d, L, dtype, tree = shape
    g = torch.Generator().manual_seed(T)
    par = {"recursive": tree_random_recursive(T, g), "bfs": tree_bfs_fanout(T, (4, 3, 2)),
           "depth6": tree_random_depth_limited(T, 6, g), "chain": tree_chain(T),
           "star": tree_star(T), "binary": tree_binary(T)}[tree]
    case = attn_case(B, T, Hq, Hkv, d, L, dtype, par, seed=B * T)
    o, lse, _, st = _gpu(case)
    import tree_verification_verify_b200 as tv
    # bf16 with d = 128 and a power-of-two group runs the tensor-core kernel
    assert tv.last_attn_path in ((1, 4, 5) if (dtype == "bf16" and d == 128) else (0,))
    assert tv.last_attn_launches == (1 if tv.last_attn_path in (1, 4, 5) else 3)
    ref = _oracle(case)
    check_attn(o, ref, o.dtype, lse_gpu=lse, poison=POISON)
    assert st == ref["status"] == 0


@pytest.mark.parametrize("L", [[250, 40, 3], [2500, 40, 3]], ids=["one-chunk", "split"])
def test_partial_trees_and_malformed_input(L):
    T = 21
    par = tree_random_recursive(T, torch.Generator().manual_seed(2))
    par[13] = 17                                      # malformed: 17 >= 13
    case = attn_case(3, T, 8, 2, 128, L, "bf16", par, seed=5, n_nodes=[21, 9, 0])
    o, lse, _, st = _gpu(case)
    ref = _oracle(case)
    check_attn(o, ref, torch.bfloat16, lse_gpu=lse, poison=POISON)
    assert st == ref["status"] and st & ST_BAD_PARENT
    bad_pl = torch.tensor([L[0], max(L) + 999, 3], dtype=torch.int32)
    bad_nn = torch.tensor([21, 9, 30], dtype=torch.int32)
    o, lse, _, st = _gpu(case, n_nodes=bad_nn, prefix_len=bad_pl)
    ref = _oracle(case, n_nodes=bad_nn, prefix_len=bad_pl)
    check_attn(o, ref, torch.bfloat16, poison=POISON)
    assert st == ref["status"] and st & ST_BAD_LEN


def test_strided_query_view():
    T, Hq, d = 12, 8, 64
    case = attn_case(2, T, Hq, 2, d, [100, 31], "bf16", tree_binary(T), seed=3)
    big = torch.randn(2, T, Hq + 3, d + 64).to(torch.bfloat16)
    big[:, :, 1:Hq + 1, 32:32 + d] = case.q
    qv = big[:, :, 1:Hq + 1, 32:32 + d]                 # non-contiguous heads / rows
    o, lse, _, st = _gpu(case, q=qv)
    ref = _oracle(case)
    check_attn(o, ref, torch.bfloat16, lse_gpu=lse)


def _sample_rows(B, T, per_b, seed):
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(B):
        for i in rng.choice(T, size=min(per_b, T), replace=False):
            rows.add((b, int(i)))
        rows.add((b, 0))
        rows.add((b, T - 1))
    return rows


def _rows_mask(rows, B, T):
    m = np.zeros((B, T), dtype=bool)
    for b, i in rows:
        m[b, i] = True
    return m


@pytest.mark.parametrize("name,per_b", [("llama3_8b", 64), ("specexec70b", 24), ("serving", 2), ("longctx", 3)])
def test_full_size_dense_sampled(name, per_b):
    c = CONFIGS[name]
    case = config_attn_case(name, seed=0)
    o, lse, _, st = _gpu(case)
    import tree_verification_verify_b200 as tv
    assert tv.last_attn_path in (1, 4, 5)
    print(f"{name}: attention path {tv.last_attn_path}")
    rows = _sample_rows(c["B"], c["T"], per_b, 1)
    ref = _oracle(case, rows=rows)
    check_attn(o, ref, torch.bfloat16, lse_gpu=lse, rows_mask=_rows_mask(rows, c["B"], c["T"]))
    assert st == 0


def test_sparse_small_all_blocks_equals_dense():
    T = 13
    case = attn_case(2, T, 8, 2, 128, [300, 64], "bf16", tree_binary(T), seed=4)
    od, _, _, _ = _gpu(case, sparse_topk=0)
    os_, _, sel, st = _gpu(case, sparse_topk=5, want_sel=True)
    ref = _oracle(case, sparse_topk=5)
    check_attn(os_, ref, torch.bfloat16, poison=POISON)
    assert torch.equal(sel.cpu(), torch.from_numpy(ref["sel"]).to(torch.int32))
    assert (od.float() - os_.float()).abs().max().item() < 2e-2


# Block selection band.  The GPU scores a block as <sum_h q_h, kbar_j> in
# fp32: kbar from 64 bf16 keys and the group sum of G bf16 queries are exact
# or within one fp32 rounding, and the d-term dot product carries at most
# about d * 2^-24 * sum_i |a_i b_i| of rounding.  On these inputs sum |a_i b_i|
# stays within a few times max |score|, so two scores closer than about
# 1e-6 of max |score| can swap; SPARSE_BAND is that bound with a margin of
# ten.  Where the GPU's kept set differs from the oracle's, the oracle's
# rank-k / rank-(k+1) gap must lie inside the band, such pairs may be at
# most 1% of the checked (node, kv head) pairs, and their output is checked
# against the oracle run with the GPU's own selection.
SPARSE_BAND = 1e-5


def _check_sparse(case, rows, B, T, Hkv, G, k):
    o, lse, sel, st = _gpu(case, want_sel=True)
    ref = _oracle(case, rows=rows)
    sel = sel.cpu().numpy()
    got = o.double().cpu().numpy()
    lg = lse.double().cpu().numpy()
    bf16 = o.dtype == torch.bfloat16
    same, near = [], []
    for (b, i) in sorted(rows):
        for g in range(Hkv):
            if np.array_equal(sel[b, i, g], ref["sel"][b, i, g]):
                same.append((b, i, g))
            else:
                assert ref["sel_gap"][b, i, g] < SPARSE_BAND, (b, i, g, ref["sel_gap"][b, i, g])
                near.append((b, i, g))
    pairs = len(rows) * Hkv
    print(f"block selection: {len(same)} of {pairs} (node, kv head) pairs equal to the oracle's, "
          f"{len(near)} near-ties inside the band")
    assert len(near) <= max(1, pairs // 100)

    def compare(items, want_out, want_lse):
        g_ = np.concatenate([got[b, i, g * G:(g + 1) * G].ravel() for b, i, g in items])
        w_ = np.concatenate([want_out[b, i, g * G:(g + 1) * G].ravel() for b, i, g in items])
        d = g_ - w_
        max_abs = float(np.max(np.abs(d)))
        rel = float(np.linalg.norm(d) / max(np.linalg.norm(w_), 1e-300))
        if bf16:
            assert max_abs <= BF16_MAX_ABS and rel <= BF16_REL_L2, (max_abs, rel)
        else:
            assert max_abs <= FP32_MAX_ABS and rel <= FP32_REL_L2, (max_abs, rel)
        dl = max(float(np.max(np.abs(lg[b, i, g * G:(g + 1) * G] - want_lse[b, i, g * G:(g + 1) * G])))
                 for b, i, g in items)
        assert dl <= (2e-3 if bf16 else 2e-5), dl
        return max_abs, rel

    assert same
    compare(same, ref["out"], ref["lse"])
    if near:
        ref2 = oracle_attn(case.q, case.k_cache, case.v_cache, case.prefix_len, case.k_tree, case.v_tree,
                           case.parent, n_nodes=case.n_nodes, scale=case.scale, sparse_topk=case.sparse_topk,
                           block_size=case.block_size, rows={(b, i) for b, i, _ in near}, forced_sel=sel)
        compare(near, ref2["out"], ref2["lse"])
    return len(same), len(near), st


def test_sparse_small_offsets():
    T, L, bs = 20, 64 * 60, 64
    case = attn_case(2, T, 8, 2, 128, [L, L - 37], "bf16", tree_bfs_fanout(T, (4, 3, 2)), seed=6,
                     offset_frac=0.1, block_size=bs, sparse_topk=8)
    rows = {(b, i) for b in range(2) for i in range(T)}
    _check_sparse(case, rows, 2, T, 2, 4, 8)
    import tree_verification_verify_b200 as tv
    assert tv.last_attn_path == 3          # bf16, d = 128, blocks of 64, G = 4: tensor cores


@pytest.mark.parametrize("Hq,Hkv,d,dtype,bs,k", [
    (8, 8, 64, "bf16", 100, 6),     # G = 1, blocks wider than one 64-key tile, ragged last block
    (32, 4, 128, "bf16", 16, 12),   # G = 8, narrow blocks
    (64, 2, 32, "fp32", 40, 5),     # G = 32 (two heads per warp), fp32, d = 32
])
def test_sparse_shapes(Hq, Hkv, d, dtype, bs, k):
    """The block top-k path over head groups, head dims, dtypes and block
    widths (blocks of more than 64 keys are streamed in two tiles)."""
    T, L = 11, [bs * 9 + 7, bs * 3]
    case = attn_case(2, T, Hq, Hkv, d, L, dtype, tree_random_recursive(T, torch.Generator().manual_seed(2)),
                     seed=9, offset_frac=0.2, block_size=bs, sparse_topk=k)
    rows = {(b, i) for b in range(2) for i in range(T)}
    _check_sparse(case, rows, 2, T, Hkv, Hq // Hkv, k)
    import tree_verification_verify_b200 as tv
    assert tv.last_attn_path == 2          # outside the tensor-core variant: CUDA cores


def test_full_size_sparse_sampled():
    c = CONFIGS["longctx"]
    case = config_attn_case("longctx", seed=0, sparse=True)
    rows = _sample_rows(c["B"], c["T"], 64, 2)          # 64 sampled nodes per sequence, plus the first and last
    checked, near, st = _check_sparse(case, rows, c["B"], c["T"], c["Hkv"], c["Hq"] // c["Hkv"], 32)
    assert st == 0
    import tree_verification_verify_b200 as tv
    assert tv.last_attn_path == 3


@pytest.mark.parametrize("B,T,L,G", [(1, 256, 65536, 4), (1, 300, 70000, 4)])
def test_two_tile_workspace_merge(B, T, L, G):
    """A long prefix whose tile pairs split into more chunks than a cluster
    fills the GPU with: the two-tile kernel merges its chunks through the
    workspace (path 5; 9 and 11 chunks here).  Sampled rows against the
    oracle, including tree rows (the last chunk's) and a ragged last tile."""
    import tree_verification_verify_b200 as tv
    case = attn_case(B, T, 8 * G, 8, 128, [L] * B, "bf16", tree_bfs_fanout(T, (4, 3, 2)), seed=L)
    o, lse, _, st = _gpu(case)
    assert tv.last_attn_path == 5, tv.last_attn_path
    rows = _sample_rows(B, T, 24, 3)
    ref = _oracle(case, rows=rows)
    check_attn(o, ref, torch.bfloat16, lse_gpu=lse, rows_mask=_rows_mask(rows, B, T))
    assert st == 0

