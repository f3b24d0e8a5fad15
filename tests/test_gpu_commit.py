"""GPU parity of tree_commit_kv against the fp64 oracle (through the C ABI).

A copy: the caches and prefix_len must equal the oracle's bit for bit.
Cases: random accepted paths (including the root alone and long chains
that take many shared-memory chunks), bf16 and fp32, head sizes whose rows
allow 16-, 4- or 2-byte words, a tree stored inside the cache right after
the prefix (compacted in place), malformed lengths and paths, the path that
tree_accept itself returns, and the Llama-3-8B layer's cache at full size."""

import numpy as np
import pytest
import torch

from oracle.commit import tree_commit_kv as oracle_commit, ST_BAD_LEN, ST_BAD_ROW
from synth import config_accept_case, tree_random_recursive, CONFIGS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tree_verification_verify_b200 import build
    build.build()


DT = {"bf16": torch.bfloat16, "fp32": torch.float32}


def _root_path(parent_row, x):
    p = [x]
    while p[-1] != 0:
        p.append(int(parent_row[p[-1]]))
    return p[::-1]


def _paths(B, T, gen, root_only=()):
    """Accepted paths of random trees: root .. a random node, root excluded."""
    acc = np.full((B, T), -1, dtype=np.int32)
    n = np.zeros(B, dtype=np.int32)
    for b in range(B):
        if b in root_only or T == 1:
            continue
        par = tree_random_recursive(T, gen)
        x = int(torch.randint(1, T, (1,), generator=gen))
        path = _root_path(par, x)[1:]
        acc[b, :len(path)] = path
        n[b] = len(path)
    return acc, n


def _run(kc, vc, L, kt, vt, n, acc, tree_in_cache_at=None):
    import tree_verification_verify_b200 as tv
    ref = oracle_commit(kc.cpu(), vc.cpu(), L, None if tree_in_cache_at is not None else kt.cpu(),
                        None if tree_in_cache_at is not None else vt.cpu(), n, acc,
                        tree_in_cache_at=tree_in_cache_at)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pl = torch.from_numpy(np.asarray(L, dtype=np.int32)).cuda()
    tv.tree_commit_kv(kc, vc, pl, kt, vt, torch.from_numpy(n).cuda(), torch.from_numpy(acc).cuda(),
                      dev_status=st)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(kc.double().cpu().numpy(), ref["k_cache"])
    np.testing.assert_array_equal(vc.double().cpu().numpy(), ref["v_cache"])
    np.testing.assert_array_equal(pl.cpu().numpy(), ref["prefix_len"])
    assert int(st.item()) == ref["status"]
    return ref


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("B,T,Hkv,d,Lmax", [
    (3, 12, 2, 64, 64), (2, 64, 8, 128, 4200), (2, 300, 1, 32, 700), (3, 10, 2, 36, 80),
    (2, 10, 3, 33, 80), (2, 12, 2, 3, 60), (1, 1, 4, 128, 9),
])
def test_random_paths(dtype, B, T, Hkv, d, Lmax):
    gen = torch.Generator().manual_seed(B * 1000 + T + d)
    dt = DT[dtype]
    kc = torch.randn(B, Lmax, Hkv, d, generator=gen).to(dt).cuda()
    vc = torch.randn(B, Lmax, Hkv, d, generator=gen).to(dt).cuda()
    kt = torch.randn(B, T, Hkv, d, generator=gen).to(dt).cuda()
    vt = torch.randn(B, T, Hkv, d, generator=gen).to(dt).cuda()
    acc, n = _paths(B, T, gen, root_only=(1,))
    L = torch.randint(0, Lmax - T + 1, (B,), generator=gen).numpy()
    ref = _run(kc, vc, L, kt, vt, n, acc)
    assert ref["status"] == 0


def test_long_chain_takes_many_chunks():
    """A chain accepted almost whole: 1000 rows of 8 kv heads, 63 chunks."""
    B, T, Hkv, d, Lmax = 1, 1001, 8, 128, 1500
    gen = torch.Generator().manual_seed(7)
    kc = torch.randn(B, Lmax, Hkv, d, generator=gen).to(torch.bfloat16).cuda()
    vc = torch.randn(B, Lmax, Hkv, d, generator=gen).to(torch.bfloat16).cuda()
    kt = torch.randn(B, T, Hkv, d, generator=gen).to(torch.bfloat16).cuda()
    vt = torch.randn(B, T, Hkv, d, generator=gen).to(torch.bfloat16).cuda()
    acc = np.full((B, T), -1, dtype=np.int32)
    acc[0, :999] = np.arange(1, 1000)
    _run(kc, vc, [300], kt, vt, np.array([999], dtype=np.int32), acc)


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp32", 64), ("bf16", 33)])
def test_tree_inside_the_cache_is_compacted_in_place(dtype, d):
    B, T, Hkv, Lmax, L0 = 3, 40, 4, 200, 57
    gen = torch.Generator().manual_seed(d)
    dt = DT[dtype]
    kc = torch.randn(B, Lmax, Hkv, d, generator=gen).to(dt).cuda()
    vc = torch.randn(B, Lmax, Hkv, d, generator=gen).to(dt).cuda()
    acc, n = _paths(B, T, gen)
    L = np.full(B, L0)
    # the tree's K/V are the cache rows L0 .. L0 + T - 1 (views, not copies)
    kt, vt = kc[:, L0:L0 + T], vc[:, L0:L0 + T]
    ref = _run(kc, vc, L, kt, vt, n, acc, tree_in_cache_at=L)
    assert ref["status"] == 0


@pytest.mark.parametrize("L,n,path,bit", [
    (5, 3, [1, 2, 3], ST_BAD_LEN),
    (-1, 0, [], ST_BAD_LEN),
    (9, 0, [], ST_BAD_LEN),
    (0, 5, [1, 2, 3, 4, 5], ST_BAD_LEN),
    (0, 2, [2, 2], ST_BAD_ROW),
    (0, 2, [0, 2], ST_BAD_ROW),
    (0, 1, [5], ST_BAD_ROW),
])
def test_malformed_input(L, n, path, bit):
    B, T, Hkv, d, Lmax = 2, 5, 2, 64, 8
    gen = torch.Generator().manual_seed(11)
    kc = torch.randn(B, Lmax, Hkv, d, generator=gen).to(torch.bfloat16).cuda()
    vc = torch.randn(B, Lmax, Hkv, d, generator=gen).to(torch.bfloat16).cuda()
    kt = torch.randn(B, T, Hkv, d, generator=gen).to(torch.bfloat16).cuda()
    vt = torch.randn(B, T, Hkv, d, generator=gen).to(torch.bfloat16).cuda()
    acc = np.full((B, T), -1, dtype=np.int32)
    acc[0, :len(path)] = path
    acc[1, :2] = [1, 3]
    ref = _run(kc, vc, [L, 2], kt, vt, np.array([n, 2], dtype=np.int32), acc)
    assert ref["status"] == bit


def test_path_from_tree_accept():
    """The acceptance walk's own outputs feed the commit (correlated target
    and draft, so that paths go deep), on the tiny configuration's shapes."""
    import tree_verification_verify_b200 as tv
    case = config_accept_case("tiny", temperature=0.8, seed=3, correlated=True)
    B, T, V = case.target_logits.shape
    g = tv.tree_accept(case.target_logits.cuda(), case.draft_tokens.cuda(), case.parent.cuda(),
                       draft_probs=case.draft_probs.cuda(), mode="specsample", temperature=0.8,
                       seed=case.seed, step=0)
    n = g["n_accepted"].cpu().numpy().astype(np.int32)
    acc = g["accepted_nodes"].cpu().numpy().astype(np.int32)
    Hkv, d, Lmax = 1, 64, 160
    gen = torch.Generator().manual_seed(12)
    kc = torch.randn(B, Lmax, Hkv, d, generator=gen).cuda()
    vc = torch.randn(B, Lmax, Hkv, d, generator=gen).cuda()
    kt = torch.randn(B, T, Hkv, d, generator=gen).cuda()
    vt = torch.randn(B, T, Hkv, d, generator=gen).cuda()
    ref = _run(kc, vc, [128] * B, kt, vt, n, acc)
    assert ref["status"] == 0


def test_llama3_8b_cache_full_size():
    """The Llama-3-8B layer: a 4096-token prefix in a cache of 8192 rows,
    8 kv heads of 128 (bf16), a 64-node tree and a 5-node accepted path."""
    c = CONFIGS["llama3_8b"]
    B, T, Hkv, d, Lmax = 1, c["T"], c["Hkv"], c["d"], 8192
    gen = torch.Generator().manual_seed(13)
    kc = torch.randn(B, Lmax, Hkv, d, generator=gen).to(torch.bfloat16).cuda()
    vc = torch.randn(B, Lmax, Hkv, d, generator=gen).to(torch.bfloat16).cuda()
    kt = torch.randn(B, T, Hkv, d, generator=gen).to(torch.bfloat16).cuda()
    vt = torch.randn(B, T, Hkv, d, generator=gen).to(torch.bfloat16).cuda()
    acc = np.full((B, T), -1, dtype=np.int32)
    acc[0, :5] = [2, 9, 30, 41, 63]
    _run(kc, vc, [c["L"]], kt, vt, np.array([5], dtype=np.int32), acc)
