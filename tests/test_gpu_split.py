"""GPU parity of the split-prefix path (through the C ABI): prefix-only
partials of tree_verify_attn on each kernel path against the oracle's, the
tree_verify_attn_merge kernel against the oracle's log-sum-exp merge, and a
prefix split into slices (partials on the GPU, merged on the GPU) against
the oracle's tree attention over the whole prefix."""

import numpy as np
import pytest
import torch

from oracle.attention import tree_verify_attn as oracle_attn, merge_partials
from synth import attn_case, tree_bfs_fanout, tree_random_recursive
from parity_util import BF16_MAX_ABS, BF16_REL_L2, FP32_MAX_ABS, FP32_REL_L2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tree_verification_verify_b200 import build
    build.build()


def _errs(got, want):
    d = got - want
    return float(np.max(np.abs(d))), float(np.linalg.norm(d) / max(np.linalg.norm(want), 1e-300))


def _check(got, want, bf16):
    m, r = _errs(got, want)
    if bf16:
        assert m <= BF16_MAX_ABS and r <= BF16_REL_L2, (m, r)
    else:
        assert m <= FP32_MAX_ABS and r <= FP32_REL_L2, (m, r)


def _slice(case, lo, hi, dev="cuda"):
    L = case.prefix_len.numpy()
    pl = torch.from_numpy(np.clip(L - lo, 0, hi - lo).astype(np.int32))
    return case.k_cache[:, lo:hi].to(dev), case.v_cache[:, lo:hi].to(dev), pl.to(dev)


@pytest.mark.parametrize("B,T,Hq,Hkv,d,L,dtype,paths", [
    (2, 40, 32, 8, 128, [1000, 0], "bf16", (1,)),           # one-tile tensor-core kernel
    (1, 256, 32, 8, 128, [32768], "bf16", (4, 5)),          # two-tile tensor-core kernel
    (1, 256, 32, 8, 128, [65536], "bf16", (5,)),            # ... chunks merged through the workspace
    (2, 17, 8, 2, 64, [300, 0], "fp32", (0,)),              # CUDA cores
])
def test_prefix_only_partial(B, T, Hq, Hkv, d, L, dtype, paths):
    import tree_verification_verify_b200 as tv
    case = attn_case(B, T, Hq, Hkv, d, L, dtype, tree_bfs_fanout(T, (4, 3, 2)), seed=T)
    dev = "cuda"
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    o, lse, _ = tv.tree_verify_attn(case.q.to(dev), case.k_cache.to(dev), case.v_cache.to(dev),
                                    case.prefix_len.to(dev), case.k_tree.to(dev), case.v_tree.to(dev),
                                    case.parent.to(dev), prefix_only=True, dev_status=st)
    torch.cuda.synchronize()
    assert tv.last_attn_path in paths and int(st.item()) == 0
    rows = None if T * B <= 80 else {(b, i) for b in range(B) for i in range(0, T, 16)}
    ref = oracle_attn(case.q, case.k_cache, case.v_cache, case.prefix_len, case.k_tree, case.v_tree, case.parent,
                      prefix_only=True, rows=rows)
    m = ref["written"]
    g = o.double().cpu().numpy()
    _check(g[m], ref["out"][m], dtype == "bf16")
    gl = lse.double().cpu().numpy()
    fin = np.isfinite(ref["lse"][m])
    assert np.max(np.abs(gl[m][fin] - ref["lse"][m][fin])) <= (2e-3 if dtype == "bf16" else 2e-5)
    # an empty prefix: out 0, lse -inf
    if 0 in L:
        b0 = L.index(0)
        assert torch.all(o[b0] == 0) and torch.all(lse[b0] == float("-inf"))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_merge_kernel(dtype):
    import tree_verification_verify_b200 as tv
    g = torch.Generator().manual_seed(1)
    N, B, T, Hq, d = 5, 2, 7, 4, 128
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    o = torch.randn(N, B, T, Hq, d, generator=g).to(dt)
    lse = torch.randn(N, B, T, Hq, generator=g) * 3.0
    lse[2, 0, 1, :] = float("-inf")                  # one empty partial
    lse[:, 1, 2, 0] = float("-inf")                  # a row with no keys at all
    lse[3, 1, 4, 2] = float("nan")                   # an invalid partial
    out, l = tv.tree_verify_attn_merge(o.cuda(), lse.cuda())
    torch.cuda.synchronize()
    ro, rl = merge_partials(o.double().numpy(), lse.double().numpy())
    go, gl = out.double().cpu().numpy(), l.double().cpu().numpy()
    assert np.all(np.isnan(go[1, 4, 2])) and np.isnan(gl[1, 4, 2])
    assert np.all(go[1, 2, 0] == 0) and gl[1, 2, 0] == -np.inf
    ok = np.isfinite(rl)
    _check(go[ok], ro[ok], dtype == "bf16")
    assert np.max(np.abs(gl[ok] - rl[ok])) <= 1e-5


@pytest.mark.parametrize("nslices", [2, 3])
def test_split_prefix_equals_tree_attention(nslices):
    """A long prefix cut into slices (one per GPU in a multi-GPU run, here
    one after another on one GPU), prefix-only partials for all but the
    last slice, which also takes the tree keys, merged on the GPU."""
    import tree_verification_verify_b200 as tv
    T, L = 64, [20000, 9000]
    case = attn_case(2, T, 32, 8, 128, L, "bf16", tree_random_recursive(T, torch.Generator().manual_seed(5)), seed=3)
    Lmax = case.k_cache.shape[1]
    bounds = [round(Lmax * r / nslices) for r in range(nslices + 1)]
    outs, lses = [], []
    for r in range(nslices):
        kc, vc, pl = _slice(case, bounds[r], bounds[r + 1])
        o, l, _ = tv.tree_verify_attn(case.q.cuda(), kc, vc, pl, case.k_tree.cuda(), case.v_tree.cuda(),
                                      case.parent.cuda(), prefix_only=(r != nslices - 1))
        outs.append(o)
        lses.append(l)
    out, l = tv.tree_verify_attn_merge(torch.stack(outs).contiguous(), torch.stack(lses).contiguous())
    torch.cuda.synchronize()
    rows = {(b, i) for b in range(2) for i in range(0, T, 4)}
    ref = oracle_attn(case.q, case.k_cache, case.v_cache, case.prefix_len, case.k_tree, case.v_tree, case.parent,
                      rows=rows)
    m = ref["written"]
    _check(out.double().cpu().numpy()[m], ref["out"][m], True)
    assert np.max(np.abs(l.double().cpu().numpy()[m] - ref["lse"][m])) <= 2e-3
