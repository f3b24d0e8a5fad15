"""The C-ABI library loads, exports every symbol include/*.h declares, and its
argument structs have the layout the Python binding marshals.  Host-side
only: no kernel is launched here."""

import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from tree_verification_verify_b200 import build as b
    b.build()
    import tree_verification_verify_b200 as tv
    return tv.lib()


def _declared():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names += re.findall(r"^TV_API\s+[\w\s\*]+?\b(\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", L._name], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(names) <= exported


def test_struct_layouts_match_the_header(L, tmp_path):
    import tree_verification_verify_b200 as tv
    structs = {"tv_attn_args": tv.AttnArgs, "tv_accept_args": tv.AcceptArgs,
               "tv_expand_args": tv.ExpandArgs, "tv_commit_args": tv.CommitArgs}
    src = ['#include <stdio.h>', '#include <stddef.h>', '#include "tree_verify.h"', "int main(void){"]
    for cname, py in structs.items():
        src.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for f, _ in py._fields_:
            src.append(f'printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    src.append("return 0;}")
    c = tmp_path / "layout.c"
    c.write_text("\n".join(src))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)], check=True)
    lines = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {}
    for ln in lines:
        if ln:
            s, f, v = ln.split()
            got[(s, f)] = int(v)
    for cname, py in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for f, _ in py._fields_:
            assert got[(cname, f)] == getattr(py, f).offset, (cname, f)


def test_version_and_status_strings(L):
    import tree_verification_verify_b200 as tv
    assert tv.version().startswith("treeverify")
    assert "sm_100a" in tv.version()
    assert tv.status_string(0) == "ok"
    assert "workspace" in tv.status_string(3)


def test_host_argument_checks(L):
    import tree_verification_verify_b200 as tv
    a = tv.AcceptArgs()
    a.B, a.T, a.V = 1, 2, 0                      # V < 1
    assert L.tree_accept(ctypes.byref(a), None, 0, None) == 1
    a.V, a.mode = 5, 9                           # unknown mode
    assert L.tree_accept(ctypes.byref(a), None, 0, None) == 1
    e = tv.ExpandArgs()
    e.V, e.R, e.Bsel, e.budget, e.draft_temperature = 10, 0, 4, 9000, 1.0
    assert L.tree_expand_topb(ctypes.byref(e), None, 0, None) == 2   # budget > 8192
    e.budget, e.draft_temperature = 16, 0.0
    assert L.tree_expand_topb(ctypes.byref(e), None, 0, None) == 1
    at = tv.AttnArgs()
    at.dtype, at.B, at.T, at.Hq, at.Hkv, at.d = 1, 1, 1, 6, 4, 128   # Hq % Hkv != 0
    assert L.tree_verify_attn(ctypes.byref(at), None, 0, None) == 1
    at.Hq, at.d = 8, 96                                              # d unsupported
    assert L.tree_verify_attn(ctypes.byref(at), None, 0, None) == 2
    c = tv.CommitArgs()
    c.dtype, c.B, c.T, c.Hkv, c.d, c.Lmax = 1, 0, 4, 2, 64, 16      # B = 0: nothing to do
    assert L.tree_commit_kv(ctypes.byref(c), None) == 0
    c.B = 1                                                          # B > 0 without arrays
    assert L.tree_commit_kv(ctypes.byref(c), None) == 1
    c.k_cache = c.v_cache = c.k_tree = c.v_tree = 1024
    c.prefix_len = c.n_accepted = c.accepted_nodes = 2048
    c.k_tree = 1025                                                  # not element-aligned
    assert L.tree_commit_kv(ctypes.byref(c), None) == 1
    c.k_tree, c.d = 1024, 2048                                       # d > 1024
    assert L.tree_commit_kv(ctypes.byref(c), None) == 2
    c.d, c.dtype = 64, 7                                             # unknown dtype
    assert L.tree_commit_kv(ctypes.byref(c), None) == 1
    c.dtype, c.T = 1, 0                                              # B > 0 with T = 0
    assert L.tree_commit_kv(ctypes.byref(c), None) == 1


def test_pool_bytes_grow_with_budget(L):
    a = L.tree_expand_pool_bytes(64, 256)
    b = L.tree_expand_pool_bytes(2048, 32000)
    assert 0 < a < b
    assert b >= 2048 * 2047 * 8
    assert L.tree_expand_pool_bytes(0, 10) == 0


def test_host_argument_checks_of_the_split_beam_and_diagnostic_calls(L):
    """The later entry points reject bad arguments on the host, before any
    launch: the partial merge, prefix-only partials, the expansion mode and
    the exponential diagnostic."""
    import tree_verification_verify_b200 as tv
    m = tv.AttnMergeArgs()
    m.dtype, m.N, m.B, m.T, m.Hq, m.d = 1, 0, 1, 1, 1, 128           # N < 1
    assert L.tree_verify_attn_merge(ctypes.byref(m), None) == 1
    m.N = 65                                                        # more partials than supported
    assert L.tree_verify_attn_merge(ctypes.byref(m), None) == 2
    m.N, m.d = 2, 96                                                # d unsupported
    assert L.tree_verify_attn_merge(ctypes.byref(m), None) == 2
    m.d, m.dtype = 128, 7                                           # unknown dtype
    assert L.tree_verify_attn_merge(ctypes.byref(m), None) == 1
    m.dtype = 1                                                     # rows but no arrays
    assert L.tree_verify_attn_merge(ctypes.byref(m), None) == 1
    m.B = 0                                                         # nothing to merge
    assert L.tree_verify_attn_merge(ctypes.byref(m), None) == 0
    at = tv.AttnArgs()
    at.dtype, at.B, at.T, at.Hq, at.Hkv, at.d = 1, 1, 1, 8, 2, 128
    at.sparse_topk, at.block_size, at.prefix_only = 4, 64, 1        # prefix-only with block top-k
    assert L.tree_verify_attn(ctypes.byref(at), None, 0, None) == 2
    assert L.tv_attn_path(ctypes.byref(at)) == -1
    at.sparse_topk, at.prefix_only = 0, 2                           # prefix_only is 0 or 1
    assert L.tree_verify_attn(ctypes.byref(at), None, 0, None) == 1
    e = tv.ExpandArgs()
    e.V, e.R, e.Bsel, e.budget, e.draft_temperature, e.mode = 10, 0, 4, 16, 1.0, 5   # unknown mode
    assert L.tree_expand_topb(ctypes.byref(e), None, 0, None) == 1
    assert L.tv_expand_exp(None, None, -1, None) == 1               # n < 0
    assert L.tv_expand_exp(None, None, 0, None) == 0                # nothing to do
    assert L.tv_expand_exp(None, None, 3, None) == 1                # arrays missing
