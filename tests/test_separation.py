"""Structure that the parity claims rest on, checked on CPU.

* The oracle and the CUDA path share no code: nothing under oracle/ imports
  the package or reads its sources, and the package never imports the
  oracle.  Only the seeded input generators (synth/) serve both, and synth/
  holds none of the method's arithmetic.
* The product path has no CPU fallback: every entry point refuses host
  tensors with an error instead of computing.
"""

import ast
import os

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names |= {a.name.split(".")[0] for a in node.names}
        elif isinstance(node, ast.ImportFrom):
            if node.level == 0 and node.module:
                names.add(node.module.split(".")[0])
    return names


def _py_files(d):
    for base, _, files in os.walk(os.path.join(ROOT, d)):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(base, f)


def test_oracle_does_not_touch_the_cuda_path():
    for f in _py_files("oracle"):
        imps = _imports(f)
        assert "tree_verification_verify_b200" not in imps, f
        assert "synth" not in imps, f
        src = open(f).read()
        assert "csrc" not in src and "libtreeverify" not in src, f


def test_package_and_inputs_do_not_import_the_oracle():
    for d in ("tree_verification_verify_b200", "synth"):
        for f in _py_files(d):
            assert "oracle" not in _imports(f), f


def test_entry_points_refuse_host_tensors():
    import tree_verification_verify_b200 as tv
    from synth import accept_case, attn_case, tree_binary
    par = tree_binary(7)
    a = attn_case(1, 7, 4, 1, 64, [16], "fp32", [par], seed=0)
    with pytest.raises(tv.TVError):
        tv.tree_verify_attn(a.q, a.k_cache, a.v_cache, a.prefix_len, a.k_tree, a.v_tree, a.parent)
    c = accept_case(1, 7, 32, par, 0.8, seed=0)
    with pytest.raises(tv.TVError):
        tv.tree_accept(c.target_logits, c.draft_tokens, c.parent, draft_probs=c.draft_probs,
                       temperature=0.8)
    kc = torch.zeros(1, 30, 1, 64)
    with pytest.raises(tv.TVError):
        tv.tree_commit_kv(kc, kc.clone(), torch.zeros(1, dtype=torch.int32), a.k_tree, a.v_tree,
                          torch.zeros(1, dtype=torch.int32), torch.full((1, 7), -1, dtype=torch.int32))
