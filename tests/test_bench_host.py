"""Host-side logic of bench.py's JSON line, on CPU: the roofline denominators
(measured peaks, else the stated fallback), the DRAM traffic taken from the
committed ncu summary only while the kernel's source is the one captured,
the workload block of the line, the attention's algorithmic FLOPs and bytes
against a brute-force count, and the roofline fractions."""

import hashlib
import json
import types

import bench


def test_peaks_measured_then_fallback(tmp_path, monkeypatch):
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps({"hbm_gbs": 6000.5, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1300.0}))
    monkeypatch.setattr(bench, "PEAKS_PATH", str(f))
    assert bench.peaks() == (6000.5, 1500.0, 1300.0, "measured")
    monkeypatch.setattr(bench, "PEAKS_PATH", str(tmp_path / "absent.json"))
    hbm, bf16, _, src = bench.peaks()
    assert (hbm, bf16, src) == (bench.FALLBACK_HBM_GBS, bench.FALLBACK_BF16_TFLOPS, "fallback")


def test_traffic_is_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// a kernel\n")
    sha = hashlib.sha1(src.read_bytes()).hexdigest()
    traffic = tmp_path / "traffic.txt"
    traffic.write_text("# comment line\n"
                       f"fake_kernel llama3_8b dram_bytes_per_launch=12345 source_sha1={sha} capture=x.md\n"
                       "fake_kernel serving dram_bytes_per_launch=999 source_sha1=0000 capture=y.md\n")
    monkeypatch.setattr(bench, "TRAFFIC_PATH", str(traffic))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "fake_kernel", str(src))
    assert bench.measured_traffic("fake_kernel", "llama3_8b") == 12345.0
    assert bench.measured_traffic("fake_kernel", "serving") is None          # other source
    assert bench.measured_traffic("fake_kernel", "longctx") is None          # no capture
    src.write_text("// a kernel, changed\n")
    assert bench.measured_traffic("fake_kernel", "llama3_8b") is None        # stale capture
    assert bench.measured_traffic("no_such_kernel", "llama3_8b") is None


def test_committed_traffic_entries_name_existing_kernels_and_captures():
    import os
    for line in open(bench.TRAFFIC_PATH):
        f = line.split()
        if not f or f[0].startswith("#"):
            continue
        kv = dict(x.split("=", 1) for x in f[2:])
        assert f[0] in bench.KERNEL_SOURCES
        assert float(kv["dram_bytes_per_launch"]) > 0
        assert len(kv["source_sha1"]) == 40
        assert os.path.exists(os.path.join(bench.ROOT, kv["capture"]))


def test_config_block_names_the_workload():
    from synth import CONFIGS
    step = types.SimpleNamespace(c=CONFIGS["llama3_8b"], name="llama3_8b", temperature=0.8, sparse=False,
                                 B=1, T=64)
    blk = bench.config_block(step, 2)
    assert blk["workload"].startswith("llama3_8b: B=1 Hq=32 Hkv=8 d=128 bf16 prefix=4096 T=64 V=128256")
    assert blk["tree_nodes_per_rank"] == 64
    assert blk["parallelism"] == "replicas x2"
    assert "flush" in blk["l2"]
    assert "model" not in blk


def _ancestor_counts(parent):
    """|root path ∪ self| of every node, by walking parent[] (no helper of
    the bench or of synth)."""
    out = []
    for i in range(len(parent)):
        n, j = 0, i
        while j >= 0:
            n += 1
            j = int(parent[j])
        out.append(n)
    return out


def test_attention_work_counts_every_key_a_node_attends_to():
    """attn_work's FLOPs and bytes against a brute-force count: node i of
    sequence b attends to prefix_len[b] prefix keys plus its root path, two
    matmuls of 2 d FLOPs per (query head, key); every prefix and tree K/V
    element is read once."""
    import numpy as np
    rng = np.random.default_rng(3)
    B, T, Hq, Hkv, d, elt = 3, 23, 8, 2, 64, 2
    parents = []
    for _ in range(B):
        par = [-1] + [int(rng.integers(0, i)) for i in range(1, T)]
        parents.append(par)
    L = [0, 17, 1000]
    flops, nbytes = bench.attn_work(parents, L, T, Hq, Hkv, d, elt)
    keys = sum(L[b] + c for b in range(B) for c in _ancestor_counts(parents[b]))
    assert flops == 4.0 * d * Hq * keys
    assert nbytes == (sum(L) + B * T) * Hkv * d * 2 * elt
    # block top-k: the kept prefix keys per (node, kv head) and the union of
    # kept blocks replace the dense prefix
    kept, union = 5 * 64 * B * T * Hkv, 9
    f2, b2 = bench.attn_work(parents, L, T, Hq, Hkv, d, elt, kept_keys=kept, union_blocks=union,
                             block_size=64, means_in_call=True)
    path = sum(c for b in range(B) for c in _ancestor_counts(parents[b]))
    assert f2 == 4.0 * d * (Hq // Hkv) * kept + 4.0 * d * Hq * path
    assert b2 == union * 64 * d * 2 * elt + B * T * Hkv * d * 2 * elt + sum(L) * Hkv * d * elt


def test_roofline_fractions_take_the_slower_bound(monkeypatch):
    """The fraction is (the slower of bytes / bandwidth and FLOPs / peak) /
    time, against both denominators."""
    monkeypatch.setattr(bench, "peaks", lambda: (5000.0, 1000.0, "m", "m"))
    r = bench.roofline_fracs(1e-3, nbytes=2.5e9, flops=0.0)          # 0.5 ms of HBM time
    assert r["frac_measured"] == 0.5
    assert r["frac_target"] == round(2.5e9 / 8000e9 / 1e-3, 4)
    r = bench.roofline_fracs(2e-3, nbytes=1e9, flops=1e12)          # 1 ms of tensor time
    assert r["frac_measured"] == 0.5
    assert r["frac_target"] == round(1e12 / 2250e12 / 2e-3, 4)


def test_acceptance_bytes_read_the_rows_the_walk_needs():
    """accept_work: B T target rows, plus one draft row per node with at
    least one child when draft probabilities are given."""
    import numpy as np
    rng = np.random.default_rng(5)
    B, T, V = 4, 19, 1000
    parents = [np.array([-1] + [int(rng.integers(0, i)) for i in range(1, T)]) for _ in range(B)]
    with_children = sum(sum(1 for j in range(T) if any(par[i] == j for i in range(1, T))) for par in parents)
    assert bench.accept_work(parents, T, V, True) == (B * T + with_children) * V * 4
    assert bench.accept_work(parents, T, V, False) == B * T * V * 4
