"""Host-side logic of bench.py's JSON line, on CPU: the roofline denominators
(measured peaks, else the stated fallback), the DRAM traffic taken from the
committed ncu summary only while the kernel's source is the one captured,
and the workload block of the line."""

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
