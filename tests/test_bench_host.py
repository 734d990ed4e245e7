"""Host-side checks of bench.py's bookkeeping (CPU only): the source lists behind the
recorded DRAM traffic name existing kernel sources, every recorded traffic entry belongs to
a known kernel, the q8 decode workload is attributed to the storage-order q8 kernel, and a
recorded figure is reported only while its kernel's source is the one it was captured on
(a kernel edited after its ncu capture shows null traffic until it is captured again)."""
import json
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gated_deltanet_recurrent_la_b200", "csrc")


def test_kernel_source_lists_name_existing_files():
    for kernel, files in bench.KERNEL_SOURCES.items():
        assert files, kernel
        for f in files:
            assert os.path.exists(os.path.join(CSRC, f)), f"{kernel}: {f}"


def test_step_workloads_map_to_their_kernels():
    assert bench.step_kernel("q8_decode64") == ("step_q8", "la::step_q8s_kernel")
    for w in ("decode512", "decode64", "mamba2", "kda_decode64", "qgroup_decode256", "conv_decode64"):
        assert bench.step_kernel(w) == ("step", "la::step_kernel")


def test_recorded_traffic_keys_and_hashes():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
        rec = json.load(fh)
    assert rec
    for key, entry in rec.items():
        kernel, workload = key.split("/")
        assert kernel in bench.KERNEL_SOURCES, key
        assert entry["dram_bytes_per_launch"] > 0 and entry["capture"], key
        fresh = entry["source_hash"] == bench.kernel_source_hash(bench.KERNEL_SOURCES[kernel])
        assert bench.recorded_traffic(kernel, workload) == (entry["dram_bytes_per_launch"] if fresh else None), key


def test_source_hash_ignores_comments(tmp_path, monkeypatch):
    """The hash covers code, not comments or blank lines."""
    a = tmp_path / "a.cuh"
    b = tmp_path / "b.cuh"
    a.write_text("int x = 1;  // one\n\n/* a block\n   comment */\nint y = 2;\n")
    b.write_text("int x = 1;\n// another comment\nint y = 2;   /* tail */\n")
    import builtins
    real_open = builtins.open

    def fake_open(path, *args, **kw):
        base = os.path.basename(str(path))
        if base in ("a.cuh", "b.cuh"):
            return real_open(tmp_path / base, *args, **kw)
        return real_open(path, *args, **kw)
    monkeypatch.setattr(builtins, "open", fake_open)
    assert bench.kernel_source_hash(["a.cuh"]) == bench.kernel_source_hash(["b.cuh"])
    b.write_text("int x = 1;\nint y = 3;\n")
    assert bench.kernel_source_hash(["a.cuh"]) != bench.kernel_source_hash(["b.cuh"])
