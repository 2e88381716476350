"""bench.py host logic: the per-family kernel source hashes that key the
recorded DRAM traffic, and the traffic table's workload names."""
import os
import shutil

import bench
import workloads


def _copy_sources(tmp_path):
    src = os.path.join(bench.ROOT, "long_context_exact_blockwise_b200", "csrc")
    dst = tmp_path / "long_context_exact_blockwise_b200" / "csrc"
    shutil.copytree(src, dst)
    return dst


def _hashes():
    return {f: bench.kernel_source_hash(f) for f in ("fwd", "decode", "bwd")}


def test_hash_changes_only_for_families_that_include_the_file(tmp_path, monkeypatch):
    csrc = _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = _hashes()
    for name in sorted(os.listdir(csrc)):
        path = csrc / name
        original = path.read_bytes()
        path.write_bytes(original + b"\n// edited\n")
        edited = _hashes()
        path.write_bytes(original)
        for fam in ("fwd", "decode", "bwd"):
            covered = name not in bench._NOT_IN_HASH[fam]
            assert (edited[fam] != base[fam]) == covered, (name, fam)
    assert _hashes() == base


def test_backward_hash_ignores_forward_and_decode_kernels():
    assert "fwd_sm100.cuh" in bench._NOT_IN_HASH["bwd"]
    assert "decode_sm100.cuh" in bench._NOT_IN_HASH["bwd"]
    assert "bwd_sm100.cuh" in bench._NOT_IN_HASH["fwd"]
    assert "bwd_sm100.cuh" in bench._NOT_IN_HASH["decode"]
    # The CTA-pair forward kernel changes neither the decode nor the backward kernels.
    assert "fwd2_sm100.cuh" in bench._NOT_IN_HASH["decode"]
    assert "fwd2_sm100.cuh" in bench._NOT_IN_HASH["bwd"]


def test_traffic_entries_name_known_workloads():
    names = {w.name for w in workloads.CONFIGS.values()}
    for key, entry in bench.NCU_TRAFFIC.items():
        base = key[:-len(" bwd")] if key.endswith(" bwd") else key
        assert base in names, key
        assert entry["bytes"] > 0 and len(entry["src"]) == 16, key
