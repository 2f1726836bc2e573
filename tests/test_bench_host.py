"""bench.py's host-side helpers, on CPU: the FLOP convention, the traffic
figures keyed to the CUDA sources they were measured on, per-rank seeds, and
the argument contract (at least 3 warm-up steps)."""

import json
import os

import pytest

import bench


def test_flop_convention_is_8dV_per_token():
    c = dict(T=8192, d=3072, V=128256)
    assert bench.flops_per_token(c) == 8 * 3072 * 128256


def test_traffic_is_reported_only_for_the_sources_it_was_measured_on(tmp_path, monkeypatch):
    h = bench.kernel_source_hash()            # of the real tree's CUDA sources
    assert len(h) == 16
    prof = tmp_path / "profiles"
    prof.mkdir()
    entry = {"kernels": {"8k": {"bwd_dhdw": {"dram_bytes_per_launch": 123}}}}
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: h)
    (prof / "traffic.json").write_text(json.dumps(dict(entry, source_hash="stale")))
    assert bench.profiled_traffic("bwd_dhdw", "8k") is None
    (prof / "traffic.json").write_text(json.dumps(dict(entry, source_hash=h)))
    assert bench.profiled_traffic("bwd_dhdw", "8k") == 123.0
    assert bench.profiled_traffic("bwd_dz", "8k") is None


def test_committed_traffic_file_is_well_formed():
    # bench.py reports these figures only while the sources hash the same
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    assert len(t["source_hash"]) == 16 and "ncu" in t["command"]
    for k in ("fwd_gemm", "bwd_dz", "bwd_dhdw"):
        e = t["kernels"]["8k"][k]
        assert e["dram_bytes_per_launch"] > e["algorithmic_bytes"] > 0


def test_rank_seeds_differ_and_warmup_contract():
    assert len({bench.rank_seed(0, r) for r in range(8)}) == 8
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])
