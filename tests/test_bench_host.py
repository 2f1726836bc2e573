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
    assert len(t["source_hash"]) == 16
    for k in ("fwd_gemm", "bwd_dz", "bwd_dhdw"):
        assert "ncu" in t["commands"][k] and "--clock-control none" in t["commands"][k]
        e = t["kernels"]["8k"][k]
        assert e["dram_bytes_per_launch"] > e["algorithmic_bytes"] > 0


def test_rank_seeds_differ_and_warmup_contract():
    assert len({bench.rank_seed(0, r) for r in range(8)}) == 8
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_clock_summary_keeps_only_samples_inside_the_timed_region():
    # idle samples before and after the window (1965 MHz) must not enter the
    # median; the loaded ones inside it (1300-1400 MHz, power cap) do
    samples = [(0.0, 1965.0, 1965.0, 150.0, set()), (0.1, 1965.0, 1965.0, 150.0, set())]
    samples += [(1.0 + 0.02 * i, 1300.0 + 5 * i, 1965.0, 990.0, {"sw_power_cap"})
                for i in range(21)]
    samples += [(2.0, 1965.0, 1965.0, 200.0, set())]
    s = bench.summarise_clocks(samples, 0.9, 1.5, "test")
    assert s["samples"] == 21 and s["sm_mhz"] == 1350.0 and s["sm_min_mhz"] == 1300.0
    assert s["sm_max_mhz"] == 1965.0 and s["reasons"] == ["sw_power_cap"]
    assert s["power_w"] == 990.0
    assert bench.summarise_clocks(samples, 5.0, 6.0) is None


def test_cpu_description_names_the_host():
    model, n = bench.cpu_description()
    assert n >= 1 and (model is None or isinstance(model, str))


def test_backward_flops_add_up_to_6dV_per_token():
    # the per-kernel split of the backward (each block's dZ recompute and its
    # dH + dW) covers 6 d V per token exactly, whatever the blocking
    for T, d, V, plan in ((8192, 3072, 128256, (8192, 14336, 9)),
                          (262144, 4096, 128256, (6144, 64256, 2)),
                          (1000, 64, 3000, (256, 3008, 1))):
        f = bench.kernel_flops_per_step(T, d, V, plan)
        back = f["bwd_dz"] + f["bwd_dhdw"]
        assert abs(back - 6.0 * T * V * d) <= 1e-9 * back
        n = bench.backward_launches(T, V, plan)
        assert n["bwd_dz"] == n["bwd_dhdw"] == len(bench.backward_blocks(T, V, plan))
