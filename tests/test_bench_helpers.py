"""CPU checks of bench.py's host-side helpers: the clock-sample summary (median
SM clock inside the timed window, throttle reasons seen there), the
committed-traffic lookup keyed by kernel source hash (null once the source
differs), and the fused-MLP workload check."""
import json
import os
import tempfile

import bench
from activation_sparsity_prep_b200 import workloads as wl


def _sampler_with(lines, window):
    s = bench.ClockSampler(0)
    fd, s.path = tempfile.mkstemp(suffix=".csv")
    with os.fdopen(fd, "w") as f:
        f.write("\n".join(lines) + "\n")
    s.window = window
    return s


def _line(ts, sm, reasons=("Not Active",) * 4):
    return f"{ts}, 0, {sm}, 1965, 700.0, 0x0, " + ", ".join(reasons)


def test_clock_summary_keeps_samples_inside_the_window():
    import time
    t0 = time.mktime(time.strptime("2026/12/02 10:00:00", "%Y/%m/%d %H:%M:%S"))
    lines = [_line("2026/12/02 10:00:00.100", 1200),                        # before the window
             _line("2026/12/02 10:00:01.100", 1965),
             _line("2026/12/02 10:00:01.200", 1950, ("Not Active", "Not Active", "Not Active", "Active")),
             _line("2026/12/02 10:00:01.300", 1965),
             _line("2026/12/02 10:00:03.000", 900, ("Active", "Not Active", "Not Active", "Not Active"))]
    s = _sampler_with(lines, (t0 + 1.0, t0 + 1.5))
    out = s.summary()
    assert out["samples"] == 3 and out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]                                  # hw_slowdown fell outside
    assert out["window"] == "samples inside the timed region"


def test_clock_summary_without_samples_in_the_window_says_so():
    lines = [_line("2026/12/02 10:00:00.100", 1965)]
    s = _sampler_with(lines, (0.0, 1.0))
    out = s.summary()
    assert out["samples"] == 1 and out["window"].startswith("all samples")


def test_profiled_traffic_needs_the_same_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps({"k": {"dram_bytes": 123, "source_sha": "abc"}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k", "abc") == 123
    assert bench.profiled_traffic("k", "def") is None
    assert bench.profiled_traffic("missing", "abc") is None


def test_fused_mlp_workloads():
    assert bench.mlp_fusable(wl.WORKLOADS["llama8b"]) and bench.mlp_fusable(wl.WORKLOADS["qwen3moe"])
    assert bench.mlp_fusable(wl.WORKLOADS["tiny_mlp"])
    assert not bench.mlp_fusable(wl.WORKLOADS["tiny"]) and not bench.mlp_fusable(wl.WORKLOADS["sweep"])


def test_prepare_bytes_per_element():
    """Read X (bf16) + backbone codes and scales + residual codes and scales:
    zero-filled backbones store K/2 code bytes a row, the pair backbone K/4
    plus K/16 bytes of pair indices."""
    assert bench.PREP_BYTES_PER_ELEM[(0, 1)] == 2 + 0.5 + 1 / 16 + 0.5 + 1 / 16
    assert bench.PREP_BYTES_PER_ELEM[(1, 1)] == 2 + 0.5 + 1 / 32 + 0.5 + 1 / 32
    assert bench.PREP_BYTES_PER_ELEM[(1, 0)] == 2 + 0.25 + 1 / 16 + 1 / 32 + 0.5 + 1 / 32


def test_nm_parsing():
    import argparse
    a = argparse.Namespace(nm="4:8p")
    assert bench.nm_of(a) == (4, 8) and bench.pairs_of(a)
    a = argparse.Namespace(nm="2:4")
    assert bench.nm_of(a) == (2, 4) and not bench.pairs_of(a)


def test_traffic_key_names_the_kernel_form():
    """A capture of the own-scale launch must not be reported for the shared
    residual scale or the pair backbone, which run other kernel instances."""
    import argparse
    ns = lambda nm="2:4", residual="own", fuse_mlp=False: argparse.Namespace(nm=nm, residual=residual,
                                                                            fuse_mlp=fuse_mlp)
    assert bench.traffic_tag(ns()) == ""
    assert bench.traffic_tag(ns(residual="shared")) == "_shared"
    assert bench.traffic_tag(ns(nm="4:8p")) == "_pairs"
    assert bench.traffic_tag(ns(fuse_mlp=True)) == "_fused"
