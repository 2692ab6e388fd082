"""Host-side logic of bench.py, on the CPU: the ncu-summary traffic lookup, the
clock-sample summary and the replica throughput arithmetic."""
import os

import pytest

import bench


def test_stored_traffic_parses_the_committed_summaries():
    for kernel, (fname, _) in bench.TRAFFIC_PROFILES.items():
        assert os.path.exists(os.path.join(bench.ROOT, "profiles", fname)), fname
        v = bench.stored_traffic(kernel)
        # null is allowed (sources changed since the capture); a value must be a byte count
        assert v is None or v > 1e6, (kernel, v)


def test_stored_traffic_is_null_once_the_sources_change(monkeypatch):
    monkeypatch.setattr(bench, "kernel_source_hash", lambda names: "0" * 16)
    for kernel in bench.TRAFFIC_PROFILES:
        assert bench.stored_traffic(kernel) is None
    assert bench.stored_traffic("no_such_kernel") is None


def test_decode_traffic_matches_its_algorithmic_bytes():
    """The fused decode stack reads each selected expert and each router once:
    48 x (10 x 1,769,472 + 4,194,304) bytes per token."""
    v = bench.stored_traffic("stack_decode")
    if v is None:
        pytest.skip("decode kernel sources changed since the committed capture")
    algorithmic = 48 * (10 * 1_769_472 + 4_194_304)
    assert 1.0 <= v / algorithmic < 1.05


def _clock_summary(tmp_path, lines):
    c = object.__new__(bench.Clocks)
    c.path = str(tmp_path / "clocks.csv")
    with open(c.path, "w") as f:
        f.write("\n".join(lines) + "\n")
    c.f = open(os.devnull, "w")
    c.p = None
    return c.stop()


def test_clock_summary_median_max_and_reasons(tmp_path):
    row = "2026/01/01 00:00:00.000, {sm}, 1965, 700.0, 0x0, {hw}, Not Active, Not Active, {cap}"
    lines = [row.format(sm=s, hw="Not Active", cap=c) for s, c in
             ((1965, "Not Active"), (1950, "Active"), (1965, "Not Active"))]
    s = _clock_summary(tmp_path, lines)
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    lines.append(row.format(sm=1200, hw="Active", cap="Not Active"))
    s = _clock_summary(tmp_path, lines)
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_nvml_sample_summary_reasons_from_the_bitmask():
    # bits: sw_power_cap 0x4, hw_slowdown 0x8, sw_thermal 0x20, hw_thermal 0x40; idle (0x1) is not a reason
    s = bench.summarize_clock_samples([(1965.0, 0x0), (1950.0, 0x4), (1965.0, 0x1)], 1965.0)
    assert s["sm_mhz"] == 1965.0 and s["sm_mhz_min"] == 1950.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    s = bench.summarize_clock_samples([(1200.0, 0x8 | 0x40), (1965.0, 0x20)], 1965.0)
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert bench.summarize_clock_samples([], 1965.0)["sm_mhz"] is None


def test_clock_summary_without_samples(tmp_path):
    s = _clock_summary(tmp_path, [])
    assert s["sm_mhz"] is None and s["reasons"] == ["nvidia-smi unavailable"]


def test_replica_throughput_sums_work_over_the_slowest_rank():
    # 4 replicas, 10 steps of 1 token each, slowest rank 20 ms: 40 tokens / 0.02 s
    assert bench.replica_throughput(4, 10, 1, 20.0) == pytest.approx(2000.0)
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_workload_descriptions_name_the_block_formats():
    from synth import configs
    cfg = configs.get(2)
    assert bench.format_desc(cfg) == "Q2"
    mx = configs.mixed(cfg, bench.MIXED_EVERY)
    assert len(mx.fmt_layers) == 48 and mx.fmt_layers[:5] == (4, 2, 2, 2, 4)
    assert bench.format_desc(mx).startswith("mixed: Q4 in 12 of 48 layers")
    # a mixed stack's bytes per layer follow each layer's own format
    per_layer = [mx.for_layer(l).expert_bytes() for l in range(48)]
    assert per_layer.count(2_949_120) == 12 and per_layer.count(1_769_472) == 36


def test_ngram_workload_bytes():
    """4096 tokens x 16 rows: 160-byte Q4 rows of 256 read, 1 KB of fp32 written
    per row, 12 bytes of ids per token."""
    from synth import configs
    nc = configs.NGRAM
    assert nc.row_bytes() == 160 and nc.R * nc.row_bytes() == 671_088_640
    assert nc.T * (12 + 16 * (nc.row_bytes() + 4 * nc.D)) == 77_643_776
