"""Host-side pieces of bench.py (no GPU): the algorithmic bytes the
roofline divides by, the source-hash keyed traffic records, the peaks."""
import json
import os

import bench


def test_algorithmic_bytes_per_parameter():
    # theta r+w 8, BF16 grad 2, m and v codes r+w 4, (k, s) x 2 states x r+w / G
    assert bench.bytes_per_param(128) == 14.25
    assert bench.bytes_per_param(32) == 15.0
    assert bench.bytes_per_param(1024) == 14.03125


def test_step_traffic_record_is_keyed_by_the_kernel_sources():
    with open(os.path.join(bench.ROOT, "profiles", "adamw_fp8_step_traffic.json")) as f:
        rec = json.load(f)
    n = 6888095744
    got = bench.recorded_traffic(n, 128)
    if rec["kernel_source_hash"] == bench.kernel_source_hash():
        assert got == rec["dram_bytes_per_param"] * n
        assert 14.0 <= rec["dram_bytes_per_param"] <= 14.25      # no re-reads
    else:
        assert got is None
    assert bench.recorded_traffic(n, 64) is None                  # captured at G = 128 only


def test_activation_traffic_record():
    with open(os.path.join(bench.ROOT, "profiles", "group_quant_1xG_traffic.json")) as f:
        rec = json.load(f)
    got = bench.recorded_act_traffic(rec["elements"])
    if rec["kernel_source_hash"] == bench.kernel_source_hash(bench.ACT_KERNEL_SOURCES):
        assert got == rec["dram_bytes_read"] + rec["dram_bytes_write"]
        # the BF16 input is read exactly once
        assert rec["dram_bytes_read"] <= 2 * rec["elements"] * 1.01
    else:
        assert got is None
    assert bench.recorded_act_traffic(rec["elements"] + 1) is None


def test_peaks_come_from_the_measured_file():
    peaks, kind = bench.measured_peaks()
    assert kind in ("measured", "fallback")
    assert peaks["hbm_gbs"] > 1000
