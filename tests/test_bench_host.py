"""Host-side pieces of bench.py (no GPU): the algorithmic bytes the
roofline divides by, the source-hash keyed traffic records, the peaks."""
import json
import os

import pytest

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


def test_clock_samples_are_summarised(tmp_path, monkeypatch):
    """The clock record of the timed region: median SM clock, the maximum,
    and every throttle reason seen active at least once (the lines are
    nvidia-smi's csv,noheader,nounits output; malformed lines are skipped)."""
    monkeypatch.setenv("COAT_BENCH_LOG_DIR", str(tmp_path))
    s = bench.ClockSampler(None)

    class Done:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    rows = ["1965, 1965, 900.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
            "1800, 1965, 1000.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
            "1750, 1965, 998.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
            "garbage line",
            "[N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active"]
    with open(s.path, "w") as f:
        f.write("\n".join(rows) + "\n")
    s.proc, s.out = Done(), open(os.devnull, "w")
    got = s.stop()
    assert got == {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "samples": 3,
                   "reasons": ["sw_power_cap"]}
    s2 = bench.ClockSampler(None)
    assert s2.stop() is None                    # never started (no nvidia-smi): no record


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores, no GPU)
    prints one JSON line with the keys the bench contract asks of that arm."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2",
                        "--warmup", "1", "--ref-sample", "16384"], cwd=bench.ROOT,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "params/s" and line["higher_is_better"] is True
    assert line["steps"] == 2 and line["warmup"] == 1 and line["value"] > 0
    assert line["config"]["group_size"] == 128 and line["config"]["v_fmt"] == "e4m3"
    assert "16384" in line["config"]["workload"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "params/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_launch_command_runs_this_script_under_torchrun_on_localhost():
    cmd = bench.launch_command(8, ["--gpus", "8", "--steps", "3"], 900, 29555)
    assert cmd[:4] == ["timeout", "-k", "60", "900"]
    i = cmd.index("torch.distributed.run")
    assert cmd[i - 1] == "-m"
    assert "--nproc-per-node=8" in cmd and "--nnodes=1" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[cmd.index("--master-port") + 1] == "29555"
    assert cmd[-4:] == [os.path.abspath(bench.__file__), "--gpus", "8", "--steps", "3"][-4:]


def test_gpus_n_starts_n_ranks_that_all_join():
    """`bench.py --gpus 2` outside torchrun starts two ranks itself; with no
    GPU here they join over gloo, and rank 0's JSON line reports both."""
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    out = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--gpus", "2",
                          "--workload", "ranks", "--launch-timeout", "240"],
                         capture_output=True, text=True, timeout=300, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(l) for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    assert lines[0]["n_gpus"] == 2 and lines[0]["ranks_joined"] == 2


def test_clock_normalised_scales_by_max_over_median_clock():
    import bench
    got = bench.clock_normalised(3.0e11, {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0})
    assert got["params_per_s_at_max_clock"] == pytest.approx(3.0e11 * 1965.0 / 1800.0)
    assert bench.clock_normalised(1.0, None) is None
    assert bench.clock_normalised(1.0, {"sm_mhz": None, "sm_max_mhz": 1965.0}) is None


def test_zero1_peer_step_bytes():
    """One rank's one-kernel ZeRO-1 step on L shard parameters: HBM = the
    step's bytes + the BF16 copy of its shard + its gradient read by and the
    others' shards written into its memory, 2 (W - 1) B each; NVLink per
    direction 4 (W - 1) B per shard parameter; one rank moves nothing over
    links."""
    L = 1 << 20
    one = bench.zero1_peers_bytes(L, 1, 128)
    assert one["hbm"] == (14.25 + 2) * L and one["link_per_direction"] == 0
    eight = bench.zero1_peers_bytes(L, 8, 128)
    assert eight["link_per_direction"] == 28 * L
    assert eight["hbm"] == (14.25 + 2 + 28) * L


def test_source_hash_up_to_a_marker(tmp_path):
    """A (path, marker) source counts only the text before the marker line:
    an edit after it keeps the hash, an edit before it changes it."""
    f = tmp_path / "k.cuh"
    f.write_text("a\n// ---- B\nb\n")
    h0 = bench.kernel_source_hash([(str(f), "// ---- B")])
    f.write_text("a\n// ---- B\nb changed\n")
    assert bench.kernel_source_hash([(str(f), "// ---- B")]) == h0
    f.write_text("a changed\n// ---- B\nb\n")
    assert bench.kernel_source_hash([(str(f), "// ---- B")]) != h0
    with pytest.raises(ValueError):
        bench.kernel_source_hash([(str(f), "// ---- missing")])
