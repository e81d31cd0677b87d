"""Host logic of the benchmark, on the CPU: the nvidia-smi clock record, the rule
that rejects a number taken under a slowdown or a clock lock, the ncu traffic
figure tied to the kernel sources it was taken on, and the reference arm's
sample budget."""
import json
import os

import pytest

import bench

# index, clocks.sm, clocks.max.sm, power.draw, reasons.active, hw_slowdown,
# hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
LOADED = "0, 1755, 1965, 912.40, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"
CAPPED = "0, 1350, 1965, 996.49, 0x0000000000000004, Not Active, Not Active, Not Active, Active"
THERMAL = "0, 1200, 1965, 850.00, 0x0000000000000020, Not Active, Not Active, Active, Not Active"
LOCKED = "0, 900, 1965, 500.00, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"


def test_clock_lines_are_summarised():
    c = bench.summarise_clock_lines([LOADED, LOADED, CAPPED, "garbage", "0, 17"])
    assert c["samples"] == 3
    assert c["sm_mhz"] == 1755.0  # median of 1755, 1755, 1350
    assert c["sm_max_mhz"] == 1965.0 and c["power_w_max"] == pytest.approx(996.49)
    assert c["reasons"] == ["sw_power_cap"]
    empty = bench.summarise_clock_lines([])
    assert empty["samples"] == 0 and empty["sm_mhz"] is None and empty["reasons"] == []


def test_every_field_maps_to_its_reason():
    fields = bench.ClockSampler.FIELDS.split(",")
    assert len(fields) == 9
    for k, name in enumerate(bench.ClockSampler.NAMES):
        assert fields[5 + k] == "clocks_event_reasons." + name
        parts = ["0", "1800", "1965", "700"] + ["0x0"] + ["Not Active"] * 4
        parts[5 + k] = "Active"
        assert bench.summarise_clock_lines([", ".join(parts)])["reasons"] == [name]


def test_verdict_keeps_power_cap_and_clean_runs():
    assert bench.clock_verdict(bench.summarise_clock_lines([LOADED] * 5)) is None
    assert bench.clock_verdict(bench.summarise_clock_lines([CAPPED] * 5)) is None
    assert bench.clock_verdict({"sm_mhz": None, "sm_max_mhz": None, "reasons": []}) is None


def test_verdict_rejects_slowdowns_and_clock_locks():
    why = bench.clock_verdict(bench.summarise_clock_lines([LOADED, THERMAL, LOADED]))
    assert why is not None and "sw_thermal_slowdown" in why
    for name in bench.REJECTING_REASONS:
        assert bench.clock_verdict({"sm_mhz": 1900.0, "sm_max_mhz": 1965.0,
                                    "reasons": [name]}) is not None
    why = bench.clock_verdict(bench.summarise_clock_lines([LOCKED] * 5))
    assert why is not None and "no reason" in why
    # low clocks under the power cap have a reason and stand
    low_capped = CAPPED.replace("1350", "900")
    assert bench.clock_verdict(bench.summarise_clock_lines([low_capped] * 5)) is None


def test_traffic_is_reported_only_for_the_profiled_sources(monkeypatch):
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    with open(path) as f:
        table = json.load(f)
    # one forward and one backward main kernel (one-CTA or persistent form)
    assert any(k.startswith("fa_fwd_") for k in table)
    assert any(k.startswith("fa_bwd_") for k in table)
    for kernel, ent in table.items():
        assert ent["bytes_per_launch"] > 0 and len(ent["source_sha"]) == 16
        monkeypatch.setattr(bench, "kernel_source_sha", lambda: ent["source_sha"])
        assert bench.profiled_traffic(kernel, ent["workload"]) == ent["bytes_per_launch"]
        assert bench.profiled_traffic(kernel, ent["workload"] + "_other") is None
        monkeypatch.setattr(bench, "kernel_source_sha", lambda: "0" * 16)
        assert bench.profiled_traffic(kernel, ent["workload"]) is None
    assert bench.profiled_traffic("no_such_kernel", "long_b1h8_n16384_d128") is None


def test_source_hash_covers_every_kernel_source(tmp_path, monkeypatch):
    csrc = tmp_path / "io_aware_attention_flashattention_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cu").write_text("int a;")
    (csrc / "b.cuh").write_text("int b;")
    (csrc / "notes.txt").write_text("x")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_sha()
    (csrc / "notes.txt").write_text("y")
    assert bench.kernel_source_sha() == h0
    (csrc / "b.cuh").write_text("int b; ")
    assert bench.kernel_source_sha() != h0


def test_peaks_come_from_the_measured_file():
    peaks, src = bench.load_peaks()
    if os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")):
        assert src == "measured"
    else:
        assert src == "fallback" and peaks == bench.FALLBACK_PEAKS
    assert peaks["bf16_tflops"] > 0 and peaks["hbm_gbs"] > 0


def test_oracle_sample_is_bounded_and_counts_visible_pairs():
    import time

    from io_aware_attention_flashattention_b200.inputs import WORKLOADS

    w = WORKLOADS["gpt2_causal_b8h12_n1024_d64"]
    t0 = time.perf_counter()
    flops, secs, rows, threads = bench.oracle_sample(w, 0.3, rng_seed=3)
    wall = time.perf_counter() - t0
    assert rows >= 1 and threads >= 1 and 0 < secs < wall
    assert wall < 30.0
    # causal: a row sees between 1 and N keys; 10 flops per (row, key, head-dim element)
    per_row = flops / rows / (10.0 * w.d)
    assert 1.0 <= per_row <= w.N
    assert per_row == pytest.approx((w.N + 1) / 2, rel=0.5)


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` runs the oracle alone on the host cores (no GPU)
    and prints one JSON line with the reference arm's keys."""
    import subprocess
    import sys

    out = subprocess.run(
        [sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference",
         "--workload", "gpt2_causal_b8h12_n1024_d64", "--steps", "2", "--warmup", "1",
         "--reference-seconds", "1.5"],
        capture_output=True, text=True, timeout=120, cwd=bench.ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["value"] > 0
    assert d["config"]["workload"] == "gpt2_causal_b8h12_n1024_d64"
    # the same config object our arm prints, so the two lines compare as one workload
    from io_aware_attention_flashattention_b200.inputs import WORKLOADS
    assert d["config"] == bench.workload_config(WORKLOADS["gpt2_causal_b8h12_n1024_d64"], 1)
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun only rank 0 runs the oracle; the other ranks exit 0 at once."""
    import subprocess
    import sys

    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run(
        [sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference",
         "--gpus", "2", "--steps", "3", "--warmup", "3"],
        capture_output=True, text=True, timeout=60, cwd=bench.ROOT, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    assert not [ln for ln in out.stdout.splitlines() if ln.startswith("{")]


def test_visible_pairs_match_brute_force():
    """The masked FLOP count of the secondary configurations: pairs kept by causal, a
    window and a block mask, against an N x N boolean matrix."""
    import numpy as np

    rng = np.random.default_rng(3)
    for N in (1, 77, 128, 300, 1000):
        T = (N + 127) // 128
        for causal in (False, True):
            for window in (None, (5, 7), (-1, 3), (10, -1), (512, 512)):
                for bm in (None, (rng.random((T, T)) < 0.5).astype(np.uint8)):
                    i = np.arange(N)[:, None]
                    j = np.arange(N)[None, :]
                    vis = np.ones((N, N), bool)
                    if causal:
                        vis &= j <= i
                    if window:
                        left, right = window
                        if left >= 0:
                            vis &= j >= i - left
                        if right >= 0:
                            vis &= j <= i + right
                    if bm is not None:
                        vis &= bm[i // 128, j // 128] != 0
                    assert bench.visible_pairs(N, causal, window, bm) == int(vis.sum())
