"""Host-side pieces of bench.py: the clock-sample window and the oracle sample sizing."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


IDLE = ["Not Active"] * 4
CAP = ["Not Active", "Not Active", "Not Active", "Active"]


def test_clock_summary_keeps_only_the_timed_window(bench):
    rows = [(100.0, 1965, 1965, 150, IDLE), (100.1, 1965, 1965, 150, IDLE),
            (100.2, 1400, 1965, 990, CAP), (100.3, 1380, 1965, 995, CAP), (100.4, 1390, 1965, 990, CAP),
            (100.5, 1965, 1965, 200, IDLE)]
    s = bench.ClockSampler.summarize(rows, (100.15, 100.45))
    assert s["sm_mhz"] == 1390 and s["samples"] == 3 and s["reasons"] == ["sw_power_cap"]
    assert s["scope"] == "timed region" and s["sm_max_mhz"] == 1965


def test_clock_summary_short_window_and_thermal(bench):
    hot = ["Active", "Not Active", "Active", "Not Active"]
    rows = [(10.0, 1965, 1965, 100, IDLE), (10.1, 1200, 1965, 900, hot), (10.9, 1965, 1965, 100, IDLE)]
    s = bench.ClockSampler.summarize(rows, (10.12, 10.15))  # no sample inside: within one period
    assert s["samples"] == 1 and s["sm_mhz"] == 1200
    assert s["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"] and s["scope"].startswith("within")
    s = bench.ClockSampler.summarize(rows, (20.0, 21.0))
    assert s["sm_mhz"] is None and s["reasons"] == ["unsampled"]
    assert bench.ClockSampler.summarize([], None)["reasons"] == ["unsampled"]


def test_nvidia_smi_timestamp_parses(bench):
    t = bench.ClockSampler._stamp("2026/12/02 10:00:00.250")
    assert t is not None and abs((t % 1) - 0.25) < 1e-6
    assert bench.ClockSampler._stamp("garbage") is None


def test_oracle_sample_sizing_separates_fixed_cost(bench, monkeypatch):
    # a call costs 1 s fixed + 5 ms per row: 12 s of work is 2200 rows, not 8 * 12 / t(8)
    monkeypatch.setattr(bench, "oracle_sample", lambda d, n, Wf: 1.0 + 0.005 * n)
    assert bench.calibrate_rows(None, None, 12.0, 4096) == 2200
    assert bench.calibrate_rows(None, None, 100.0, 4096) == 4096
    assert bench.calibrate_rows(None, None, 0.5, 4096) == 8


def test_reference_arm_runs_on_the_host_and_samples_at_most_the_batch():
    """bench.py --impl reference: the oracle as it stands, one JSON line, a
    sample no larger than the workload's batch."""
    import json
    import subprocess
    import sys

    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["dtype"] == "f64" and line["config"]["workload"] == "tiny"
    assert line["config"]["sample_tokens_per_step"] <= 512
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["value"] > 0 and line["unit"] == "tokens/s"


def test_recorded_traffic_follows_the_source_hash(bench, tmp_path, monkeypatch):
    """The roofline's traffic figure is read from the committed capture only while
    the five sources that decide the captured launches hash to the recorded value."""
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    src = tmp_path / "linear_cross_entropy_04_b200" / "csrc"
    src.mkdir(parents=True)
    for f in bench.KERNEL_SOURCES:
        (tmp_path / f).write_text("kernel " + f)
    assert {os.path.basename(f) for f in bench.KERNEL_SOURCES} >= {"flce.cu", "aux_kernels.cuh", "tc_gemm2.cuh"}
    h = bench.kernel_source_hash()
    (prof / "tc_gemm_pair_kernel_toy_dram.md").write_text(
        f"# toy\n- kernel_source_sha256_16: `{h}`\n- dram_bytes_per_launch: `123456`\n")
    assert bench.recorded_traffic("toy")["bytes_per_launch"] == 123456.0
    (tmp_path / bench.KERNEL_SOURCES[-1]).write_text("changed")
    assert bench.recorded_traffic("toy") is None
    assert bench.recorded_traffic("no_such_workload") is None


def test_workload_size_overrides_rename_the_workload(bench, monkeypatch):
    import sys

    monkeypatch.setattr(sys, "argv", ["bench.py", "--BT", "1024", "--V", "32768"])
    w = bench.workload(bench.parse())
    assert (w.BT, w.H, w.V) == (1024, 4096, 32768) and w.name != "llama3_8b_seq"
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    assert bench.workload(bench.parse()).name == "llama3_8b_seq"


def test_grad_w_exchange_choice(bench):
    """N > 1 reduce-scatters grad_W by rows by default (all-reduce when V does not
    divide by N); one GPU has no exchange unless --dp asks for the path."""
    import argparse

    b = bench
    ns = lambda **k: argparse.Namespace(**{"grad_w_exchange": "reduce_scatter", "dp_fused_grad_w": False,
                                          "dp": False, **k})
    assert b.grad_w_exchange(ns(), 128256, 1) is None
    assert b.grad_w_exchange(ns(dp=True), 128256, 1) == "reduce_scatter"
    assert b.grad_w_exchange(ns(), 128256, 8) == "reduce_scatter"
    assert b.grad_w_exchange(ns(), 128257, 8) == "all_reduce"
    assert b.grad_w_exchange(ns(grad_w_exchange="all_reduce"), 128256, 8) == "all_reduce"
    assert b.grad_w_exchange(ns(dp_fused_grad_w=True), 128256, 8) == "fused"


def test_source_hash_ignores_comments_but_not_code(bench):
    """The recorded DRAM traffic stays valid across comment edits and is voided by
    any code edit: the hash is taken over the code with comments removed."""
    src = open(os.path.join(ROOT, "linear_cross_entropy_04_b200", "csrc", "tc_gemm2.cuh"), encoding="utf-8").read()
    assert "constexpr int KSYNC_EVERY = 16;" in src
    reworded = src.replace("// Soft K-synchronisation", "// Soft K-sync (reworded)") + "\n/* a new\n block */\n"
    assert reworded != src and bench.code_only(reworded) == bench.code_only(src)
    assert bench.code_only(src.replace("KSYNC_EVERY = 16;", "KSYNC_EVERY = 8;")) != bench.code_only(src)
    assert bench.code_only('x = 1; // a\n/* b\n c */ y =\t2;') == "x = 1; y = 2;"
