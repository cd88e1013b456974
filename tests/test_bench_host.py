"""Host-side pieces of bench.py that need no GPU: the DRAM-traffic lookup (scaled by units, null
once the kernel's source has changed), the nvidia-smi clock parsing (median clock, throttle
reasons), the measured peaks, and the token count of every workload."""
import hashlib
import json
import os

import bench


def test_traffic_scales_with_units_and_follows_the_source_hash():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        kernels = json.load(f)["kernels"]
    checked = 0
    for name, e in kernels.items():
        with open(os.path.join(bench.ROOT, e["source"]), "rb") as f:
            current = hashlib.sha256(f.read()).hexdigest() == e["sha256"]
        got = bench.kernel_traffic(name, 2 * e["units"])
        if not current:
            assert got is None, name
            continue
        checked += 1
        assert got["bytes"] == 2 * (e["read"] + e["write"])
        assert got["scale"] == 2.0 and got["profile"] == e["profile"]
    assert checked > 0
    assert bench.kernel_traffic("no_such_kernel", 1.0) is None
    assert bench.kernel_traffic(next(iter(kernels)), None) is None


def test_traffic_is_null_once_the_source_changes(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    src = root / "k.cu"
    src.write_text("kernel v1\n")
    entry = {"source": "k.cu", "sha256": hashlib.sha256(b"kernel v1\n").hexdigest(), "capture": "c",
             "read": 100, "write": 50, "units": 10, "unit": "row", "profile": "p.md"}
    (root / "profiles" / "traffic.json").write_text(json.dumps({"kernels": {"k": entry}}))
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.kernel_traffic("k", 20)["bytes"] == 300
    src.write_text("kernel v2\n")
    assert bench.kernel_traffic("k", 20) is None


def test_clock_samples_parse():
    s = bench.ClockSampler(0)

    class _Proc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    s.proc = _Proc()
    s.lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 990.3, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 710.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    out = s.stop()
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0 and out["samples"] == 3
    assert out["reasons"] == ["sw_power_cap"]
    s2 = bench.ClockSampler(0)
    assert s2.stop()["reasons"] == ["nvidia-smi unavailable"]


def test_measured_peaks_and_token_counts():
    p = bench.measured_peaks()
    assert p["hbm_gbs"] > 1000 and p["bf16_tflops"] > 100
    if os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")):
        assert p["source"] == "measured"
    for w in bench.WORKLOADS:
        assert bench._tokens(w) > 0, w
    assert bench.DEFAULT_WORKLOAD in bench.WORKLOADS


def test_oracle_sample_scales_to_the_whole_step():
    """The oracle's bounded sample for the prefill workload: one thread runs 1 head x 1024 tokens,
    and the estimate scales it by 32 (tokens) x 64 (heads) to the 32,768-token step."""
    smp = bench.OracleSample("kda_prefill_32k", nth=1)
    assert len(smp.parts) == 1 and abs(smp.parts[0][1] - 32 * 64) < 1e-9
    assert "1 heads x 1024 tokens" in smp.sample
    est = smp.run()
    assert est > 0
    r = bench.cpu_oracle_rate("kda_prefill_32k", nth=1, repeats=3)
    assert r["repeats"] == 3 and r["cores"] == 1 and r["value"] > 0 and r["spread"] >= 0


def test_reference_arm_reports_the_samples_it_ran(capsys):
    """--impl reference: K timed steps, each one bounded sample; ms_per_step is a sample's wall
    time, so ms_per_step x steps is the time the timed samples actually took."""
    import time
    t0 = time.perf_counter()
    assert bench.main(["--impl", "reference", "--workload", "kda_prefill_32k", "--steps", "3", "--warmup", "3"]) == 0
    wall = time.perf_counter() - t0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 3 and line["warmup"] == 3
    assert line["ms_per_step"] * line["steps"] / 1000.0 < wall
    assert line["cpu_baseline"]["single_thread"]["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
