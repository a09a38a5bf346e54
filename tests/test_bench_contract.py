"""The benchmark's output contract, checked on the CPU: the reference arm (the
oracle timed on the host cores) prints one JSON line with the contract's keys,
only rank 0 prints under a multi-rank launch, and the GPU arm fails loudly when
there is no GPU instead of falling back to anything else."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT,
                          env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _run(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1",
              "--cpu-seconds", "0.05"])
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "gpu_launches"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["steps"] == 2 and line["warmup"] == 1 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["config"]["workload"] == "tiny"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["gpu_launches"] == 0
    # the line says what ran: `steps` bounded samples of ms_per_step each, whose
    # throughput is extrapolated to the full workload
    assert line["extrapolated"] is True and line["est_full_step_s"] > 0
    assert line["steps"] * line["ms_per_step"] / 1e3 <= line["wall_s"] + 1e-6


def test_reference_arm_prints_on_rank_zero_only():
    r = _run(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0",
              "--cpu-seconds", "0.05"], {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert not [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]


def test_gpu_arm_fails_loudly_without_a_gpu():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    r = _run(["--workload", "tiny", "--steps", "1", "--warmup", "3", "--no-cpu-baseline"])
    assert r.returncode != 0
    assert '"metric"' not in r.stdout


def test_clock_summary_takes_the_median_and_the_active_reasons_in_the_window(tmp_path):
    """The clock record of the JSON line, from nvidia-smi's CSV rows: only rows
    inside the timed region count; the SM clock is their median; a throttle
    reason is listed when any counted row shows it active."""
    import datetime
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0)

    def row(dt_s, sm, reasons):
        ts = (t0 + datetime.timedelta(seconds=dt_s)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        flags = ["Active" if r in reasons else "Not Active"
                 for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                           "sw_power_cap")]
        return ", ".join([ts, "0", str(sm), "1965", "700.0", "0x0"] + flags)

    path = tmp_path / "clocks.csv"
    path.write_text("\n".join([
        row(0.0, 900, {"hw_slowdown"}),          # before the window: ignored
        row(1.0, 1700, set()),
        row(1.5, 1600, {"sw_power_cap"}),
        row(2.0, 1800, set()),
        "garbled line",
        row(9.0, 500, {"sw_thermal_slowdown"}),  # after the window: ignored
    ]) + "\n")
    s = bench.ClockSampler(0)
    s.proc, s.path = object(), str(path)        # as if nvidia-smi had written the file
    got = s.summary((t0 + datetime.timedelta(seconds=0.5)).timestamp(),
                    (t0 + datetime.timedelta(seconds=2.5)).timestamp())
    assert got == {"sm_mhz": 1700.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 3}


def test_roofline_traffic_scales_with_a_rank_share_of_the_heads():
    """The committed DRAM record is for a whole call; a rank that runs 32/N of
    the heads reports that share per launch, a replica the whole."""
    import importlib.util
    import json as _json
    import synth
    spec = importlib.util.spec_from_file_location("bench_mod2", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    with open(bench.TRAFFIC_FILE) as f:
        rec = _json.load(f)["720p"]
    if rec["kernel_hash"] != bench.kernel_hash():
        pytest.skip("the record predates the current kernel source")
    wl = synth.WORKLOADS["720p"]
    assert bench.load_traffic(wl) == rec["bytes_per_launch"]
    for world in (2, 4, 8):
        part, _, _ = bench.rank_problem(wl, 1, world, "heads")
        assert bench.load_traffic(part) == rec["bytes_per_launch"] / world
    rep, _, _ = bench.rank_problem(wl, 1, 2, "replicas")
    assert bench.load_traffic(rep) == rec["bytes_per_launch"]
    assert bench.load_traffic(synth.WORKLOADS["tiny"]) is None     # no record
