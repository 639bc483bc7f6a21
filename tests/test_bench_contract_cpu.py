"""bench.py's host-side contract on CPU: the reference arm's JSON line (the
float64 oracle timed on the host cores, so it runs here), its behaviour on
ranks other than 0, and the parsing of the clock samples taken during the
timed region."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_bench(args, env_extra=None, timeout=600):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT,
                          env=env, capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_contract_line():
    r = _run_bench(["--impl", "reference", "--workload", "small", "--steps", "1",
                    "--warmup", "0"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] == 0
    assert line["dtype"] == "f64" and line["vs_baseline"] is None
    assert line["config"]["workload"] == "hybrid_layer_T12_N4032_H24_d128"
    assert "0.30 GB per activation" in line["config"]["l2"]
    cpu = line["cpu_baseline"]
    assert set(cpu) == {"value", "unit", "cores", "kind", "sample"}
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # tokens per step over the step time
    assert line["value"] == pytest.approx(12 * 4032 / (line["ms_per_step"] / 1e3), rel=1e-9)


def test_reference_arm_other_ranks_exit_without_work():
    r = _run_bench(["--impl", "reference", "--workload", "small", "--steps", "1",
                    "--warmup", "0"], env_extra={"RANK": "1", "WORLD_SIZE": "2"}, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


class _FakeSampler:
    """Stands in for the nvidia-smi process (already written its samples)."""

    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass


def _clocks(tmp_path, rows):
    import bench
    path = tmp_path / "clocks.csv"
    path.write_text("".join(r + "\n" for r in rows))
    out = bench.clocks_stop((_FakeSampler(), str(path)))
    assert not path.exists()  # the sample file is removed
    return out


def test_clock_samples_power_cap_only(tmp_path):
    rows = ["0, 1650, 1965, 998.12, 0x0000000000000004, Not Active, Not Active, Not Active, "
            "Active",
            "0, 1665, 1965, 1001.40, 0x0000000000000004, Not Active, Not Active, Not Active, "
            "Active",
            "0, 1635, 1965, 990.00, 0x0000000000000004, Not Active, Not Active, Not Active, "
            "Active",
            "garbled line",
            "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active"]
    out = _clocks(tmp_path, rows)
    assert out == {"sm_mhz": 1650.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 3}


def test_clock_samples_report_every_slowdown_seen(tmp_path):
    rows = ["0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active",
            "0, 1200, 1965, 700.0, 0x8, Active, Not Active, Not Active, Not Active",
            "0, 1100, 1965, 700.0, 0x40, Not Active, Active, Active, Not Active"]
    out = _clocks(tmp_path, rows)
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert out["sm_mhz"] == 1200.0 and out["samples"] == 3


def test_clock_sampler_missing():
    import bench
    out = bench.clocks_stop((None, None))
    assert out["sm_mhz"] is None and out["reasons"] == ["nvidia-smi unavailable"]
