"""Host logic of bench.py that needs no GPU: the clock sampler keeps only the samples
taken inside the timed region and reads the throttle reasons from them."""
import os
import stat
import sys
import time

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

# A stand-in for nvidia-smi's query loop: prints one CSV sample every -lms milliseconds.
# The SM clock counts up from 1000 so the test can tell which samples were kept; the
# power-cap column reads "Active" from the fourth sample on.
FAKE = """#!{py}
import sys, time
period = int(sys.argv[sys.argv.index("-lms") + 1]) / 1000.0
i = 0
while True:
    cap = "Active" if i >= 3 else "Not Active"
    print(f"0, {{1000 + i}}, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, {{cap}}", flush=True)
    i += 1
    time.sleep(period)
"""


@pytest.fixture
def fake_smi(tmp_path):
    p = tmp_path / "fake-smi"
    p.write_text(FAKE.format(py=sys.executable))
    p.chmod(p.stat().st_mode | stat.S_IEXEC)
    return str(p)


def test_sampler_keeps_only_samples_inside_the_region(fake_smi):
    with bench.ClockSampler("0", period_ms=20, exe=fake_smi) as clk:
        assert clk.samples, "the sampler waits for its first sample before the region starts"
        time.sleep(0.3)
    time.sleep(0.1)   # samples printed after the region are not counted
    s = clk.summary()
    inside = [t for t, _ in clk.samples if clk.t0 <= t <= clk.t1]
    assert s["samples"] == len(inside) >= 5
    assert len(clk.samples) > s["samples"]   # the first sample came before the region
    assert s["sm_max_mhz"] == 1965.0
    assert 1000 < s["sm_mhz"] < 1000 + len(clk.samples)
    assert s["reasons"] == ["sw_power_cap"]
    assert s["period_ms"] == 20


def test_sampler_without_the_tool_reports_no_samples(tmp_path):
    with bench.ClockSampler("0", exe=str(tmp_path / "missing-smi")) as clk:
        pass
    s = clk.summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None and s["reasons"] == []


def test_device_id_follows_cuda_visible_devices(monkeypatch):
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES", raising=False)
    assert bench.smi_device_id(0) == "0"
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "3, 5")
    assert bench.smi_device_id(0) == "3" and bench.smi_device_id(1) == "5"
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "GPU-8d1c2f3e-0000-1111-2222-333344445555")
    assert bench.smi_device_id(0) == "GPU-8d1c2f3e-0000-1111-2222-333344445555"


def _run_bench(*argv, env=None):
    import json
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    e = dict(os.environ, **(env or {}))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *argv], capture_output=True, text=True,
                       timeout=600, cwd=root, env=e)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    return [json.loads(ln) for ln in lines[-1:]]


def test_reference_arm_prints_the_contract_line():
    """The reference arm (the fp64 oracle on the host cores) prints one JSON line with
    the headline metric, unit and config of the library's own arm."""
    (line,) = _run_bench("--impl", "reference", "--steps", "1", "--warmup", "0")
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "modules/s" and line["value"] > 0
    assert line["higher_is_better"] is True and line["steps"] == 1 and line["warmup"] == 0
    assert line["config"] == bench.headline_config(bench.N_ADAPTERS, 1)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "modules/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    assert _run_bench("--impl", "reference", "--steps", "1", "--warmup", "0",
                      env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []


def test_traffic_record_is_dropped_once_the_kernel_source_changes(tmp_path, monkeypatch):
    import hashlib
    import json
    src = tmp_path / "k.cuh"
    src.write_text("kernel v1\n")
    (tmp_path / "profiles").mkdir()
    rec = {"leaf": {"bytes_per_unit": 1000.5, "source": "k.cuh",
                    "source_sha256": hashlib.sha256(src.read_bytes()).hexdigest()}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("leaf", 10) == 10005          # scaled by the units one launch processes
    assert bench.kernel_traffic("other", 10) is None
    src.write_text("kernel v2\n")                             # the kernel changed since the capture
    assert bench.kernel_traffic("leaf", 10) is None


def test_committed_traffic_records_name_their_captures():
    import json
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    recs = json.load(open(os.path.join(root, "profiles", "traffic.json")))
    for name, r in recs.items():
        assert os.path.exists(os.path.join(root, r["capture"])), name
        assert os.path.exists(os.path.join(root, r["source"])), name
        assert r["bytes_per_unit"] * r["units_captured"] == pytest.approx(r["dram_read"] + r["dram_write"])
