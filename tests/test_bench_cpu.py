"""bench.py's host-side pieces on the CPU: the roofline denominators and their sources, the clock
record's parsing (median SM clock, maximum, throttle reasons), and the reference arm's JSON line
(the oracle on a bounded sample) with every key the contract asks for."""
import argparse
import io
import json
import os
from contextlib import redirect_stdout

import pytest

import bench


def test_peaks_measured_and_fallback():
    assert bench.int8_peak({"bf16_tflops": 1659.0})[0] == pytest.approx(3318.0)
    assert bench.int8_peak({"bf16_tflops": 1659.0})[1].startswith("of measured")
    assert bench.int8_peak({})[0] == pytest.approx(3180.0) and bench.int8_peak({})[1].startswith("of fallback")
    assert bench.bf16_peak({"bf16_tflops": 1659.0}) == (1659.0, "of measured: bf16 burst cuBLAS")
    assert bench.bf16_peak({})[0] == 1590.0
    assert bench.hbm_peak({"hbm_gbs": 6525.0})[0] == 6525.0 and bench.hbm_peak({})[0] == 6650.0


class _Done:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_record_parsing(tmp_path):
    c = bench.Clocks(0)
    c.path = str(tmp_path / "clocks.csv")
    rows = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1845, 1965, 999.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 950.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, [N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]",
        "garbage line",
    ]
    with open(c.path, "w") as fh:
        fh.write("\n".join(rows) + "\n")
    c.proc = _Done()
    rec = c.stop()
    assert rec["sm_mhz"] == 1965.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"] and rec["samples"] == 4
    assert not os.path.exists(c.path)
    # no sampler (nvidia-smi absent): no record rather than an error
    assert bench.Clocks(0).stop() is None


def test_reference_arm_prints_the_contract_line():
    args = argparse.Namespace(steps=1, warmup=0, gpus=1, workload="prefill-370M")
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(args, bench.WORKLOADS["prefill-370M"]) == 0
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert (line["n_gpus"], line["steps"], line["warmup"]) == (1, 1, 0)
    assert line["ms_per_step"] > 0 and "extrapolated" in line["ms_per_step_kind"]
    assert line["vs_baseline"] is None and line["data"] == "synthetic" and line["scaling"] == "weak"
    assert line["config"]["workload"] == "prefill-370M"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == "tokens/s"
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_do_no_work(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(steps=1, warmup=0, gpus=2, workload="prefill-370M")
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(args, bench.WORKLOADS["prefill-370M"]) == 0
    assert buf.getvalue() == ""


def test_an_extra_measurement_failure_is_reported_not_raised(capsys):
    assert bench.guarded(lambda a, b: a * b, 3, 4) == 12
    out = bench.guarded(lambda: [][1])
    assert out == {"error": "IndexError: list index out of range"}
    assert "IndexError" in capsys.readouterr().err
