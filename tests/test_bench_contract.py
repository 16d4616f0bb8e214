"""The benchmark's reference arm (the float64 oracle timed on the host cores) prints the
JSON line the benchmark contract asks for.  Run on the tiny geometry so that it takes
seconds; the r2 / r3 workloads differ only in sizes."""
import argparse
import json
import os
import sys

import kva_inputs as KI

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setattr(bench, "geometry", lambda name: KI.TINY)
    args = argparse.Namespace(workload="r3", steps=2, warmup=1)
    bench.run_reference(args, 0, 1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 2
    assert line["higher_is_better"] is True and line["dtype"] == "f64"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_is_silent_on_other_ranks(capsys):
    sys.path.insert(0, ROOT)
    import bench
    bench.run_reference(argparse.Namespace(workload="r3", steps=1, warmup=0), 1, 2)
    assert capsys.readouterr().out == ""
