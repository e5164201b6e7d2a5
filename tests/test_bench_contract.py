"""The reference arm of bench.py on the CPU: one JSON line with the contract's keys.

The arm times the oracle on a bounded sample of the decode workload; here the
sample is tiny (0.2 % of each call's output columns, one step) so the check
runs in seconds.
"""
import contextlib
import io
import json
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_arm_json_line():
    out = io.StringIO()
    args = types.SimpleNamespace(steps=1, warmup=0, ref_fraction=0.002)
    with contextlib.redirect_stdout(out):
        assert bench.run_reference(args, 1, 0) == 0
    lines = [ln for ln in out.getvalue().splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["steps"] == 1 and d["n_gpus"] == 1 and d["data"] == "synthetic"
    assert d["config"] == bench.workload_config()
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
