"""The benchmark's reference arm (the CPU oracle on the host cores) prints the
contract's JSON line: one line, every key it names, with consistent values.
Run on the tiny workload with a short CPU budget."""
import json

import bench

KEYS = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
        "cpu_baseline", "e2e"]


def test_reference_arm_json_line(capsys, monkeypatch):
    monkeypatch.setattr(bench, "REF_BUDGET_S", 2.0)
    rc = bench.main(["--impl", "reference", "--config", "c1_tiny_dualscale", "--steps", "1",
                     "--warmup", "3"])
    assert rc == 0
    lines = capsys.readouterr().out.strip().splitlines()
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert all(k in j for k in KEYS)
    assert j["impl"] == "reference" and j["metric"] == bench.METRIC and j["unit"] == "TOPS"
    assert j["steps"] == 1 and j["warmup"] == 3 and j["n_gpus"] == 1
    assert j["higher_is_better"] is True and j["value"] > 0 and j["ms_per_step"] > 0
    assert j["config"]["workload"].startswith("c1_tiny_dualscale")
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == j["value"]
    assert cb["unit"] == j["unit"] and cb["sample"]
    e = j["e2e"]
    assert e["value"] == j["value"] and e["unit"] == j["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0
