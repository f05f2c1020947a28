"""bench.py's own arm on a B200 prints the contract's JSON line: one line, the
contract's keys, the roofline / cpu_baseline / e2e / clocks objects, and a
launch count of this library's kernels.  Tiny workload, few steps."""
import json

import pytest

import bench

pytestmark = pytest.mark.gpu


def test_bench_json_line(capsys):
    rc = bench.main(["--config", "c1_tiny_dualscale", "--steps", "5", "--warmup", "3",
                     "--e2e-steps", "3", "--cpu-seconds", "1"])
    assert rc == 0
    lines = [ln for ln in capsys.readouterr().out.strip().splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for k in ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "cpu_baseline", "e2e", "clocks", "gpu_launches"]:
        assert k in j, k
    assert j["metric"] == bench.METRIC and j["n_gpus"] == 1 and j["steps"] == 5
    assert j["value"] > 0 and j["higher_is_better"] is True and j["scaling"] == "weak"
    rf = j["roofline"]
    assert rf["bound"] == "tensor" and rf["unit"] == "TOPS" and rf["peak"] > 0
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-3
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0 and cb["sample"]
    e = j["e2e"]
    assert e["value"] > 0 and e["unit"] == j["unit"]
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    ck = j["clocks"]
    assert isinstance(ck["reasons"], list) and ck["samples"] >= 0
    if ck["samples"]:
        assert ck["sm_max_mhz"] > 0 and ck["sm_mhz"] > 0
    # quantize + GEMM per layer and step
    assert j["gpu_launches"] == 2 * 5
