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


def test_ffn_pairs_found_in_the_ffn_configurations():
    from w8a8_gemm_b200 import workloads as wl
    pairs = {c: bench.ffn_pairs(wl.config_layers(c, seed=0)) for c in wl.CONFIGS}
    assert pairs["c4_sd35_ffn"] == [(0, 1)]
    assert pairs["c5_flux_block"] == [(3, 4)]
    assert pairs["c1_tiny_dualscale"] == [] and pairs["c2_sd35_adanorm"] == []
    assert pairs["c3_sd35_attn_out"] == []


def test_reference_arm_fused_producer(capsys, monkeypatch):
    """--fused-gelu: the oracle leg feeds fc2 with bf16(gelu(bf16(fc1 output)))."""
    monkeypatch.setattr(bench, "REF_BUDGET_S", 2.0)
    rc = bench.main(["--impl", "reference", "--config", "c4_sd35_ffn", "--fused-gelu",
                     "--steps", "1", "--warmup", "3"])
    assert rc == 0
    j = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert j["impl"] == "reference" and j["value"] > 0
    assert j["config"]["producer"].startswith("fused")


def test_fused_producer_rejects_configurations_without_ffn():
    import pytest
    with pytest.raises(SystemExit):
        bench.main(["--config", "c3_sd35_attn_out", "--fused-gelu"])
    with pytest.raises(SystemExit):
        bench.main(["--fused-gelu", "--fp8"])
