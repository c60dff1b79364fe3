"""The bench's JSON line (CPU: the reference arm, which times the fp64 oracle on the host)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "dual_f32_B1H2T256_d32C16", "--steps", "2",
                          "--warmup", "1"], capture_output=True, text=True, timeout=300,
                         cwd=ROOT, check=True).stdout.strip().splitlines()
    lines = [ln for ln in out if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True and d["n_gpus"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    # the same workload description as the measured arm prints
    sys.path.insert(0, ROOT)
    import bench
    from weight_linear_attention_ttt_b200 import inputs as inp

    assert d["config"] == bench.config_of(inp.WORKLOADS["dual_f32_B1H2T256_d32C16"], 1)
    assert d["metric"] == bench.metric_of(inp.WORKLOADS["dual_f32_B1H2T256_d32C16"])
