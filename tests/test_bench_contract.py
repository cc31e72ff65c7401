"""The benchmark's reference arm (the oracle timed on the host's cores) runs
without a GPU and prints one JSON line with the fields the contract asks for."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["value"] > 0 and j["unit"] == "frames/s"
    assert j["config"]["workload"] == "single-hybrid-layer-bf16"
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == j["value"] and cb["sample"]
    assert j["e2e"] == {"value": j["value"], "unit": "frames/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_bench_accounting_helpers():
    """The launch count and the traffic figure the bench line carries: one
    state-write launch while a frame's chunks fit one cluster, three beyond;
    traffic only for the workload the capture was taken on."""
    sys.path.insert(0, ROOT)
    import bench
    from hybrid_linear_attention_arl2_b200 import workloads as W
    cfg1 = W.CONFIGS[1]
    assert bench.state_launches(cfg1) == 1  # 1560 tokens: 13 chunks of 128
    long = W.Config(99, "long", 1, 12, 128, 16 * 128 + 1, 1, 1, "bf16")
    assert bench.state_launches(long) == 3
    t = bench.attn_traffic(cfg1.name)
    assert t is None or t == bench.ATTN_TRAFFIC["bytes"]
    assert bench.attn_traffic(W.CONFIGS[4].name) is None
