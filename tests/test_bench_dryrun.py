"""bench.py's control flow without a GPU (tests/bench_fakes.py replaces the
device and the library calls): exactly K frames are timed whatever K is, the
launch count and the timing labels follow, and the JSON line carries the
contract's keys.  The numbers in these lines mean nothing."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "roofline", "clocks", "gpu_launches")


def run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "bench_fakes.py"), *args, "--no-e2e",
                          "--no-cpu-baseline"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    calls = [int(l.split()[1]) for l in out.stdout.splitlines() if l.startswith("CALLS")]
    assert len(lines) == 1 and len(calls) == 1
    return json.loads(lines[0]), calls[0]


@pytest.mark.parametrize("steps,graphs", [(40, True), (47, True), (7, True), (5, False)])
def test_layer_bench_times_exactly_k_frames(steps, graphs):
    warmup = 3
    args = ["--steps", str(steps), "--warmup", str(warmup)] + ([] if graphs else ["--no-graphs"])
    j, calls = run(*args)
    for k in KEYS:
        assert k in j, k
    assert j["steps"] == steps and j["warmup"] == warmup
    assert j["gpu_launches"] == 6 * steps  # 5 attention launches + 1 state write per frame
    n_rep, n_tail = divmod(steps, 20) if graphs else (0, steps)
    # layer calls executed: warm-up frames, one untimed replay of each of the two
    # graphs, then the timed replays and eager frames (5 calls per frame)
    assert calls == 5 * (warmup + (2 * 20 if n_rep else 0) + n_rep * 20 + n_tail)
    assert j["config"]["workload"] == "single-hybrid-layer-bf16"
    timing = j["config"]["timing"]
    assert (f"{n_rep} replays" in timing) == bool(n_rep) and (f"{n_tail} eager" in timing) == bool(n_tail)
    rf = j["roofline"]
    assert rf["kernel"] == "attn_pair_kernel" and rf["unit"] == "TFLOP/s" and "span / 4" in rf["duration_basis"]


def test_block_bench_covers_the_pool_and_times_exactly_k_frames():
    j, calls = run("--block", "--steps", "19", "--warmup", "3")
    assert j["steps"] == 19
    # graphs of 8 frames (the 40-matrix pool): warm-up 3, one untimed replay,
    # 2 timed replays and 3 eager frames, 5 calls per frame
    assert calls == 5 * (3 + 8 + 2 * 8 + 3)


@pytest.mark.parametrize("args,calls_expected", [
    (("--config", "3", "--steps", "2", "--warmup", "1"), 3 * 5 * 30),   # warm-up frame + 2 frames, 30 layers
    (("--token", "--steps", "3", "--warmup", "1"), None),
    (("--profile-kv", "2", "--steps", "1", "--warmup", "1"), None),
])
def test_other_bench_lines_run(args, calls_expected):
    j, calls = run(*args)
    for k in ("metric", "value", "unit", "n_gpus", "higher_is_better", "dtype", "data", "config"):
        assert k in j, k
    if calls_expected is not None:
        assert calls == calls_expected
