"""bench.py's reference arm (the oracle on host cores) runs on a machine
without a GPU and prints the JSON line the benchmark contract asks for."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
         "--warmup", "1", "--ref-cols", "64"],
        capture_output=True, text=True, timeout=600, cwd=ROOT, check=True).stdout
    lines = [ln for ln in out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "large_p8_1gib_g128"


def test_oracle_all_cores_run_on_cpu():
    """The all-cores CPU baseline: the oracle over column ranges in spawned
    processes, inputs in shared memory (here 2 workers, tiny workload)."""
    import bench
    from bit_error_compensated_echo_b200 import workloads as W
    x = W.generate(W.TINY, 0, "cpu")
    gbs, dt, nw = bench.oracle_parallel_run(W.TINY, True, 64, x, workers=2, reps=1)
    assert nw == 2 and gbs > 0 and dt > 0
