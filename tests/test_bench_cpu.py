"""bench.py's host-side legs on a machine without a GPU: the reference arm
(the oracle on host cores) prints the JSON line the benchmark contract asks
for, and the parity verdict of the benchmark line compares the right
elements."""
import json
import os
import subprocess
import sys

import numpy as np
import torch

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


class _OraclePlan:
    """A stand-in plan for bench.sampled_parity on the CPU: every call is
    the oracle on all group columns; `flip` plants one wrong bit in the
    outputs or a state at a sampled element."""

    def __init__(self, w, flip=None):
        import oracle
        self.oracle, self.w, self.flip = oracle, w, flip
        self.prm = oracle.Params(P=w.P, N=w.N, G=w.G, compensate=True)
        self.reset_state()

    def reset_state(self):
        self.mf = np.zeros((self.w.P, self.w.N), np.float32)
        self.ms = np.zeros_like(self.mf)

    def allreduce(self, x, out=None, side_stream=None):
        from bit_error_compensated_echo_b200 import workloads as W
        r = self.oracle.allreduce(self.prm, W.bf16_bits(x), self.mf, self.ms)
        y = torch.from_numpy(np.broadcast_to(r.y, (self.w.P, self.w.N)).copy().view(np.int16))
        out.copy_(y.view(torch.bfloat16))
        if self.flip and self.flip[0] == "y":
            out.view(torch.int16)[0, self.flip[1]] ^= 1
        return out

    def get_state(self):
        mf, ms = torch.from_numpy(self.mf.copy()), torch.from_numpy(self.ms.copy())
        if self.flip and self.flip[0] == "m":
            ms.view(torch.int32)[1, self.flip[1]] ^= 1
        return mf, ms


def test_sampled_parity_verdict():
    """bench.sampled_parity compares the right elements: it passes for
    calls that equal the oracle and fails on one planted bit at a sampled
    element, in the outputs or in a state."""
    import bench
    from bit_error_compensated_echo_b200 import workloads as W
    w = W.TINY
    x = W.generate(w, 0, "cpu")
    out = torch.empty_like(x)
    ref = {}
    bench.oracle_sample_run(w, True, 40, x_dev=x, calls=2, keep=ref)
    e = int(ref["idx"][len(ref["idx"]) // 2])          # a sampled element
    good = bench.sampled_parity(_OraclePlan(w), x, out, ref, True, 2, None)
    assert good["outputs_bit_exact"] and good["states_bit_exact"]
    bad_y = bench.sampled_parity(_OraclePlan(w, ("y", e)), x, out, ref, True, 2, None)
    assert not bad_y["outputs_bit_exact"] and bad_y["states_bit_exact"]
    bad_m = bench.sampled_parity(_OraclePlan(w, ("m", e)), x, out, ref, True, 2, None)
    assert bad_m["outputs_bit_exact"] and not bad_m["states_bit_exact"]
