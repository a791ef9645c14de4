"""Benchmark of Echo's compensated 4-bit all-reduce on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload large|llama|depth|tiny] [--fixup exit|side|deferred]
                    [--uncompensated] [--mode step|sweep|overlap|depth-chain|group|rank-stages]

Default (mode "step"): one step = one echo_allreduce call (entry kernel, then
the reduce kernel that also writes every rank's output) of P=8 virtual ranks
x 2^29 bf16 elements (1 GiB) per rank,
G=128, compensator on, inputs resident in HBM.  Prints ONE JSON line with
the input GB/s per call (all ranks' input bytes / call time), the whole-call
fraction of the HBM roofline (minimal bytes of a call / measured copy
bandwidth / call time), the roofline of the dominant kernel (echo_entry)
from CUDA events on its launch stream, the end-to-end figure through the
host-buffer C call (host<->device copies inside the timed region), the
oracle timed on host cores as the CPU baseline, and the SM clocks sampled
during the timed region.

With --gpus N under torchrun every rank runs its own independent call on
its own GPU (the path is emulated on one GPU; there is no cross-GPU data
exchange), timed between barriers and reported as the max over ranks.

--mode group runs the rank path instead: the N processes of the torchrun
form ONE Echo group (P = N real ranks, one GPU each, the workload's N
elements per rank), the two exchanges go over NCCL, and the line compares
the call with NCCL's bf16 all-reduce of the same tensors (max over ranks of
CUDA-event times).  With one GPU it runs a one-rank group.

--mode rank-stages times the rank path's three stage kernels for P ranks
emulated on one GPU (the fused transport inside one process, no NVLink).

--impl reference times the CPU oracle on bounded samples of the same
workload (rank 0 only) and prints the same JSON line with "impl":
"reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_error_compensated_echo_b200 import workloads as W  # noqa: E402

METRIC = "compensated 4-bit reduce input GB/s & % HBM roofline, P=8 virtual ranks, 1 GB/rank"
UNIT = "GB/s"
# fix-up placement timed by default (bit-identical to the others; fewest bytes)
BENCH_FIXUP = "deferred"
FALLBACK_HBM_GBS = 6650.0
# sources of the dominant kernel (echo_entry): an ncu traffic figure is
# reported only if it was captured from exactly these files
KERNEL_FILES = ("bit_error_compensated_echo_b200/csrc/echo_common.cuh",
                "bit_error_compensated_echo_b200/csrc/echo_entry.cuh")

WORKLOADS = {"large": W.LARGE, "llama": W.LLAMA, "depth": W.DEPTH, "tiny": W.TINY}


# ------------------------------------------------------------ byte counts

def transport_bytes_per_elem(G: int, bits: int = 4) -> float:
    """q: packed codes (bits/8 bytes) + fp32 scale per G elements."""
    return bits / 8.0 + 4.0 / G


def call_min_bytes(P: int, N: int, G: int, comp: bool, bits: int = 4) -> float:
    """Minimal HBM bytes of one call when each stage boundary is an HBM
    wire: read x, (read+write both states), write the P outputs, write and
    read the entry transport, write and read the reduced transport once,
    (write e_req and read it once)."""
    q = transport_bytes_per_elem(G, bits)
    if comp:
        return P * N * (2 + 16 + 2 + 2 * q) + N * (2 * q + 8)
    return P * N * (2 + 2 + 2 * q) + N * 2 * q


def rs_min_bytes(P: int, N: int, G: int, comp: bool, bits: int = 4) -> float:
    """Minimal HBM bytes of one reduce-scatter call: read x, (read+write both
    states), write and read the entry transport, write each owner's bf16
    chunk, (write e_req and read it once in the next entry)."""
    q = transport_bytes_per_elem(G, bits)
    if comp:
        return P * N * (2 + 16 + 2 * q) + N * (2 + 8)
    return P * N * (2 + 2 * q) + N * 2


def entry_bytes(P: int, N: int, G: int, comp: bool, fixup: str, bits: int = 4) -> float:
    """Algorithmic bytes of one echo_entry launch: read x (2 B), read and
    write both states (16 B), write codes + scales (q B) per rank-element;
    in deferred mode also read e_req of each rank's own chunk (4 B per
    element of N)."""
    q = transport_bytes_per_elem(G, bits)
    b = P * N * (2 + q)
    if comp:
        b += P * N * 16
        if fixup == "deferred":
            b += N * 4
    return b


def reduce_bytes(P: int, N: int, G: int, comp: bool, fixup: str, bits: int = 4) -> float:
    """Algorithmic bytes of one echo_reduce launch of the virtual plan: read
    the entry transport (P*q per element of N), write the reduced transport
    (q); uncompensated also the P bf16 outputs (2P); compensated, write
    e_req (4) or, with the fix-up in the kernel, read and write the owner's
    states (16)."""
    q = transport_bytes_per_elem(G, bits)
    b = P * N * q + N * q
    if comp:
        b += N * (16 if fixup == "exit" else 4)
    else:
        b += P * N * 2
    return b


def rs_kernel_bytes(P: int, N: int, G: int, comp: bool, fixup: str, bits: int = 4) -> float:
    """Algorithmic bytes of the reduce-scatter's second kernel (echo_rs): read
    the entry transport (P*q per element of N), write each owner's bf16
    chunk (2); compensated, write the owner residual (4) or, with the fix-up
    in the kernel, read and write the owner's states (16)."""
    b = P * N * transport_bytes_per_elem(G, bits) + 2 * N
    if comp:
        b += N * (16 if fixup == "exit" else 4)
    return b


def kernel_rooflines(prof: dict, P: int, N: int, G: int, comp: bool, fixup: str, bits: int,
                     peak: float, rs: bool = False) -> dict:
    """Each kernel's algorithmic bytes per launch over its average launch
    time (the plan's CUDA events on the launch stream), against the HBM peak.
    On one GPU the reduce writes the P outputs (there is no exit launch), so
    its bytes include them; for a reduce-scatter call the second kernel is
    echo_rs."""
    calls = max(int(prof["calls"]), 1)
    rb = reduce_bytes(P, N, G, comp, fixup, bits) + (P * N * 2 if comp else 0)
    kernels = [("echo_entry", entry_bytes(P, N, G, comp, fixup, bits), "entry_ms")]
    if rs:
        kernels.append(("echo_rs", rs_kernel_bytes(P, N, G, comp, fixup, bits), "reduce_ms"))
    else:
        kernels.append(("echo_reduce", rb, "reduce_ms"))
    out = {}
    for name, b, key in kernels:
        ms = prof[key] / calls
        if ms <= 0.0:
            continue
        gbs = b / (ms / 1e3) / 1e9
        out[name] = {"bytes": b, "avg_launch_ms": round(ms, 4), "achieved": round(gbs, 1),
                     "frac": round(gbs / peak, 4)}
    return out


# ------------------------------------------------------------ environment

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    """Hash of the dominant kernel's code with comments and whitespace
    removed, so that only a change of code invalidates an ncu capture."""
    import re
    h = hashlib.sha256()
    for rel in KERNEL_FILES:
        with open(os.path.join(ROOT, rel)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, comp: bool, fixup: str, bits: int = 4):
    """DRAM bytes per echo_entry launch from the committed ncu summary, if
    it was captured from the current kernel sources for this workload, mode
    and code width (else None)."""
    path = os.path.join(ROOT, "profiles", "echo_entry_traffic.md")
    if not os.path.exists(path):
        return None
    want = "%s comp=%d fixup=%s" % (workload, int(comp), fixup)
    src = kernel_source_hash()
    with open(path) as f:
        for line in f:
            if line.startswith("traffic:"):
                # traffic: <workload> comp=<0|1> fixup=<mode> [bits=<4|8>] src=<hash> bytes=<int>
                parts = line.split()
                key = " ".join(parts[1:4])
                kv = dict(p.split("=", 1) for p in parts[4:] if "=" in p)
                if key == want and kv.get("src") == src and kv.get("bits", "4") == str(bits):
                    return float(kv["bytes"])
    return None


class ClockSampler:
    """nvidia-smi SM clocks and throttle reasons, sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="echo_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [s.strip() for s in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------ distributed

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        from bit_error_compensated_echo_b200.rank import init_process_group
        init_process_group(timeout_s=120.0)
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, ws: int, device) -> float:
    if ws == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, ws: int, device) -> float:
    if ws == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(per_rank_ms, per_rank_bytes):
    """Whole-job throughput: bytes of all ranks / slowest rank's time."""
    t = max(per_rank_ms)
    return sum(per_rank_bytes) / (t / 1e3) / 1e9, t


# ------------------------------------------------------------ CPU baseline

def oracle_sample_run(w: W.Workload, comp: bool, ncols: int, x_dev=None, seed: int = 7,
                      bits: int = 4, op: str = "all-reduce", calls: int = 1, keep=None):
    """Time the oracle (as it stands, one host thread) on ``ncols`` group
    columns of workload ``w``: ``calls`` consecutive calls on the same inputs
    from zero state, as the benchmark's steps repeat the call on its resident
    inputs; inputs are the device inputs at those columns when given, else a
    host draw of the same distribution.  Returns (input GB/s, seconds,
    columns); a dict given as ``keep`` receives the element indices, the
    last call's outputs and the states after it."""
    import oracle
    cols = W.column_sample(w, ncols, seed=seed)
    idx = W.column_elements(cols, w.G)
    if x_dev is not None:
        ti = torch.from_numpy(idx).to(x_dev.device)
        xb = W.bf16_bits(x_dev.index_select(1, ti))
    else:
        small = W.with_size(w, rows=1, hidden=idx.size)
        xb = W.bf16_bits(W.generate(small, 0, "cpu"))
    prm = oracle.Params(P=w.P, N=w.N, G=w.G, compensate=comp, bits=bits)
    mf = np.zeros((w.P, idx.size), np.float32)
    ms = np.zeros_like(mf)
    call = oracle.reduce_scatter if op == "reduce-scatter" else oracle.allreduce
    t0 = time.perf_counter()
    for _ in range(calls):
        res = call(prm, xb, mf, ms, cols)
    dt = time.perf_counter() - t0
    if keep is not None:
        keep.update(idx=idx, y=res.y, m_fast=mf, m_slow=ms)
    del res
    nbytes = 2 * w.P * idx.size * calls
    return nbytes / dt / 1e9, dt, cols.size


def sampled_parity(plan, x, out, ref: dict, comp: bool, calls: int, side) -> dict:
    """The benchmark's own configuration against the oracle: after the
    timed region, the plan's state is reset and the oracle's calls (the same
    inputs, from zero state) are made again on the GPU; the outputs of the
    last call and the two states after it are compared, bit for bit, at the
    oracle's sampled group columns."""
    plan.reset_state()
    for _ in range(calls):
        plan.allreduce(x, out=out, side_stream=side)
    if x.is_cuda:
        torch.cuda.synchronize(x.device)
    ti = torch.from_numpy(ref["idx"]).to(x.device)
    y = out.index_select(1, ti).view(torch.int16).cpu().numpy().view(np.uint16)
    res = {"calls_from_zero_state": calls,
           "outputs_bit_exact": bool((y == ref["y"][None, :]).all())}
    if comp:
        states_equal = True
        for m_gpu, m_ref in zip(plan.get_state(), (ref["m_fast"], ref["m_slow"])):
            m = m_gpu.index_select(1, ti).view(torch.int32).cpu().numpy()
            states_equal &= bool(np.array_equal(m, m_ref.view(np.int32)))
            del m_gpu
        res["states_bit_exact"] = states_equal
    return res


def _oracle_part(job):
    """Worker of oracle_parallel_run: the oracle on one column range of the
    shared input sample; returns its own compute seconds."""
    from multiprocessing import shared_memory

    import oracle
    name, shape, prm_kw, c0, c1, G, cols = job
    shm = shared_memory.SharedMemory(name=name)
    try:
        xb = np.ndarray(shape, dtype=np.uint16, buffer=shm.buf)[:, c0 * G:c1 * G].copy()
    finally:
        shm.close()
    prm = oracle.Params(**prm_kw)
    mf = np.zeros(xb.shape, np.float32)
    ms = np.zeros_like(mf)
    t0 = time.perf_counter()
    oracle.allreduce(prm, xb, mf, ms, np.asarray(cols[c0:c1], np.int64))
    return time.perf_counter() - t0


def oracle_parallel_run(w: W.Workload, comp: bool, ncols: int, x_dev, bits: int = 4,
                        workers: int = 0, reps: int = 3):
    """The same oracle, as it stands, on the same column sample split over
    all host cores (processes started with spawn, inputs in shared memory):
    every quantity depends only on its group column, so the split is exact.
    Returns (GB/s, median wall seconds, workers)."""
    import multiprocessing as mp
    from multiprocessing import shared_memory
    workers = workers or len(os.sched_getaffinity(0))
    cols = W.column_sample(w, ncols, seed=7)
    idx = W.column_elements(cols, w.G)
    if x_dev is not None:
        ti = torch.from_numpy(idx).to(x_dev.device)
        xb = W.bf16_bits(x_dev.index_select(1, ti))
    else:   # a host draw of the same distribution, only the sampled columns
        xb = W.bf16_bits(W.generate(W.with_size(w, rows=1, hidden=idx.size), 0, "cpu"))
    shm = shared_memory.SharedMemory(create=True, size=xb.nbytes)
    try:
        np.ndarray(xb.shape, dtype=np.uint16, buffer=shm.buf)[:] = xb
        prm_kw = dict(P=w.P, N=w.N, G=w.G, compensate=comp, bits=bits)
        bounds = np.linspace(0, cols.size, workers + 1).astype(int)
        jobs = [(shm.name, xb.shape, prm_kw, int(bounds[i]), int(bounds[i + 1]), w.G, cols)
                for i in range(workers) if bounds[i + 1] > bounds[i]]
        times = []
        with mp.get_context("spawn").Pool(len(jobs)) as pool:
            pool.map(_oracle_part, jobs)                 # start-up and warm-up
            for _ in range(reps):
                t0 = time.perf_counter()
                pool.map(_oracle_part, jobs)
                times.append(time.perf_counter() - t0)
    finally:
        shm.close()
        shm.unlink()
    dt = statistics.median(times)
    return 2 * w.P * idx.size / dt / 1e9, dt, len(jobs)


# ------------------------------------------------------------ modes

def metric_of(comp: bool, rs: bool, bits: int) -> str:
    """The step line's metric for this mode (the headline one by default)."""
    metric = METRIC if comp else METRIC.replace("compensated", "uncompensated")
    if rs:
        metric = metric.replace("reduce input", "reduce-scatter input")
    if bits == 8:
        metric = metric.replace("4-bit", "8-bit")
    return metric


def dtypes_of(bits: int) -> dict:
    """The types the path moves and computes in (the line's dtype is the
    arithmetic one, f32)."""
    return {"inputs_outputs": "bf16", "transport": "int%d codes + f32 group scales" % bits,
            "sums_states_residuals": "f32"}


def step_config(args, w: W.Workload, comp: bool, fixup: str, ws: int) -> dict:
    """The workload of a step line, the same for both arms."""
    return {"workload": w.name, "op": args.op, "bits": args.bits, "P": w.P, "N_per_rank": w.N,
            "G": w.G, "compensate": comp, "fixup": fixup, "alpha": 0.5, "beta_fast": 0.5,
            "beta_slow": 0.95,
            "l2": "inputs larger than L2 (%.1f GiB of x per step)" % (2 * w.P * w.N / 2**30),
            "parallelism": "replicas" if ws > 1 else "1 GPU"}


def run_step_mode(args, ws, rank, local):
    from bit_error_compensated_echo_b200.api import EchoPlan

    dev = torch.device("cuda", local)
    w = WORKLOADS[args.workload]
    comp = not args.uncompensated
    fixup = args.fixup
    P, N, G = w.P, w.N, w.G
    peak, peak_kind = load_peaks()

    x = torch.empty((P, N), dtype=torch.bfloat16, device=dev)
    W.generate(w, rank, dev, out=x)
    out = torch.empty_like(x)
    plan = EchoPlan(P, N, G, compensate=comp, fixup=fixup, device=local, bits=args.bits)
    side = torch.cuda.Stream(device=dev) if fixup == "side" else None
    stream = torch.cuda.current_stream(dev)
    rs = args.op == "reduce-scatter"
    if rs:
        out = torch.empty((P, N // P), dtype=torch.bfloat16, device=dev)

    def one_call():
        if rs:
            plan.reduce_scatter(x, out=out, side_stream=side)
        else:
            plan.allreduce(x, out=out, side_stream=side)

    for _ in range(args.warmup):
        one_call()
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(local)
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    plan.profile_enable(True)
    plan.profile_read(reset=True)
    barrier(ws)
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        one_call()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(ws)
    prof = plan.profile_read(reset=True)
    plan.profile_enable(False)
    clk = clocks.stop() if rank == 0 else None
    ms_local = t0.elapsed_time(t1) / args.steps
    ms = max_over_ranks(ms_local, ws, dev)
    total_in = sum_over_ranks(2.0 * P * N, ws, dev)
    value = total_in / (ms / 1e3) / 1e9

    # end to end: host buffers through echo_allreduce_host
    e2e = None
    if not args.no_e2e and not rs:
        # one pinned buffer, outputs written over the inputs (the host call
        # allows it): 2 bytes per rank-element of host memory per process
        xh = torch.empty((P, N), dtype=torch.bfloat16, pin_memory=True)
        xh.copy_(x)
        yh = xh
        with EchoPlan(P, N, G, compensate=comp, fixup=fixup, device=local, bits=args.bits) as hp:
            for _ in range(args.warmup):
                hp.allreduce_host(xh, yh)
            torch.cuda.synchronize(dev)
            barrier(ws)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.e2e_steps):
                hp.allreduce_host(xh, yh)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            barrier(ws)
            e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, ws, dev)
        e2e = {"value": round(total_in / (e_ms / 1e3) / 1e9, 3), "unit": UNIT,
               "ms_per_step": round(e_ms, 3), "h2d_bytes_per_step": 2 * P * N,
               "d2h_bytes_per_step": 2 * P * N}
        del xh, yh

    cpu = cpu_par = parity = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        ref = {}
        gbs, dt, ncols = oracle_sample_run(w, comp, args.cpu_cols, x_dev=x, bits=args.bits,
                                           calls=args.cpu_calls, keep=ref)
        if not rs:
            parity = sampled_parity(plan, x, out, ref, comp, args.cpu_calls, side)
            parity["group_columns"] = ncols
        del ref
        cpu = {"value": round(gbs, 5), "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": "%d of %d group columns (x %d ranks x G=%d) of the same inputs, %d "
                         "consecutive calls from zero state, %.1f s on one host thread" %
                         (ncols, N // G, P, G, args.cpu_calls, dt)}
        if not args.no_cpu_parallel:
            pg, pdt, nw = oracle_parallel_run(w, comp, args.cpu_cols, x, bits=args.bits)
            cpu_par = {"value": round(pg, 5), "unit": UNIT, "cores": nw, "kind": "oracle",
                       "sample": "the same %d columns split over %d spawned processes (one "
                                 "per host core), median of 3 runs, %.2f s wall" %
                                 (ncols, nw, pdt)}

    if rank == 0:
        calls = prof["calls"]
        entry_ms = prof["entry_ms"] / max(calls, 1)
        eb = entry_bytes(P, N, G, comp, fixup, args.bits)
        achieved = eb / (entry_ms / 1e3) / 1e9
        bmin = (rs_min_bytes(P, N, G, comp, args.bits) if rs
                else call_min_bytes(P, N, G, comp, args.bits))
        traffic = ncu_traffic(w.name, comp, fixup, args.bits)
        metric = metric_of(comp, rs, args.bits)
        line = {
            "metric": metric,
            "value": round(value, 3), "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "dtypes": dtypes_of(args.bits),
            "data": "synthetic (seeded N(0,0.5^2) bf16 draws, no dataset)",
            "config": step_config(args, w, comp, fixup, ws),
            "call_roofline": {"min_bytes": bmin, "achieved_gbs": round(bmin / (ms / 1e3) / 1e9, 1),
                              "peak": peak, "frac": round(bmin / (ms / 1e3) / 1e9 / peak, 4),
                              "time_at_peak_ms": round(bmin / peak / 1e6, 3),
                              "frac_of_nominal_8tbs": round(bmin / (ms / 1e3) / 8e12, 4)},
            # NCCL's algorithm bandwidth: one rank's message over the call time
            "algbw_gbs": round(2.0 * N / (ms / 1e3) / 1e9, 3),
            "roofline": {"kernel": "echo_entry", "bound": "hbm", "achieved": round(achieved, 1),
                         "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "algorithmic_bytes": eb, "avg_launch_ms": round(entry_ms, 4)},
            "kernels_ms": {k: round(prof[k] / max(calls, 1), 4)
                           for k in ("entry_ms", "reduce_ms", "exit_ms", "fixup_ms")},
            "kernels_roofline": kernel_rooflines(prof, P, N, G, comp, fixup, args.bits, peak,
                                                 rs=rs),
            "gpu_launches": int(prof["launches"]),
            "e2e": e2e, "cpu_baseline": cpu, "cpu_baseline_all_cores": cpu_par,
            "host": host_info() if cpu else None, "parity": parity, "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    plan.close()


def run_reference(args, ws, rank):
    """The CPU oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    comp = not args.uncompensated
    for i in range(args.warmup):
        oracle_sample_run(w, comp, args.ref_cols, seed=100 + i, bits=args.bits, op=args.op)
    times, nbytes = [], 0
    for i in range(args.steps):
        gbs, dt, ncols = oracle_sample_run(w, comp, args.ref_cols, seed=1000 + i,
                                           bits=args.bits, op=args.op)
        times.append(dt)
        nbytes = 2 * w.P * ncols * w.G
    ms = 1e3 * sum(times) / len(times)
    value = nbytes / (ms / 1e3) / 1e9
    sample = ("%d of %d group columns (x %d ranks x G=%d) per step, host draw of the same "
              "distribution, one call from zero state" % (args.ref_cols + 2, w.N // w.G, w.P, w.G))
    line = {
        "metric": metric_of(comp, args.op == "reduce-scatter", args.bits),
        "value": round(value, 6), "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "dtypes": dtypes_of(args.bits),
        "data": "synthetic", "impl": "reference",
        "config": step_config(args, w, comp, args.fixup, ws),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "host": host_info(),
    }
    print(json.dumps(line), flush=True)


def _time_calls(fn, steps, flush, stream):
    """Median device time of fn() over steps launches, L2 flushed between."""
    times = []
    for k in range(steps):
        flush.fill_(float(k))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def run_sweep_mode(args, ws, rank, local):
    """Sizes 1 MiB..1 GiB per rank x P in {2,4,8} x G in {32,64,128} x
    compensated / off: GB/s, fraction of the call roofline, packed ratio;
    eager and CUDA-graph-captured times, L2 flushed between timed calls."""
    from bit_error_compensated_echo_b200.api import EchoPlan
    if rank != 0:
        return
    dev = torch.device("cuda", local)
    peak, peak_kind = load_peaks()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    rows = []
    copy_rate = {}   # (P, N) -> bytes/s of a plain device copy of the same tensors
    points = W.sweep()
    if args.sweep_max_mib:
        points = [w for w in points if w.N * 2 <= args.sweep_max_mib << 20]
    for w in points:
        x = W.generate(w, 0, dev)
        out = torch.empty_like(x)
        plan = EchoPlan(w.P, w.N, w.G, compensate=w.compensate, fixup=BENCH_FIXUP, device=local)
        for _ in range(max(args.warmup, 3)):
            plan.allreduce(x, out=out)
        torch.cuda.synchronize()
        t_eager = _time_calls(lambda: plan.allreduce(x, out=out), args.steps, flush, stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            plan.allreduce(x, out=out)
        g.replay()
        torch.cuda.synchronize()
        t_graph = _time_calls(g.replay, args.steps, flush, stream)
        del g
        if (w.P, w.N) not in copy_rate:
            # calibration only (not the path): the rate a plain copy of the
            # inputs into the outputs reaches at this size, timed the same way
            for _ in range(3):
                out.copy_(x)
            t_copy = _time_calls(lambda: out.copy_(x), args.steps, flush, stream)
            copy_rate[(w.P, w.N)] = 4 * w.P * w.N / (t_copy / 1e3)
        bmin = call_min_bytes(w.P, w.N, w.G, w.compensate)
        q = transport_bytes_per_elem(w.G)
        row = {"mode": "sweep", "point": w.name, "MiB_per_rank": w.N * 2 // (1 << 20), "P": w.P,
               "G": w.G, "compensate": w.compensate, "ms_eager": round(t_eager, 4),
               "ms_graph": round(t_graph, 4),
               "input_gbs": round(2 * w.P * w.N / (min(t_eager, t_graph) / 1e3) / 1e9, 2),
               "roofline_frac": round(bmin / peak / (min(t_eager, t_graph) / 1e3) / 1e9, 4),
               "min_bytes": bmin, "packed_ratio": q / 2,
               "copy_gbs": round(copy_rate[(w.P, w.N)] / 1e9, 1),
               "frac_of_copy": round(bmin / (min(t_eager, t_graph) / 1e3) / copy_rate[(w.P, w.N)], 4)}
        dv = plan.debug_view()
        row["packed_ratio_allocated"] = (dv["codes"].numel() + 4 * dv["scales"].numel()) / (2.0 * w.P * w.N)
        rows.append(row)
        print(json.dumps(row), flush=True)
        plan.close()
        del x, out, plan
        torch.cuda.empty_cache()
    if args.sweep_table:
        with open(args.sweep_table, "w") as f:
            f.write("| MiB/rank | P | G | mode | ms eager | ms graph | input GB/s | % of call roofline "
                    "| same-size copy GB/s | % of same-size copy | packed/bf16 |\n")
            f.write("|---|---|---|---|---|---|---|---|---|---|---|\n")
            for r in rows:
                f.write("| %d | %d | %d | %s | %.4f | %.4f | %.1f | %.1f | %.1f | %.1f | %.6f |\n" % (
                    r["MiB_per_rank"], r["P"], r["G"], "comp" if r["compensate"] else "off",
                    r["ms_eager"], r["ms_graph"], r["input_gbs"], 100 * r["roofline_frac"],
                    r["copy_gbs"], 100 * r["frac_of_copy"], r["packed_ratio"]))


def run_rank_stages_mode(args, ws, rank, local):
    """The rank path's stage kernels for the workload's P ranks on this one
    GPU: P rank plans in one process whose entries store into each other's
    windows and whose exits load from them (PeerWindows.in_process, the
    fused transport without NVLink), stage by stage, so no kernel waits on
    another.  Per step: echo_rank_entry_peers of every rank, echo_rank_reduce
    of every owner, echo_rank_exit_peers of every rank, CUDA events between
    the stages.  Prints the stages' times (all ranks' work per call) and
    their algorithmic bytes over time against the measured copy rate."""
    from bit_error_compensated_echo_b200.rank import EchoRankPlan, PeerWindows
    if rank != 0:
        return
    dev = torch.device("cuda", local)
    w = WORKLOADS[args.workload]
    P, N, G, bits = w.P, w.N, w.G, args.bits
    comp = not args.uncompensated
    peak, peak_kind = load_peaks()
    x = W.generate(w, 0, dev)
    out = torch.empty_like(x)
    plans = [EchoRankPlan(P, r, N, G, compensate=comp, fixup=args.fixup, device=local, bits=bits)
             for r in range(P)]
    try:
        wins = PeerWindows.in_process(plans)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]

        def step():
            ev[0].record()
            for r, (p, win) in enumerate(zip(plans, wins)):
                p.entry_peers(x[r], win)
            ev[1].record()
            for p, win in zip(plans, wins):
                p.reduce_window(win)
            ev[2].record()
            for r, (p, win) in enumerate(zip(plans, wins)):
                p.exit_peers(win, out[r])
            ev[3].record()

        for _ in range(max(args.warmup, 3)):
            step()
        torch.cuda.synchronize()
        tot = [0.0, 0.0, 0.0]
        for _ in range(args.steps):
            step()
            torch.cuda.synchronize()
            for i in range(3):
                tot[i] += ev[i].elapsed_time(ev[i + 1])
        t = [v / args.steps for v in tot]
        q = transport_bytes_per_elem(G, bits)
        stage_bytes = {
            "entry_peers": entry_bytes(P, N, G, comp, args.fixup, bits),
            # the owner reads P received chunks and writes its reduced chunk, no outputs
            "reduce": N * (P * q + q) + (N * (16 if args.fixup == "exit" else 4) if comp else 0),
            # every rank reads every owner's reduced chunk and writes its own output
            "exit_peers": P * N * (q + 2),
        }
        stages = {}
        for (name, b), ms in zip(stage_bytes.items(), t):
            gbs = b / (ms / 1e3) / 1e9
            stages[name] = {"ms": round(ms, 4), "bytes": b, "achieved_gbs": round(gbs, 1),
                            "frac": round(gbs / peak, 4)}
        print(json.dumps({"mode": "rank-stages", "workload": w.name, "P": P, "N_per_rank": N,
                          "G": G, "bits": bits, "compensate": comp, "fixup": args.fixup,
                          "steps": args.steps, "stages_all_ranks": stages,
                          "call_ms_all_ranks": round(sum(t), 4), "peak_gbs": peak,
                          "peak_kind": peak_kind,
                          "note": "P ranks' plans on one GPU, fused transport in one process "
                                  "(no NVLink); each stage timed over all ranks"}), flush=True)
    finally:
        for p in plans:
            p.close()


def run_overlap_mode(args, ws, rank, local):
    """1 GiB per rank, P=8: the stand-in next matmul (bf16 8192^3) after each
    call, with the owner fix-up in the reduce kernel, on a side stream beside
    the matmul, or deferred; plus the fused compensation cost (compensated
    minus uncompensated call) and the compensator written as separate torch
    operations, for context."""
    from bit_error_compensated_echo_b200.api import EchoPlan
    if rank != 0:
        return
    dev = torch.device("cuda", local)
    w = W.LARGE
    x = torch.empty((w.P, w.N), dtype=torch.bfloat16, device=dev)
    W.generate(w, 0, dev, out=x)
    out = torch.empty_like(x)
    ga = torch.randn((8192, 8192), device=dev).to(torch.bfloat16)
    gb = torch.randn((8192, 8192), device=dev).to(torch.bfloat16)
    gc = torch.empty((8192, 8192), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(device=dev)

    def timed(fn, steps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    res = {"mode": "overlap", "workload": w.name, "gemm": "bf16 8192x8192x8192 torch.matmul"}
    res["gemm_ms"] = round(timed(lambda: torch.matmul(ga, gb, out=gc), args.steps), 4)
    for comp, fixup in ((False, "exit"), (True, "exit"), (True, "side"), (True, "deferred")):
        plan = EchoPlan(w.P, w.N, w.G, compensate=comp, fixup=fixup, device=local)
        key = ("comp_" + fixup) if comp else "off"
        res["call_ms_" + key] = round(timed(lambda: plan.allreduce(x, out=out, side_stream=side),
                                            args.steps), 4)

        def step():
            plan.allreduce(x, out=out, side_stream=side)
            torch.matmul(ga, gb, out=gc)
        res["call_plus_gemm_ms_" + key] = round(timed(step, args.steps), 4)
        plan.close()
    res["fused_compensation_ms"] = round(res["call_ms_comp_deferred"] - res["call_ms_off"], 4)

    # the compensator as separate torch ops (correction, quantize-dequantize
    # for the entry error, both EMA updates), rank by rank
    mf = torch.zeros((w.N,), dtype=torch.float32, device=dev)
    ms = torch.zeros_like(mf)

    def torch_compensator():
        for r in range(w.P):
            c = 0.5 * mf + 0.5 * ms
            xt = x[r].float() + c
            g = xt.view(-1, w.G)
            scale = g.abs().amax(dim=1, keepdim=True) / 7.0
            k = torch.where(scale > 0, torch.round(g / scale), torch.zeros_like(g)).clamp_(-7, 7)
            e = (g - k * scale).view(-1)
            mf.mul_(0.5).add_(0.5 * e)
            ms.mul_(0.95).add_(0.05 * e)
    res["torch_ops_compensator_ms"] = round(timed(torch_compensator, max(2, args.steps // 3)), 3)
    res["note"] = ("call_plus_gemm = one all-reduce followed by the matmul on the same stream; "
                   "side = owner fix-up on a second stream beside the matmul")
    print(json.dumps(res), flush=True)


def run_group_mode(args, ws, rank, local):
    """The rank path over NCCL: this process is rank ``rank`` of a group of
    ws ranks; per step one EchoRankPlan.allreduce (entry, all-to-all of the
    packed chunks, reduce, all-gather, exit), timed with CUDA events between
    barriers, max over ranks; then the same call over the fused transport
    (allreduce_peers: the entry stores into the owners' windows, the exit
    loads from them, two one-element NCCL all-reduces as barriers), and
    NCCL's bf16 all-reduce of the same input, timed the same way."""
    import torch.distributed as dist

    from bit_error_compensated_echo_b200.rank import (EchoRankPlan, PeerWindows,
                                                      TorchDistBarrier, TorchDistTransport,
                                                      init_process_group)
    if ws == 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", str(29500 + (os.getpid() % 1000)))
        init_process_group("nccl", timeout_s=120.0, rank=0, world_size=1)
    dev = torch.device("cuda", local)
    w = WORKLOADS[args.workload]
    comp = not args.uncompensated
    P, N, G = ws, w.N, w.G
    if N % (P * G):
        raise SystemExit("N=%d is not a multiple of P*G=%d" % (N, P * G))
    one = W.with_size(w, P=1)
    x = W.generate(one, rank, dev)[0].contiguous()
    out = torch.empty_like(x)
    plan = EchoRankPlan(P, rank, N, G, compensate=comp, fixup=args.fixup, device=local,
                        bits=args.bits)
    transport = TorchDistTransport()
    stream = torch.cuda.current_stream(dev)

    def timed(fn, steps):
        times = []
        for _ in range(steps):
            dist.barrier()
            torch.cuda.synchronize(dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            times.append(e0.elapsed_time(e1))
        return times

    echo_fn = lambda: plan.allreduce(x, transport, out=out)  # noqa: E731
    win = PeerWindows.exchange(plan)
    barrier = TorchDistBarrier(dev)
    peers_fn = lambda: plan.allreduce_peers(x, win, barrier, out=out)  # noqa: E731
    y = x.clone()
    nccl_fn = lambda: dist.all_reduce(y)  # noqa: E731
    timed(echo_fn, max(args.warmup, 3))
    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
    t_echo = timed(echo_fn, args.steps)
    clocks = sampler.stop() if sampler else None
    timed(peers_fn, max(args.warmup, 3))
    t_peers = timed(peers_fn, args.steps)
    timed(nccl_fn, max(args.warmup, 3))
    t_nccl = timed(nccl_fn, args.steps)
    ms_echo = max_over_ranks(statistics.median(t_echo), ws, dev)
    ms_peers = max_over_ranks(statistics.median(t_peers), ws, dev)
    ms_nccl = max_over_ranks(statistics.median(t_nccl), ws, dev)
    # no rank unmaps, and no owner frees, a window a peer may still read
    torch.cuda.synchronize(dev)
    dist.barrier()
    win.close()
    dist.barrier()
    wire = plan.bufs.wire_bytes()
    if rank == 0:
        line = {
            "mode": "group", "metric": "Echo all-reduce over NCCL: input GB/s (P ranks x N bf16 "
            "/ call time), against NCCL's bf16 all-reduce", "unit": UNIT,
            "value": round(2.0 * P * N / (ms_echo / 1e3) / 1e9, 3), "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_call": round(ms_echo, 4),
            "nccl_bf16_allreduce_ms": round(ms_nccl, 4),
            "speedup_vs_nccl_bf16": round(ms_nccl / ms_echo, 3),
            "wire_bytes_per_rank": wire, "bf16_ring_wire_bytes_per_rank": 2 * (P - 1) * N * 2 // P,
            "higher_is_better": True, "scaling": "weak", "data": "synthetic",
            "config": {"workload": w.name, "P": P, "N_per_rank": N, "G": G, "bits": args.bits,
                       "compensate": comp, "fixup": args.fixup,
                       "transport": "torch.distributed NCCL all_to_all_single + "
                       "all_gather_into_tensor"},
            "gpu_launches_per_call": plan.launches_per_call(), "clocks": clocks,
            "fused_transport": {
                "ms_per_call": round(ms_peers, 4),
                "value": round(2.0 * P * N / (ms_peers / 1e3) / 1e9, 3),
                "speedup_vs_nccl_bf16": round(ms_nccl / ms_peers, 3),
                "transport": "entry stores into the owners' windows, exit loads from them "
                "(CUDA IPC), two one-element NCCL all-reduces as barriers"},
        }
        print(json.dumps(line), flush=True)
    plan.close()
    if ws == 1:
        dist.destroy_process_group()


def host_info() -> dict:
    """The host the CPU legs ran on: CPU model and logical CPUs."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "logical_cpus": os.cpu_count()}


def run_cpu_mode(args, ws, rank, local):
    """The oracle, as it stands, on the host cores for each configuration:
    one call (the tiny workload whole, the others on a sample of group
    columns), on one thread and split by group columns over all cores.
    Prints one JSON line per configuration."""
    if rank != 0:
        return
    cases = [(W.TINY, None), (W.LLAMA, 65536), (W.DEPTH, 65536), (W.LARGE, 262144)]
    for w, ncols in cases:
        # the tiny workload whole; the others: only the sampled columns are drawn
        x = W.generate(w, 0, "cpu") if ncols is None else None
        n = ncols - 2 if ncols else w.N // w.G
        gbs1, dt1, c1 = oracle_sample_run(w, True, n, x_dev=x)
        gbs_all, dt_all, nw = oracle_parallel_run(w, True, n, x, reps=3)
        elems = w.P * c1 * w.G
        print(json.dumps({
            "mode": "cpu", "workload": w.name, "kind": "oracle", "host": host_info(),
            "group_columns": c1,
            "of_columns": w.N // w.G, "rank_elements": elems,
            "one_thread": {"seconds": round(dt1, 4), "ns_per_rank_element": round(dt1 / elems * 1e9, 2),
                           "input_gbs": round(gbs1, 5)},
            "all_cores": {"cores": nw, "seconds": round(dt_all, 4),
                          "ns_per_rank_element": round(dt_all / elems * 1e9, 3),
                          "input_gbs": round(gbs_all, 5)}}), flush=True)
        del x


def run_depth_chain_mode(args, ws, rank, local):
    """Deviation from the exact fp32 chain per site, forward and backward."""
    from bit_error_compensated_echo_b200 import depth_chain
    if rank != 0:
        return
    t0 = time.perf_counter()
    res = depth_chain.run(P=8, tokens=W.DEPTH.rows, hidden=W.DEPTH.hidden, sites=W.DEPTH.calls,
                          G=W.DEPTH.G, seed=W.DEPTH.seed, device="cuda:%d" % local)
    line = {"mode": "depth-chain", "workload": W.DEPTH.name,
            "seconds": round(time.perf_counter() - t0, 1),
            "note": "RMS deviation from the exact fp32 chain after each site (and relative "
                    "Frobenius deviation), compensated / uncompensated 4-bit / bf16 all-reduce"}
    for k, v in res.items():
        line[k] = {c: [float("%.4g" % x) for x in arr] for c, arr in v.items()}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="large")
    ap.add_argument("--fixup", choices=("exit", "side", "deferred"), default=BENCH_FIXUP)
    ap.add_argument("--uncompensated", action="store_true")
    ap.add_argument("--op", choices=("all-reduce", "reduce-scatter"), default="all-reduce")
    ap.add_argument("--bits", type=int, choices=(4, 8), default=4)
    ap.add_argument("--mode", choices=("step", "depth-chain", "sweep", "overlap", "group",
                                       "rank-stages", "cpu"),
                    default="step")
    ap.add_argument("--sweep-max-mib", type=int, default=0,
                    help="sweep only points up to this many MiB per rank (0: all)")
    ap.add_argument("--sweep-table", default="", help="also write the sweep as a markdown table")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-cpu-parallel", action="store_true",
                    help="skip the all-cores run of the oracle beside the CPU baseline")
    ap.add_argument("--cpu-cols", type=int, default=655360,
                    help="group columns of the CPU-baseline sample")
    ap.add_argument("--cpu-calls", type=int, default=2,
                    help="consecutive oracle calls on that sample (about 7-8 s each on one "
                         "core of the GPU hosts)")
    ap.add_argument("--ref-cols", type=int, default=131072,
                    help="group columns per step of the reference arm")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)

    ws, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, ws, rank)
        elif args.mode == "depth-chain":
            run_depth_chain_mode(args, ws, rank, local)
        elif args.mode == "sweep":
            run_sweep_mode(args, ws, rank, local)
        elif args.mode == "overlap":
            run_overlap_mode(args, ws, rank, local)
        elif args.mode == "group":
            run_group_mode(args, ws, rank, local)
        elif args.mode == "rank-stages":
            run_rank_stages_mode(args, ws, rank, local)
        elif args.mode == "cpu":
            run_cpu_mode(args, ws, rank, local)
        else:
            run_step_mode(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
