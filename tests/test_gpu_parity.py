"""CUDA path vs the CPU oracle, call by call, through the C ABI.

Covers the tiny correctness workload in full (16 calls, compensator on and
off, every fix-up mode), shapes spanning several thread blocks with ragged
tails for every P and G, the edge cases (zero, grid-exact, extreme and
subnormal inputs, in-place calls, P = 1), and the full-size Llama-shaped
and 1 GiB-per-rank workloads on sampled group columns.
"""
import numpy as np
import pytest
import torch

import oracle
import oracle_pins
from bit_error_compensated_echo_b200 import workloads as W
from bit_error_compensated_echo_b200.api import EchoPlan
from parity import SequenceChecker, oracle_params

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _plan(P, N, G, comp=True, fixup="exit", **kw):
    return EchoPlan(P, N, G, compensate=comp, fixup=fixup, device=0, **kw)


@pytest.mark.parametrize("comp", [True, False], ids=["comp", "off"])
@pytest.mark.parametrize("fixup", ["exit", "side", "deferred"])
def test_tiny_sequence_full(comp, fixup):
    """P=2, N=4096, G=32, N(0,1) from seed 0, 16 calls, every element."""
    w = W.TINY
    if not comp and fixup != "exit":
        pytest.skip("fix-up mode is irrelevant without the compensator")
    with _plan(w.P, w.N, w.G, comp, fixup) as plan:
        chk = SequenceChecker(plan, oracle_params(plan))
        side = torch.cuda.Stream() if fixup == "side" else None
        for t in range(w.calls):
            x = W.generate(w, t, DEV)
            chk.step(x, side_stream=side)


RAGGED = [(1, 32, 37), (2, 64, 75), (3, 128, 41), (4, 32, 513), (5, 64, 29),
          (6, 128, 33), (7, 32, 97), (8, 128, 37), (8, 64, 259), (8, 32, 1)]


@pytest.mark.parametrize("P,G,k", RAGGED, ids=lambda v: str(v))
@pytest.mark.parametrize("fixup", ["exit", "deferred"])
def test_ragged_shapes(P, G, k, fixup):
    """N = P*G*k: owner chunks of k groups, so blocks of 256 threads end in
    a ragged tail; 4 calls, every element."""
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    with _plan(P, N, G, True, fixup) as plan:
        chk = SequenceChecker(plan, oracle_params(plan))
        for t in range(4):
            chk.step(W.generate(w, t, DEV))


def test_uncompensated_ragged():
    for P, G, k in RAGGED[:5]:
        N = P * G * k
        w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
        with _plan(P, N, G, False) as plan:
            chk = SequenceChecker(plan, oracle_params(plan))
            for t in range(2):
                chk.step(W.generate(w, t, DEV))


def _bf16(x_f32: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x_f32, np.float32)).to(torch.bfloat16).to(DEV)


def test_zero_inputs():
    P, G, N = 4, 64, 4 * 64 * 8
    with _plan(P, N, G) as plan:
        chk = SequenceChecker(plan, oracle_params(plan))
        out, _ = chk.step(torch.zeros((P, N), dtype=torch.bfloat16, device=DEV))
        assert not out.float().any()
        dv = plan.debug_view()
        assert not dv["scales"].any() and not dv["rscales"].any()


@pytest.mark.parametrize("comp", [True, False])
def test_grid_exact_inputs(comp):
    """Inputs on the int4 grid whose sums stay on it reduce exactly and
    leave the states at zero."""
    rng = np.random.default_rng(5)
    for P, G in ((2, 32), (8, 128), (5, 64)):
        N = P * G * 6
        with _plan(P, N, G, comp) as plan:
            chk = SequenceChecker(plan, oracle_params(plan))
            for _ in range(3):
                xf = oracle_pins.grid_exact_inputs(rng, P, N, G)
                out, _ = chk.step(_bf16(xf))
                exact = torch.from_numpy(xf.astype(np.float64).sum(axis=0))
                for r in range(P):
                    assert torch.equal(out[r].double().cpu(), exact)
            if comp:
                mf, ms = plan.get_state()
                assert not mf.any() and not ms.any()


def test_extreme_and_subnormal_inputs():
    """Huge values near the bf16 maximum, subnormal bf16 values (groups
    whose scale is subnormal or underflows to 0) and mixed groups."""
    P, G = 2, 32
    N = P * G * 8
    rng = np.random.default_rng(6)
    x = rng.normal(0, 1, (P, N)).astype(np.float32)
    x[:, 0:G] *= 3e37                       # large, sum stays finite
    x[:, G:2 * G] = rng.integers(-12, 13, (P, G)) * np.float32(2.0 ** -133)  # bf16 subnormals
    x[:, 2 * G:3 * G] = 0
    x[0, 2 * G] = np.float32(2.0 ** -133)  # a lone subnormal: scale underflows to 0
    x[:, 3 * G:4 * G] *= 1e-30
    with _plan(P, N, G) as plan:
        chk = SequenceChecker(plan, oracle_params(plan))
        for _ in range(3):
            chk.step(_bf16(x))


def test_in_place():
    """out[r] == in[r] is allowed and gives the same result."""
    w = W.with_size(W.TINY, P=4, rows=1, hidden=4 * 128 * 12, G=128)
    with _plan(w.P, w.N, w.G) as a, _plan(w.P, w.N, w.G) as b:
        for t in range(3):
            x = W.generate(w, t, DEV)
            ref = a.allreduce(x)
            y = x.clone()
            b.allreduce(y, out=y)
            torch.cuda.synchronize()
            assert torch.equal(ref, y)


@pytest.mark.parametrize("P,G,k,comp", [(8, 128, 1 << 13, False), (4, 32, 37, False),
                                         (4, 32, 37, True), (8, 128, 64, True)],
                         ids=["off-staged", "off", "comp-merged", "comp-merged-p8"])
def test_outputs_aligned_to_16_bytes_only(P, G, k, comp):
    """Outputs that start 16 bytes past a 32-byte boundary (the ABI asks for
    16-byte alignment; the kernels' 32-byte stores must then fall back):
    the same bits as outputs on aligned buffers, for all-reduce calls whose
    reduce writes the outputs (staged and direct) and for reduce-scatter."""
    N = P * G * k
    C = N // P
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    stride = N + 16                               # elements: a 32-byte multiple
    buf = torch.empty(8 + P * stride, dtype=torch.bfloat16, device=DEV)
    ys = [buf[8 + r * stride:8 + r * stride + N] for r in range(P)]
    zs = [buf[8 + r * stride:8 + r * stride + C] for r in range(P)]
    assert all(t.data_ptr() % 32 == 16 for t in ys + zs)
    with _plan(P, N, G, comp, "deferred") as a, _plan(P, N, G, comp, "deferred") as b:
        for t in range(3):
            x = W.generate(w, t, DEV)
            a.allreduce(x, out=ys)
            want = b.allreduce(x)
            assert torch.equal(torch.stack(ys).view(torch.int16), want.view(torch.int16)), t
        x = W.generate(w, 7, DEV)
        a.reduce_scatter(x, out=zs)
        want = b.reduce_scatter(x)
        assert torch.equal(torch.stack(zs).view(torch.int16), want.view(torch.int16))
        if comp:
            fa, sa = a.get_state()
            fb, sb = b.get_state()
            assert torch.equal(fa.view(torch.int32), fb.view(torch.int32))
            assert torch.equal(sa.view(torch.int32), sb.view(torch.int32))


def test_p1_identity_of_codes():
    """P=1: the requantization reproduces the entry codes."""
    w = W.with_size(W.TINY, P=1, rows=1, hidden=128 * 40, G=128)
    with _plan(1, w.N, 128) as plan:
        chk = SequenceChecker(plan, oracle_params(plan))
        for t in range(3):
            chk.step(W.generate(w, t, DEV))
            dv = plan.debug_view()
            assert torch.equal(dv["codes"][0], dv["rcodes"])


def test_determinism():
    w = W.with_size(W.TINY, P=8, rows=1, hidden=8 * 128 * 64, G=128)
    outs = []
    for _ in range(2):
        with _plan(w.P, w.N, w.G) as plan:
            ys = [plan.allreduce(W.generate(w, t, DEV)).clone() for t in range(3)]
            mf, ms = plan.get_state()
            torch.cuda.synchronize()
            outs.append((ys, mf, ms))
    (ya, mfa, msa), (yb, mfb, msb) = outs
    assert all(torch.equal(a, b) for a, b in zip(ya, yb))
    assert torch.equal(mfa, mfb) and torch.equal(msa, msb)


def test_fixup_modes_agree():
    """The three fix-up placements give bit-identical outputs and states."""
    w = W.with_size(W.TINY, P=8, rows=1, hidden=8 * 64 * 40, G=64)
    res = {}
    side = torch.cuda.Stream()
    for mode in ("exit", "side", "deferred"):
        with _plan(w.P, w.N, w.G, True, mode) as plan:
            ys = [plan.allreduce(W.generate(w, t, DEV), side_stream=side).clone()
                  for t in range(5)]
            torch.cuda.synchronize()
            res[mode] = (ys, plan.get_state())
            torch.cuda.synchronize()
    base_y, (bmf, bms) = res["exit"]
    for mode in ("side", "deferred"):
        ys, (mf, ms) = res[mode]
        assert all(torch.equal(a, b) for a, b in zip(base_y, ys)), mode
        assert torch.equal(mf, bmf) and torch.equal(ms, bms), mode


def test_state_roundtrip_and_reset():
    w = W.with_size(W.TINY, P=4, rows=1, hidden=4 * 32 * 16, G=32)
    with _plan(w.P, w.N, w.G, True, "deferred") as plan:
        chk = SequenceChecker(plan, oracle_params(plan))
        for t in range(3):
            chk.step(W.generate(w, t, DEV))
        mf, ms = plan.get_state()
        # restore into a fresh plan and continue: same as continuing here
        with _plan(w.P, w.N, w.G, True, "exit") as other:
            other.set_state(mf, ms)
            x = W.generate(w, 3, DEV)
            ya = plan.allreduce(x)
            yb = other.allreduce(x)
            torch.cuda.synchronize()
            assert torch.equal(ya, yb)
            assert all(torch.equal(a, b) for a, b in zip(plan.get_state(), other.get_state()))
        plan.reset_state()
        mf, ms = plan.get_state()
        torch.cuda.synchronize()
        assert not mf.any() and not ms.any()
        assert not plan.debug_view()["fixup_pending"]


@pytest.mark.parametrize("fixup", ["exit", "side", "deferred"])
@pytest.mark.parametrize("P,G,k", [(4, 128, 20), (3, 32, 37), (8, 64, 5), (2, 128, 1)],
                         ids=lambda v: str(v))
def test_host_call_matches_device_call(fixup, P, G, k):
    """The pipelined host-buffer call (slabs of every owner chunk, copies
    and kernels overlapped on three streams) gives the device call's bytes
    and states, call after call, including ragged last slabs."""
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    side = torch.cuda.Stream()
    with _plan(P, N, G, True, fixup) as a, _plan(P, N, G, True, fixup) as b:
        yh = torch.empty((P, N), dtype=torch.bfloat16, pin_memory=True)
        for t in range(4):
            x = W.generate(w, t, DEV)
            yd = a.allreduce(x, side_stream=side)
            xh = x.cpu().pin_memory()
            b.allreduce_host(xh, yh)
            torch.cuda.synchronize()
            assert torch.equal(yd.cpu(), yh), t
            ma, mb = a.get_state(), b.get_state()
            torch.cuda.synchronize()
            assert torch.equal(ma[0], mb[0]) and torch.equal(ma[1], mb[1]), t


def test_host_call_uncompensated_large_slabs():
    w = W.with_size(W.TINY, P=8, rows=1, hidden=8 * 128 * 1000, G=128)
    with _plan(w.P, w.N, w.G, False) as a, _plan(w.P, w.N, w.G, False) as b:
        x = W.generate(w, 0, DEV)
        yd = a.allreduce(x)
        yh = b.allreduce_host(x.cpu().pin_memory())
        torch.cuda.synchronize()
        assert torch.equal(yd.cpu(), yh)


def test_host_call_uncompensated_staged_slabs():
    """512 MiB per rank, P=8, G=128: each of the host call's 32 slabs holds
    2^17 runs of every owner chunk, so its reduce stages the code tiles in
    shared memory; in place on pinned memory, its outputs equal the device
    call's."""
    N = 1 << 28
    w = W.with_size(W.LARGE, P=8, rows=1, hidden=N, G=128)
    with _plan(w.P, N, w.G, False) as a, _plan(w.P, N, w.G, False) as b:
        x = W.generate(w, 0, DEV)
        yd = a.allreduce(x).cpu()
        xh = x.cpu().pin_memory()
        del x
        b.allreduce_host(xh, xh)
        torch.cuda.synchronize()
        assert torch.equal(yd, xh)
        del yd, xh
    torch.cuda.empty_cache()


@pytest.mark.parametrize("comp", [True, False])
def test_host_call_in_place(comp):
    """The host call with out_host == in_host (the bench's end-to-end leg)
    gives the device call's outputs and states over a sequence."""
    w = W.with_size(W.TINY, P=4, rows=1, hidden=4 * 64 * 300, G=64)
    with _plan(w.P, w.N, w.G, comp, "deferred") as a, _plan(w.P, w.N, w.G, comp, "deferred") as b:
        for t in range(3):
            x = W.generate(w, t, DEV)
            yd = a.allreduce(x)
            buf = x.cpu().pin_memory()
            b.allreduce_host(buf, buf)
            torch.cuda.synchronize()
            assert torch.equal(yd.cpu().view(torch.int16), buf.view(torch.int16)), t
        if comp:
            for sa, sb in zip(a.get_state(), b.get_state()):
                assert torch.equal(sa.view(torch.int32), sb.view(torch.int32))


@pytest.mark.parametrize("N", [2 * 32 * 64, 1 << 20], ids=["small", "large"])
def test_profile_counts_launches(N):
    """Entry, reduce and (compensated calls above 2^19 elements per rank)
    exit, plus the side-stream fix-up; the reduce writes the outputs
    otherwise."""
    w = W.with_size(W.TINY, P=2, rows=1, hidden=N, G=32)
    side = torch.cuda.Stream()
    for comp, mode in ((True, "exit"), (True, "side"), (True, "deferred"), (False, "exit")):
        per = 2 + int(comp and mode == "side")   # on one GPU the reduce writes the outputs
        with _plan(w.P, w.N, w.G, comp, mode) as plan:
            assert plan.launches_per_call() == per
            plan.profile_enable(True)
            for t in range(3):
                plan.allreduce(W.generate(w, t, DEV), side_stream=side)
            p = plan.profile_read(reset=True)
            assert p["calls"] == 3 and p["launches"] == 3 * per
            assert p["entry_ms"] > 0 and p["reduce_ms"] > 0


def test_argument_errors_on_device():
    from bit_error_compensated_echo_b200 import abi
    w = W.with_size(W.TINY, P=2, rows=1, hidden=2 * 32 * 8, G=32)
    with _plan(w.P, w.N, w.G) as plan:
        x = W.generate(w, 0, DEV)
        buf = torch.empty(w.N * 2 + 8, dtype=torch.bfloat16, device=DEV)
        mis = buf.data_ptr() + 2  # 2-byte offset: not 16-byte aligned
        with pytest.raises(abi.EchoError) as e:
            abi.echo_allreduce(plan.handle, [mis, x[1].data_ptr()],
                               [buf.data_ptr(), buf.data_ptr()], 0, 0)
        assert e.value.status == abi.ECHO_ERR_ALIGNMENT
        with pytest.raises(abi.EchoError) as e:  # overlapping outputs
            abi.echo_allreduce(plan.handle, [x[0].data_ptr(), x[1].data_ptr()],
                               [buf.data_ptr(), buf.data_ptr() + 16], 0, 0)
        assert e.value.status == abi.ECHO_ERR_INVALID_ARG
        with pytest.raises(abi.EchoError) as e:
            abi.echo_allreduce(plan.handle, [x[0].data_ptr(), 0], [buf.data_ptr()] * 2, 0, 0)
        assert e.value.status == abi.ECHO_ERR_INVALID_ARG
    with _plan(w.P, w.N, w.G, comp=False) as off:
        with pytest.raises(abi.EchoError) as e:
            off.get_state()
        assert e.value.status == abi.ECHO_ERR_INVALID_ARG
        off.reset_state()  # a no-op without the compensator


# ------------------------------------------------------------ full sizes

def test_llama_shape_full_sequence():
    """Llama-3-8B TP activations (8 ranks x 2048x4096, 8 outlier channels
    x50), 64 calls sharing one state; 1024 sampled group columns per call
    plus the first and the last; all ranks' outputs equal everywhere."""
    w = W.LLAMA
    cols = W.column_sample(w, 1024)
    with _plan(w.P, w.N, w.G) as plan:
        chk = SequenceChecker(plan, oracle_params(plan), cols)
        out = torch.empty((w.P, w.N), dtype=torch.bfloat16, device=DEV)
        for t in range(w.calls):
            x = W.generate(w, t, DEV)
            chk.step(x, out=out)
            assert all(torch.equal(out[0], out[r]) for r in range(1, w.P))


@pytest.mark.parametrize("comp,calls", [(True, 4), (False, 1)], ids=["comp4", "off1"])
def test_large_1gib_per_rank(comp, calls):
    """P=8, 2^29 bf16 per rank, N(0, 0.5^2), G=128, in the fix-up mode the
    benchmark times; 4096 sampled group columns plus the first and last."""
    from bench import BENCH_FIXUP
    w = W.LARGE
    cols = W.column_sample(w, 4096)
    with _plan(w.P, w.N, w.G, comp, BENCH_FIXUP) as plan:
        chk = SequenceChecker(plan, oracle_params(plan), cols)
        x = torch.empty((w.P, w.N), dtype=torch.bfloat16, device=DEV)
        out = torch.empty_like(x)
        for t in range(calls):
            W.generate(w, t, DEV, out=x)
            chk.step(x, out=out)
        assert all(torch.equal(out[0], out[r]) for r in range(1, w.P))
        del x, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("comp", [True, False], ids=["comp", "off"])
def test_message_beyond_int32_elements(comp):
    """P=2 ranks of 2^31 + 1024 elements each (4 GiB of bf16 per rank):
    every index of every kernel is past 32 bits somewhere; 2048 sampled
    group columns plus the first and the last, two calls."""
    from bench import BENCH_FIXUP
    N = (1 << 31) + 1024
    w = W.with_size(W.LARGE, P=2, rows=1, hidden=N, G=128)
    cols = W.column_sample(w, 2048)
    assert cols.max() * w.G >= (1 << 31)
    with _plan(w.P, w.N, w.G, comp, BENCH_FIXUP) as plan:
        chk = SequenceChecker(plan, oracle_params(plan), cols)
        x = torch.empty((w.P, w.N), dtype=torch.bfloat16, device=DEV)
        out = torch.empty_like(x)
        for t in range(2):
            W.generate(w, t, DEV, out=x)
            chk.step(x, out=out)
        assert torch.equal(out[0], out[1])
        del x, out
    torch.cuda.empty_cache()



def test_staged_reduce_every_element_ragged():
    """The uncompensated reduce that stages its code tiles in shared memory
    (P=8, G=128, owner chunks of at least 2^20 elements): owner chunks of
    2^20 + 384 elements, so each owner's last block of 256 runs is partial
    (24 runs); two calls, every element against the oracle."""
    P, G = 8, 128
    C = (1 << 20) + 3 * G
    N = P * C
    assert (C // 16) % 256 == 24
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    with _plan(P, N, G, False) as plan:
        chk = SequenceChecker(plan, oracle_params(plan))
        for t in range(2):
            chk.step(W.generate(w, t, DEV))

