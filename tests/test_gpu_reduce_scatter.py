"""The reduce-scatter call (echo_reduce_scatter) against the oracle's
reduce-scatter, call by call: entry codes and scales, what every owner
receives, the owner's output residual and both EMA states."""
import pytest
import torch

from bit_error_compensated_echo_b200 import workloads as W
from bit_error_compensated_echo_b200.api import EchoPlan
from parity import RSChecker, oracle_params

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _plan(P, N, G, comp=True, fixup="exit"):
    return EchoPlan(P, N, G, compensate=comp, fixup=fixup, device=0)


@pytest.mark.parametrize("comp,fixup", [(True, "exit"), (True, "side"), (True, "deferred"),
                                        (False, "exit")])
def test_tiny_rs_sequence(comp, fixup):
    w = W.TINY
    side = torch.cuda.Stream() if fixup == "side" else None
    with _plan(w.P, w.N, w.G, comp, fixup) as plan:
        chk = RSChecker(plan, oracle_params(plan))
        for t in range(w.calls):
            chk.step_rs(W.generate(w, t, DEV), side_stream=side)


@pytest.mark.parametrize("P,G,k", [(1, 32, 37), (3, 128, 41), (5, 64, 29), (8, 128, 37),
                                   (8, 32, 1)], ids=lambda v: str(v))
@pytest.mark.parametrize("fixup", ["exit", "deferred"])
def test_rs_ragged(P, G, k, fixup):
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    with _plan(P, N, G, True, fixup) as plan:
        chk = RSChecker(plan, oracle_params(plan))
        for t in range(3):
            chk.step_rs(W.generate(w, t, DEV))


@pytest.mark.parametrize("fixup", ["exit", "side", "deferred"])
def test_rs_and_allreduce_share_the_state(fixup):
    """A plan's all-reduce and reduce-scatter calls feed one compensator
    state, in any order."""
    w = W.with_size(W.TINY, P=4, rows=1, hidden=4 * 64 * 24, G=64)
    side = torch.cuda.Stream()
    with _plan(w.P, w.N, w.G, True, fixup) as plan:
        chk = RSChecker(plan, oracle_params(plan))
        for t, op in enumerate("ARRARAAR"):
            x = W.generate(w, t, DEV)
            if op == "A":
                chk.step(x, side_stream=side)
            else:
                chk.step_rs(x, side_stream=side)


def test_rs_llama_shape_sampled():
    w = W.LLAMA
    with _plan(w.P, w.N, w.G, True, "deferred") as plan:
        chk = RSChecker(plan, oracle_params(plan), W.column_sample(w, 512))
        for t in range(8):
            chk.step_rs(W.generate(w, t, DEV))


def test_rs_profile_counts_two_launches():
    w = W.with_size(W.TINY, P=2, rows=1, hidden=2 * 32 * 64, G=32)
    with _plan(w.P, w.N, w.G, True, "deferred") as plan:
        plan.profile_enable(True)
        for t in range(3):
            plan.reduce_scatter(W.generate(w, t, DEV))
        p = plan.profile_read(reset=True)
        assert p["calls"] == 3 and p["launches"] == 6


@pytest.mark.parametrize("G,comp,fixup", [(128, True, "exit"), (128, True, "side"),
                                          (128, True, "deferred"), (128, False, "deferred"),
                                          (64, True, "deferred")])
def test_rs_staged_every_element_ragged(G, comp, fixup):
    """The reduce-scatter kernel that stages its code tiles in shared memory
    (P=8, G=64 or 128, owner chunks of at least 2^20 elements): owner chunks
    of 2^20 + 3G elements, so each owner's last block of 256 runs is partial;
    two calls, every element of the owners' outputs and both states against
    the oracle."""
    P = 8
    C = (1 << 20) + 3 * G
    N = P * C
    assert (C // 16) % 256 in (12, 24)
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    side = torch.cuda.Stream() if fixup == "side" else None
    with EchoPlan(P, N, G, compensate=comp, fixup=fixup, device=0) as plan:
        chk = RSChecker(plan, oracle_params(plan))
        for t in range(2):
            chk.step_rs(W.generate(w, t, DEV), side_stream=side)
