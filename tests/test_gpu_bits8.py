"""8-bit codes (levels -127..127, one byte per code) against the oracle:
whole sequences, ragged shapes, the reduce-scatter, the pipelined host
call, grid-exact inputs and the Llama-shaped workload on sampled columns.
The pages' serving policy gives 8-bit codes to the earlier layers, half of them
(ai4snews news summary, "Perspective"): a plan made with bits=8 runs each
call at 4 or 8 bits on one compensator state, which the mixed-width
sequences below check call by call, following the layer policy."""
import numpy as np
import pytest
import torch

import oracle_pins
from bit_error_compensated_echo_b200 import workloads as W
from bit_error_compensated_echo_b200 import abi
from bit_error_compensated_echo_b200.api import EchoPlan
from bit_error_compensated_echo_b200.policy import LayerPolicy
from parity import RSChecker, SequenceChecker, oracle_params

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _plan(P, N, G, comp=True, fixup="exit"):
    return EchoPlan(P, N, G, compensate=comp, fixup=fixup, device=0, bits=8)


@pytest.mark.parametrize("comp,fixup", [(True, "exit"), (True, "side"), (True, "deferred"),
                                        (False, "exit")])
def test_tiny_sequence_8bit(comp, fixup):
    w = W.TINY
    side = torch.cuda.Stream() if fixup == "side" else None
    with _plan(w.P, w.N, w.G, comp, fixup) as plan:
        chk = SequenceChecker(plan, oracle_params(plan))
        for t in range(w.calls):
            chk.step(W.generate(w, t, DEV), side_stream=side)


@pytest.mark.parametrize("P,G,k", [(1, 32, 37), (3, 128, 41), (5, 64, 29), (8, 128, 37),
                                   (8, 32, 1)], ids=lambda v: str(v))
def test_ragged_8bit(P, G, k):
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    with _plan(P, N, G, True, "deferred") as plan:
        chk = SequenceChecker(plan, oracle_params(plan))
        for t in range(3):
            chk.step(W.generate(w, t, DEV))


def test_reduce_scatter_8bit():
    w = W.with_size(W.TINY, P=4, rows=1, hidden=4 * 64 * 24, G=64)
    with _plan(w.P, w.N, w.G, True, "deferred") as plan:
        chk = RSChecker(plan, oracle_params(plan))
        for t, op in enumerate("RARR"):
            x = W.generate(w, t, DEV)
            if op == "A":
                chk.step(x)
            else:
                chk.step_rs(x)


def test_grid_exact_8bit():
    rng = np.random.default_rng(9)
    P, G = 4, 64
    N = P * G * 6
    with _plan(P, N, G) as plan:
        chk = SequenceChecker(plan, oracle_params(plan))
        for _ in range(3):
            xf = oracle_pins.grid_exact_inputs(rng, P, N, G, L=127)
            x = torch.from_numpy(xf).to(torch.bfloat16).to(DEV)
            out, _ = chk.step(x)
            exact = torch.from_numpy(xf.astype(np.float64).sum(axis=0))
            assert torch.equal(out[0].double().cpu(), exact)


def test_host_call_8bit():
    w = W.with_size(W.TINY, P=8, rows=1, hidden=8 * 128 * 9, G=128)
    with _plan(w.P, w.N, w.G, True, "deferred") as a, _plan(w.P, w.N, w.G, True, "deferred") as b:
        yh = torch.empty((w.P, w.N), dtype=torch.bfloat16, pin_memory=True)
        for t in range(3):
            x = W.generate(w, t, DEV)
            yd = a.allreduce(x)
            b.allreduce_host(x.cpu().pin_memory(), yh)
            torch.cuda.synchronize()
            assert torch.equal(yd.cpu(), yh)


def test_llama_shape_8bit_sampled():
    w = W.LLAMA
    with _plan(w.P, w.N, w.G, True, "deferred") as plan:
        chk = SequenceChecker(plan, oracle_params(plan), W.column_sample(w, 512))
        for t in range(8):
            chk.step(W.generate(w, t, DEV))


@pytest.mark.parametrize("fixup", ["exit", "side", "deferred"])
def test_layer_policy_sequence_one_state(fixup):
    """Two passes over a 6-layer model (2 sites per layer), the first 3
    layers at 8 bits: 24 calls of both widths on one state, each against the
    oracle at the call's width."""
    pol = LayerPolicy(6, 2, 0.5)
    w = W.with_size(W.TINY, P=4, rows=1, hidden=4 * 64 * 10, G=64)
    side = torch.cuda.Stream() if fixup == "side" else None
    with _plan(w.P, w.N, w.G, True, fixup) as plan:
        chk = SequenceChecker(plan, oracle_params(plan))
        for t in range(2 * pol.sites):
            chk.step(W.generate(w, t, DEV), side_stream=side, bits=pol.bits_for_site(t))
        assert plan.bits == 4


def test_mixed_widths_reduce_scatter_and_allreduce():
    w = W.with_size(W.TINY, P=8, rows=1, hidden=8 * 128 * 5, G=128)
    with _plan(w.P, w.N, w.G, True, "deferred") as plan:
        chk = RSChecker(plan, oracle_params(plan))
        for t, (op, bits) in enumerate([("A", 8), ("R", 4), ("A", 4), ("R", 8), ("A", 8),
                                        ("A", 4), ("R", 4), ("R", 8)]):
            x = W.generate(w, t, DEV)
            if op == "A":
                chk.step(x, bits=bits)
            else:
                chk.step_rs(x, bits=bits)


def test_llama_policy_sampled():
    """The Llama-shaped workload's 64 calls (2 per layer x 32 layers) with
    the first 16 layers at 8 bits, sampled columns against the oracle."""
    w = W.LLAMA
    pol = LayerPolicy(32, 2, 0.5)
    with _plan(w.P, w.N, w.G, True, "deferred") as plan:
        chk = SequenceChecker(plan, oracle_params(plan), W.column_sample(w, 256))
        for t in range(0, pol.sites, 4):        # every 4th site, both widths
            chk.step(W.generate(w, t, DEV), bits=pol.bits_for_site(t))


def test_set_bits_limits():
    with EchoPlan(2, 2 * 32 * 4, 32, device=0, bits=4) as p4:
        with pytest.raises(abi.EchoError) as e:
            p4.set_bits(8)                       # transport sized for 4 bits
        assert e.value.status == abi.ECHO_ERR_UNSUPPORTED
    with EchoPlan(2, 2 * 32 * 4, 32, device=0, bits=8) as p8:
        for bad in (0, 5, 16):
            with pytest.raises(abi.EchoError):
                p8.set_bits(bad)
        p8.set_bits(4)
        assert p8.debug_view()["codes"].shape == (2, 2 * 32 * 4 // 2)


@pytest.mark.parametrize("op,comp", [("allreduce", False), ("reduce_scatter", True),
                                     ("reduce_scatter", False)])
def test_staged_8bit_every_element_ragged(op, comp):
    """The kernels that stage their code tiles in shared memory, at 8 bits
    (P=8, G=128, owner chunks of at least 2^20 elements): the uncompensated
    reduce that writes the outputs and the reduce-scatter kernel.  Owner
    chunks of 2^20 + 384 elements (each owner's last block of 256 runs holds
    24); two calls, every element against the oracle."""
    P, G = 8, 128
    C = (1 << 20) + 3 * G
    N = P * C
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    with _plan(P, N, G, comp, "deferred") as plan:
        if op == "allreduce":
            chk = SequenceChecker(plan, oracle_params(plan))
            for t in range(2):
                chk.step(W.generate(w, t, DEV))
        else:
            chk = RSChecker(plan, oracle_params(plan))
            for t in range(2):
                chk.step_rs(W.generate(w, t, DEV))
