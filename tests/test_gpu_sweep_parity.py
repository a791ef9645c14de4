"""Sampled parity of sweep points: every P in {2, 4, 8} and G in {32, 64,
128}, compensated and not, on N(0,1) inputs with a fresh 0.1% of the
elements scaled x30, at 1 MiB per rank (and 16 MiB for P=8, G=128);
two calls each, 256 sampled group columns plus the first and the last."""
import pytest

from bit_error_compensated_echo_b200 import workloads as W
from bit_error_compensated_echo_b200.api import EchoPlan
from parity import SequenceChecker, oracle_params

pytestmark = pytest.mark.gpu

POINTS = [(1, P, G, c) for P in W.SWEEP_P for G in W.SWEEP_G for c in (True, False)] + \
         [(16, 8, 128, True), (16, 8, 128, False)]


@pytest.mark.parametrize("mib,P,G,comp", POINTS, ids=lambda v: str(v))
def test_sweep_point_sampled(mib, P, G, comp):
    w = W.sweep_point(mib, P, G, comp)
    with EchoPlan(w.P, w.N, w.G, compensate=comp, fixup="deferred", device=0) as plan:
        chk = SequenceChecker(plan, oracle_params(plan), W.column_sample(w, 256))
        for t in range(2):
            chk.step(W.generate(w, t, "cuda:0"))
