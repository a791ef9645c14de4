"""Depth-chain property on the GPU: with the compensator the accumulated
deviation from the exact fp32 chain stays bounded over 56 sites; without it
the deviation keeps growing (Qwen3-0.6B-like shape: P=8, 32768 tokens x
1024 hidden, Student-t nu=3 inputs, Haar-orthogonal site maps, RMSNorm).

The pages state that the total error has a bound that does not grow with
the number of layers, if no direction is magnified again and again (arXiv abstract on the
fugumt mirror; ai4snews news summary, "Perspective"); orthogonal maps and
RMSNorm satisfy that assumption.  The deviation tests are property checks;
in the same run every one of the library's calls (56 forward and 56
backward sites of the compensated, uncompensated and promoted chains, the
promoted one across its 8-bit to 4-bit switch) is also checked against the
oracle, bit for bit, on a sample of group columns: entry and reduced codes
and scales, outputs, e_req and both states.  The inputs of these calls are
post-RMSNorm partial products of rotated heavy-tailed activations, and the
states carry across all 56 sites.
"""
import collections

import pytest

from bit_error_compensated_echo_b200 import depth_chain
from bit_error_compensated_echo_b200 import workloads as W
from parity import SequenceChecker, oracle_params

pytestmark = pytest.mark.gpu

# 256 random group columns plus the first and the last, of 262,144
COLS = W.column_sample(W.DEPTH, 256, seed=4242)


class OracleWatch:
    """Depth-chain observer: checks each call against the oracle on COLS.
    A chain's first mismatch is recorded and ends the checks of that chain
    (its states have left the oracle's from there on)."""

    def __init__(self, cols):
        self.cols = cols
        self.checkers = {}
        self.checked = collections.Counter()
        self.failures = {}

    def __call__(self, direction, site, chain, plan, x, y):
        key = (direction, chain)
        if key in self.failures:
            return
        chk = self.checkers.get(key)
        if chk is None or chk.plan is not plan:
            chk = self.checkers[key] = SequenceChecker(plan, oracle_params(plan), self.cols)
        try:
            chk.verify(x, y)
        except AssertionError as e:
            self.failures[key] = "site %d, %d-bit: %s" % (site, plan.bits, e)
        self.checked[key] += 1


@pytest.fixture(scope="module")
def run_with_watch():
    watch = OracleWatch(COLS)
    res = depth_chain.run(P=8, tokens=W.DEPTH.rows, hidden=W.DEPTH.hidden,
                          sites=W.DEPTH.calls, G=W.DEPTH.G, seed=W.DEPTH.seed,
                          device="cuda:0", observer=watch)
    return res, watch


@pytest.fixture(scope="module")
def chain(run_with_watch):
    return run_with_watch[0]


def test_every_call_matches_the_oracle(run_with_watch):
    """Config 4 at full size (P=8, 32768 x 1024, G=128): all 336 calls of
    the three library chains against the oracle on 258 group columns."""
    _, watch = run_with_watch
    assert not watch.failures, watch.failures
    for direction in ("forward", "backward"):
        for name in ("comp", "off", "promoted"):
            assert watch.checked[(direction, name)] == W.DEPTH.calls, (direction, name)


def test_forward_deviation_bounded_with_compensation(chain):
    comp, off, b16 = (chain["forward_rel"][k] for k in ("comp", "off", "bf16"))
    assert len(comp) == W.DEPTH.calls
    half = len(comp) // 2
    # compensated: flat over the second half of the chain
    assert comp[-1] <= comp[half - 1] * 1.05, (comp[half - 1], comp[-1])
    # uncompensated: still growing, and well above the compensated chain
    assert off[-1] >= off[half - 1] * 1.05, (off[half - 1], off[-1])
    assert comp[-1] <= 0.75 * off[-1], (comp[-1], off[-1])
    # the 16-bit all-reduce is far more accurate than either 4-bit chain
    assert b16[-1] < 0.1 * comp[-1]


def test_backward_deviation_smaller_with_compensation(chain):
    comp, off = chain["backward_rel"]["comp"], chain["backward_rel"]["off"]
    assert comp[-1] <= 0.75 * off[-1], (comp[-1], off[-1])
    assert sum(comp) < 0.75 * sum(off)


def test_layer_policy_promotion(chain):
    """The serving policy (the earlier half of the layers at 8 bits, one state;
    ai4snews news summary, "Perspective"): forward, the 8-bit half stays far
    below the 4-bit chain and the end of the chain is well below it;
    backward runs the 4-bit layers first, so the promoted chain equals the
    4-bit chain there and drops below it once the 8-bit layers come."""
    comp, prom = chain["forward_rel"]["comp"], chain["forward_rel"]["promoted"]
    half = len(comp) // 2
    assert prom[half - 1] < 0.1 * comp[half - 1], (prom[half - 1], comp[half - 1])
    assert prom[-1] < 0.6 * comp[-1], (prom[-1], comp[-1])
    bcomp, bprom = chain["backward_rel"]["comp"], chain["backward_rel"]["promoted"]
    for a, b in zip(bcomp[:half], bprom[:half]):
        assert abs(a - b) <= 1e-6 * a, (a, b)
    assert bprom[-1] < 0.5 * bcomp[-1], (bprom[-1], bcomp[-1])
