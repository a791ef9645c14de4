"""The GPU against the hand-worked sequence of tests/golden/sequence_worked.txt,
with no oracle in between.

The fixture's groups have 4 elements; the kernels take G = 32.  Each of its
groups becomes the first 4 elements of a 32-element group, the other 28
zero: absmax and scale are unchanged, zeros quantize to code 0 with zero
residual, and sums, outputs and states at the fixture's elements are those
of the fixture (chunk o is group o, as there).  Every other element must
come out as +0 (codes 0)."""
import os

import numpy as np
import pytest
import torch

from bit_error_compensated_echo_b200.api import EchoPlan

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
G = 32


def _spec():
    spec = {}
    with open(os.path.join(GOLDEN, "sequence_worked.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = [p.strip() for p in line.split("=", 1)]
                spec[k] = v
    return spec


def _spread(vals, g_small, P_groups):
    """Fixture values (per rank: groups of g_small) into groups of G."""
    out = np.zeros(P_groups * G, np.float64)
    for grp in range(P_groups):
        out[grp * G:grp * G + g_small] = vals[grp * g_small:(grp + 1) * g_small]
    return out


def _bytes_spread(hexvals, g_small, P_groups):
    """Packed 4-bit codes: each group's g_small/2 bytes, then zero bytes."""
    out = np.zeros(P_groups * G // 2, np.uint8)
    b = [int(t, 16) for t in hexvals.split()]
    for grp in range(P_groups):
        out[grp * G // 2:grp * G // 2 + g_small // 2] = b[grp * g_small // 2:(grp + 1) * g_small // 2]
    return out


@pytest.mark.parametrize("fixup", ["exit", "side", "deferred"])
def test_gpu_reproduces_hand_worked_sequence(fixup):
    s = _spec()
    P, n_small, g_small = int(s["P"]), int(s["N"]), int(s["G"])
    groups = n_small // g_small
    N = groups * G
    vec = lambda k: np.array([float(t) for t in s[k].split()])      # noqa: E731
    side = torch.cuda.Stream() if fixup == "side" else None
    with EchoPlan(P, N, G, alpha=float(s["alpha"]), beta_fast=float(s["beta_fast"]),
                  beta_slow=float(s["beta_slow"]), device=0, fixup=fixup) as plan:
        for call in (1, 2):
            x = np.stack([_spread(vec("x%d.%d" % (r, call)), g_small, groups) for r in range(P)])
            xt = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)
            assert torch.equal(xt.double(), torch.tensor(x)), "inputs must be bf16 values"
            y = plan.allreduce(xt.to(DEV), side_stream=side)
            torch.cuda.synchronize()
            want_y = _spread(vec("y.%d" % call), g_small, groups)
            zero = torch.tensor(want_y == 0)
            for r in range(P):
                yr = y[r].cpu()
                assert torch.equal(yr.double(), torch.tensor(want_y)), (call, r)
                assert not torch.signbit(yr[zero].float()).any(), (call, r)   # zeros are +0
            dv = plan.debug_view()
            for r in range(P):
                got = dv["codes"][r].cpu().numpy()
                want = _bytes_spread(s["codes%d.%d" % (r, call)], g_small, groups)
                assert np.array_equal(got, want), (call, r, got, want)
            rc = dv["rcodes"].cpu().numpy()
            assert np.array_equal(rc, _bytes_spread(s["rcodes.%d" % call], g_small, groups))
            mf, ms = plan.get_state()
            for r in range(P):
                for name, m in (("m_fast", mf), ("m_slow", ms)):
                    want = _spread(vec("%s%d.%d" % (name, r, call)), g_small, groups)
                    got = m[r].cpu().double().numpy()
                    assert np.array_equal(got, want), (call, name, r, got, want)
                    # the padding stays +0, not -0
                    assert not np.signbit(got[want == 0]).any(), (call, name, r)
