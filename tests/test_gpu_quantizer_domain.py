"""The entry quantizer over the raw bf16 domain of uncompensated calls.

Uncompensated entry inputs are bf16 values and each group's scale comes
from a bf16 absmax, so exact ties of rint(x/scale) are common.  Each group
here holds one absmax a and up to 31 other bf16 values v with |v| <= a:
for every a in the set below, every finite bf16 v of magnitude at most a
appears once.  The set holds all 128 mantissas of one binade, plus
absmaxes across the exponent range: subnormal and tiny ones, whose scale
falls outside [2^-100, 2^100] or underflows, and huge ones.  One P=1 call
per code width; the entry codes and scales must equal the oracle's bit for
bit."""
import numpy as np
import pytest
import torch

import oracle
from bit_error_compensated_echo_b200.api import EchoPlan

pytestmark = pytest.mark.gpu

G = 32


def _absmaxes():
    ones = [0x3F80 | m for m in range(128)]                       # [1, 2): every mantissa
    rng = np.random.default_rng(5)
    spread = [int((e << 7) | rng.integers(0, 128)) for e in range(1, 255, 2)]
    # subnormal and smallest, around the 2^-100 and 2^100 scale limits, largest
    edge = [0x0001, 0x0007, 0x0080, 0x0C80, 0x0D00, 0x0E80, 0x0F00, 0x0F7F,
            0x6380, 0x6400, 0x7280, 0x72FF, 0x7300, 0x7F7F]
    return sorted(set(ones + spread + edge))


def _inputs():
    allv = np.arange(65536, dtype=np.uint32)
    f = (allv << 16).view(np.float32)
    finite = np.isfinite(f)
    groups = []
    for a_bits in _absmaxes():
        a = np.float32(np.uint32(a_bits << 16).view(np.float32))
        vals = allv[finite & (np.abs(f) <= a) & (allv != a_bits)].astype(np.uint16)
        pad = (-vals.size) % (G - 1)
        vals = np.concatenate([vals, np.zeros(pad, np.uint16)]).reshape(-1, G - 1)
        col = np.full((vals.shape[0], 1), a_bits, np.uint16)
        groups.append(np.concatenate([col, vals], axis=1))
    x = np.concatenate(groups).reshape(1, -1)
    return x


@pytest.mark.parametrize("bits", [4, 8])
def test_uncompensated_entry_over_the_bf16_domain(bits):
    xb = _inputs()
    N = xb.shape[1]
    ref = oracle.allreduce(oracle.Params(P=1, N=N, G=G, compensate=False, bits=bits), xb,
                           None, None)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to("cuda:0")
    with EchoPlan(1, N, G, compensate=False, device=0, bits=bits) as plan:
        plan.allreduce(x)
        torch.cuda.synchronize()
        dv = plan.debug_view()
        codes = dv["codes"].cpu().numpy()
        scales = dv["scales"].cpu().numpy()
    assert np.array_equal(scales.view(np.uint32), ref.scales.view(np.uint32))
    bad = np.flatnonzero(codes != ref.codes)
    assert bad.size == 0, "%d code bytes differ, first at %d" % (bad.size, bad[0])
