"""The compensated entry's quantizer at and around rounding ties, against the
oracle, bit for bit.

The compensated entry rounds x~/scale by multiplying with the rounded
reciprocal of the scale; an element whose product lies within the tie
window of a half-integer (2^-18 for 4-bit codes, 2^-13 for 8-bit) takes
the IEEE division instead, and so does every group whose scale lies
outside [2^-100, 2^100].  With a zero state the corrected input is the raw
bf16 input, so ordinary sequences reach that fallback only by chance.  Here
the state is set (echo_set_state) so that the corrected input x~ = x + c
lands exactly where the decision is delicate: on half-integer quotients,
one and two ulps either side of them, and at offsets just inside and just
outside the tie window, for scales from 2^-120 to 2^115, including the
window's bounds 2^-100 and 2^100 themselves.  Codes, scales, outputs,
e_req and both states of two consecutive calls must equal the oracle's.

The definition being checked: k = clamp(rint(fl(x~/scale)), -L, L) with
rint rounding half to even, scale = fl(a/L) (arXiv abstract on the fugumt
mirror: 4-bit integer transport; the readings of the quantizer are the
library's, written out in include/echo.h).
"""
import numpy as np
import pytest
import torch

from bit_error_compensated_echo_b200 import workloads as W
from bit_error_compensated_echo_b200.api import EchoPlan
from parity import SequenceChecker, oracle_params

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
LEVELS = {4: 7, 8: 127}
WINDOW = {4: 2.0 ** -18, 8: 2.0 ** -13}
# exponents of the scales: both sides of 2^-100 and 2^100, and far out
EXPONENTS = [-120, -101, -100, -99, -40, -1, 0, 1, 40, 99, 100, 101, 115]


def _f32(v):
    return np.asarray(v, dtype=np.float32)


def near_tie_targets(P: int, N: int, G: int, bits: int, seed: int):
    """[P, N] fp32 corrected inputs x~: per group one absmax element +-a
    and G-1 elements whose quotient by scale = fl(a/L) sits on or next to
    a half-integer.  Returns (targets, scales)."""
    L = LEVELS[bits]
    rng = np.random.default_rng(seed)
    groups = P * N // G
    t = np.zeros((groups, G), np.float32)
    scales = np.zeros(groups, np.float32)
    w = WINDOW[bits]
    offsets = np.array([0.0, w / 4, w / 2, w * 0.999, w * 1.001, 2 * w, 4 * w])
    for g in range(groups):
        e = EXPONENTS[g % len(EXPONENTS)]
        m = 1.0 if (g // len(EXPONENTS)) % 4 == 0 else rng.uniform(1.0, 2.0)
        a = _f32(np.ldexp(m, e) * L)                  # the group's absmax
        s = _f32(a / _f32(L))                          # fl(a/L), IEEE
        scales[g] = s
        h = rng.integers(-L, L, size=G - 1) + 0.5      # half-integers in (-L, L)
        kind = rng.integers(0, 4, size=G - 1)
        off = offsets[rng.integers(0, len(offsets), size=G - 1)]
        off = off * np.where(rng.random(G - 1) < 0.5, -1.0, 1.0)
        v = _f32(np.float64(s) * (h + np.where(kind == 3, off, 0.0)))
        # kinds 1 and 2: one or two ulps either side of fl(h*s)
        step = np.where(rng.random(G - 1) < 0.5, -np.inf, np.inf).astype(np.float32)
        v = np.where(kind >= 1, np.where(kind <= 2, np.nextafter(v, step), v), v)
        v = np.where(kind == 2, np.nextafter(v, step), v)
        row = np.concatenate([[a if rng.random() < 0.5 else -a], v]).astype(np.float32)
        t[g] = row[rng.permutation(G)]
    return t.reshape(P, N), scales


def states_for(t: np.ndarray, seed: int):
    """bf16 inputs x and states (m_fast, m_slow) with alpha = 1/2 such that
    fl(x + fl(fl(1/2*m_fast) + fl(1/2*m_slow))) == t exactly: c = t - x
    where that subtraction and the add back are exact, else x = 0 and c = t;
    c is carried by m_fast in half of the elements and by m_slow in the
    other half (the other state 0)."""
    rng = np.random.default_rng(seed)
    xb = torch.from_numpy(rng.standard_normal(t.shape).astype(np.float32)).to(torch.bfloat16)
    x = xb.float().numpy()
    c = _f32(t - x)
    ok = (_f32(x + c) == t) & (_f32(t - c) == x) & np.isfinite(2 * c.astype(np.float64))
    x = np.where(ok, x, np.float32(0.0)).astype(np.float32)
    c = np.where(ok, c, t).astype(np.float32)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(xb.float().numpy(), x)
    fast = rng.random(t.shape) < 0.5
    mf = np.where(fast, 2 * c, 0).astype(np.float32)
    ms = np.where(fast, 0, 2 * c).astype(np.float32)
    # the corrected input the definition computes from these, in fp32
    half = np.float32(0.5)
    cc = _f32(_f32(half * mf) + _f32(half * ms))
    assert np.array_equal(_f32(x + cc), t)
    return xb, mf, ms


def construction_reaches_the_fallback(t, scales, G, bits):
    """The host-side evidence that the inputs do what they are for: many
    quotients are exact ties, and many are flagged by the fast path."""
    L = LEVELS[bits]
    s = np.repeat(scales, G).reshape(t.shape)
    q = _f32(t / s)
    frac = np.abs(q - np.floor(q)).astype(np.float64)
    exact_ties = np.mean(frac == 0.5)
    fast_ok = (s >= np.float32(2.0 ** -100)) & (s <= np.float32(2.0 ** 100))
    inv = np.where(fast_ok, _f32(np.float32(1.0) / s), np.float32(0.0)).astype(np.float32)
    qt = _f32(t * inv)
    d = np.abs(qt - np.rint(qt))
    flagged = np.mean(fast_ok & (d > 0.5 - WINDOW[bits]))
    unflagged_near = np.mean(fast_ok & (d <= 0.5 - WINDOW[bits]) & (d > 0.5 - 8 * WINDOW[bits]))
    assert np.all(np.abs(q) <= L + 1e-3)
    return exact_ties, flagged, unflagged_near, np.mean(~fast_ok)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("G", [32, 128])
@pytest.mark.parametrize("fixup", ["exit", "deferred"])
def test_compensated_entry_near_ties(bits, G, fixup):
    P = 2
    N = G * 13 * 24          # 24 groups per exponent per rank
    t, scales = near_tie_targets(P, N, G, bits, seed=G + bits)
    ties, flagged, near, slow = construction_reaches_the_fallback(t, scales, G, bits)
    assert ties > 0.1 and flagged > 0.3 and near > 0.05 and slow > 0.1, \
        (ties, flagged, near, slow)
    xb, mf, ms = states_for(t, seed=7 * G + bits)
    with EchoPlan(P, N, G, compensate=True, fixup=fixup, bits=bits, device=0) as plan:
        plan.set_state(torch.from_numpy(mf).to(DEV), torch.from_numpy(ms).to(DEV))
        chk = SequenceChecker(plan, oracle_params(plan))
        chk.mf[...] = mf
        chk.ms[...] = ms
        chk.step(xb.to(DEV))
        # the scales the entry chose are the construction's (absmax / L)
        assert np.array_equal(plan.debug_view()["scales"].cpu().numpy().reshape(-1), scales)
        # a second call on the state the first one left: ordinary inputs
        w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
        chk.step(W.generate(w, 1, DEV))
