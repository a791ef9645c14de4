"""Pins of the CPU oracle to facts outside the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with what the pages and the mathematics fix:
brute force over the 15 code levels in exact rational arithmetic, a library
routine (torch's bf16 rounding), hand-worked examples under tests/golden/,
closed forms (the telescoping identity of the dual-EMA compensator, the EMA
closed form, the packed-bytes ratio) and invariants (grid-exact inputs,
exactly two quantizations per value, column locality, determinism).

The pages ("Echo: Error-Compensated 4-Bit Tensor-Parallel Communication",
ai4snews news summary "Interpretation" and the arXiv abstract on the fugumt
mirror) print no worked numbers, so no pin compares with a printed value.

test_oracle_pins.py runs every pin on the oracle; test_oracle_mutants.py
runs them on broken copies of the oracle and requires each copy to fail one.
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

DEFAULTS = dict(alpha=0.5, beta_fast=0.5, beta_slow=0.95)


def bf16_bits(x) -> np.ndarray:
    """fp32 values -> bf16 bit patterns via torch's own rounding."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


def _params(o, P, N, G, comp=True, **kw):
    from oracle import Params
    d = dict(DEFAULTS)
    d.update(kw)
    return Params(P=P, N=N, G=G, compensate=comp, **d)


def _run_sequence(o, prm, xs):
    """Run calls on inputs xs[t] ([P, N] bf16 bits) from zero state."""
    P, N = prm.P, prm.N
    mf = np.zeros((P, N), np.float32)
    ms = np.zeros((P, N), np.float32)
    out = []
    for x in xs:
        r = o.allreduce(prm, x, mf, ms)
        out.append((r, mf.copy(), ms.copy()))
    return out


def _owner(prm, n_idx):
    return np.asarray(n_idx) // (prm.N // prm.P)


# ---------------------------------------------------------------- primitives

def pin_bf16_conversion(o):
    """fp32 <-> bf16 agrees with torch's round-to-nearest-even conversion."""
    rng = np.random.default_rng(11)
    u = rng.integers(0, 2**32, size=6000, dtype=np.uint64).astype(np.uint32)
    ties = (rng.integers(0, 2**16, size=2000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    edge = np.array([0, 0x80000000, 0x00000001, 0x00008000, 0x00018000,
                     0x7f7fffff, 0xff7fffff, 0x7f800000, 0x3f808000,
                     0x3f818000, 0x007fffff], dtype=np.uint32)
    bits = np.concatenate([u, ties, edge])
    f = bits.view(np.float32)
    f = f[~np.isnan(f)]
    ours = o.f32_to_bf16(f)
    ref = bf16_bits(f)
    assert np.array_equal(ours, ref), "fp32->bf16 differs from torch"
    hb = rng.integers(0, 2**16, size=3000, dtype=np.uint64).astype(np.uint16)
    hb = hb[~np.isnan(bits_to_f64(hb))]
    ref32 = torch.from_numpy(hb.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert np.array_equal(o.bf16_to_f32(hb).view(np.uint32), ref32.view(np.uint32))


def _exact_argmins(v: float, scale: float):
    fv, fs = Fraction(v), Fraction(scale)
    errs = [(abs(fv - k * fs), k) for k in range(-7, 8)]
    m = min(e for e, _ in errs)
    return [k for e, k in errs if e == m]


def _nearest_f32_check(value: Fraction, f: np.float32):
    """f is a float32 nearest to the rational value."""
    d = abs(Fraction(float(f)) - value)
    for nb in (np.nextafter(f, np.float32(-np.inf)), np.nextafter(f, np.float32(np.inf))):
        assert d <= abs(Fraction(float(nb)) - value), (float(f), float(value))


def _quant_groups(rng):
    groups = []
    for _ in range(60):
        G = int(rng.choice([2, 4, 8, 16, 32]))
        kind = rng.integers(0, 6)
        if kind == 0:
            v = rng.normal(0, 10.0 ** rng.integers(-3, 4), G)
        elif kind == 1:
            v = rng.uniform(-1, 1, G) * 2.0 ** rng.integers(-20, 20)
        elif kind == 2:
            v = rng.standard_t(3, G)
        elif kind == 3:
            v = rng.normal(0, 1, G) * (rng.random(G) < 0.3)
        elif kind == 4:
            # exact ties: max 7*2^e gives scale 2^e; others (j+1/2)*2^e
            e = int(rng.integers(-6, 6))
            j = rng.integers(-7, 7, G).astype(np.float64)
            v = (j + 0.5) * 2.0 ** e
            v[rng.integers(0, G)] = 7.0 * 2.0 ** e * rng.choice([-1, 1])
        else:
            # subnormal groups: the scale is a few subnormal steps, or 0
            step = np.float64(np.float32(1.4e-45))
            v = rng.integers(-12, 13, G) * step
        groups.append(np.asarray(v, np.float32))
    groups.append(np.zeros(8, np.float32))
    groups.append(np.array([1.4e-45, 0, -1.4e-45, 0], np.float32))  # scale underflows
    # a = 10 subnormal steps: the scale rounds to 1 step, so v/scale = +-10
    # and only the clamp keeps the codes at +-7
    step = np.float64(np.float32(1.4e-45))
    groups.append(np.array([10 * step, 3 * step, -10 * step, 0], np.float32))
    return groups


def pin_quantize_bruteforce(o):
    """Each code minimises |v - k*scale| over k in -7..7 (exact arithmetic),
    exact midpoints go to the even code, the scale is the fp32 nearest to
    a/7, and the largest magnitude maps to +-7."""
    rng = np.random.default_rng(12)
    for v in _quant_groups(rng):
        k, scale = o.quantize_group(v)
        a = np.float32(np.max(np.abs(v))) if v.size else np.float32(0)
        if a == 0 or np.float32(a / np.float32(7)) == 0:
            assert scale == 0 and not k.any(), (v, k, scale)
            continue
        _nearest_f32_check(Fraction(float(a)) / 7, scale)
        fs = Fraction(float(scale))
        for vj, kj in zip(v, k):
            q = Fraction(float(vj)) / fs
            cands = _exact_argmins(float(vj), float(scale))
            half = Fraction(2 * q).__floor__() / Fraction(2)
            near = [h for h in (half, half + Fraction(1, 2)) if h.denominator == 2]
            close = any(abs(q - h) <= Fraction(1, 2**19) for h in near)
            if len(cands) == 2:
                assert int(kj) == [c for c in cands if c % 2 == 0][0], (vj, scale, kj, cands)
            elif not close:
                assert int(kj) == cands[0], (vj, scale, kj, cands)
            else:
                assert int(kj) in (cands[0], cands[0] - 1, cands[0] + 1)
        imax = int(np.argmax(np.abs(v)))
        if scale >= np.finfo(np.float32).tiny:
            # a normal scale is a/7 to within half an ulp, so the largest
            # magnitude divides to 7 up to rounding (a subnormal scale is
            # coarser and may leave the maximum below 7)
            assert abs(int(k[imax])) == 7
        for vj, kj in zip(v, k):
            if abs(int(kj)) < 7:
                err = abs(Fraction(float(vj)) - int(kj) * fs)
                assert err <= fs / 2 * (1 + Fraction(1, 2**20)), (vj, kj, scale)


def pin_pack_layout(o):
    """Two codes per byte, element 2j in the low nibble, two's complement;
    unpack inverts pack for every pair of levels."""
    assert o.pack(np.array([1, -1], np.int8)).tolist() == [0xF1]
    assert o.pack(np.array([-8 + 1, 7], np.int8)).tolist() == [0x79]
    ks = np.array([(a, b) for a in range(-7, 8) for b in range(-7, 8)], np.int8).ravel()
    assert np.array_equal(o.unpack(o.pack(ks), ks.size), ks)


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line)
    return rows


def pin_golden_quantize(o):
    """Hand-worked single groups (tests/golden/quantize_worked.txt)."""
    for row in _read_golden("quantize_worked.txt"):
        vals, codes, scale, packed = [p.strip() for p in row.split("|")]
        v = np.array([float(t) for t in vals.split()], np.float32)
        k, sc = o.quantize_group(v)
        assert k.tolist() == [int(t) for t in codes.split()], (row, k)
        assert sc == np.float32(float.fromhex(scale)), (row, sc)
        assert o.pack(k).tolist() == [int(t, 16) for t in packed.split()], row


def pin_golden_call(o):
    """A hand-worked call of P=2 ranks, N=8, G=4 (tests/golden/call_worked.txt)."""
    spec = {}
    for row in _read_golden("call_worked.txt"):
        key, val = [p.strip() for p in row.split("=", 1)]
        spec[key] = val
    P, N, G = int(spec["P"]), int(spec["N"]), int(spec["G"])
    prm = _params(o, P, N, G, True)
    x = np.array([[float(t) for t in spec["x%d" % r].split()] for r in range(P)], np.float32)
    mf = np.zeros((P, N), np.float32)
    ms = np.zeros((P, N), np.float32)
    r = o.allreduce(prm, bf16_bits(x), mf, ms)
    y = bits_to_f64(r.y)
    assert y.tolist() == [float(t) for t in spec["y"].split()]
    for rr in range(P):
        assert r.codes[rr].tolist() == [int(t, 16) for t in spec["codes%d" % rr].split()]
        assert mf[rr].tolist() == [float.fromhex(t) for t in spec["m_fast%d" % rr].split()]
        assert ms[rr].tolist() == [float.fromhex(t) for t in spec["m_slow%d" % rr].split()]
    assert r.rcodes.tolist() == [int(t, 16) for t in spec["rcodes"].split()]


def pin_golden_sequence(o):
    """Two hand-worked calls on one state (tests/golden/sequence_worked.txt):
    the second starts from the first one's states, so the corrections, the
    partial update of a nonzero state and the owner fix-up are pinned by
    exact values."""
    spec = {}
    for row in _read_golden("sequence_worked.txt"):
        key, val = [p.strip() for p in row.split("=", 1)]
        spec[key] = val

    def vec(key, conv=float):
        return [conv(t) for t in spec[key].split()]

    P, N, G = int(spec["P"]), int(spec["N"]), int(spec["G"])
    prm = _params(o, P, N, G, True, alpha=float(spec["alpha"]),
                  beta_fast=float(spec["beta_fast"]), beta_slow=float(spec["beta_slow"]))
    mf = np.zeros((P, N), np.float32)
    ms = np.zeros((P, N), np.float32)
    hexbytes = lambda t: int(t, 16)    # noqa: E731
    for call in (1, 2):
        x = np.array([vec("x%d.%d" % (r, call)) for r in range(P)], np.float32)
        r = o.allreduce(prm, bf16_bits(x), mf, ms)
        assert bits_to_f64(r.y).tolist() == vec("y.%d" % call), call
        assert r.rcodes.tolist() == vec("rcodes.%d" % call, hexbytes), call
        for rr in range(P):
            assert r.codes[rr].tolist() == vec("codes%d.%d" % (rr, call), hexbytes), (call, rr)
            assert mf[rr].tolist() == vec("m_fast%d.%d" % (rr, call)), (call, rr)
            assert ms[rr].tolist() == vec("m_slow%d.%d" % (rr, call)), (call, rr)
        if call == 2:
            assert r.rscales.tolist() == vec("rscales.2")
            assert r.e_req.tolist() == vec("e_req.2")
            for rr in range(P):
                assert r.xt[rr].tolist() == vec("xt%d.2" % rr), rr
                assert r.scales[rr].tolist() == vec("scales%d.2" % rr), rr
                assert r.e_in[rr].tolist() == vec("e_in%d.2" % rr), rr


def pin_golden_sequence_padded(o):
    """The premise of the GPU's check against the hand-worked sequence: the
    fixture's 4-element groups, each padded with zeros to 32 elements, give
    the fixture's values at its elements and +0 (code 0) everywhere else."""
    spec = {}
    for row in _read_golden("sequence_worked.txt"):
        key, val = [p.strip() for p in row.split("=", 1)]
        spec[key] = val
    P, g, G = int(spec["P"]), int(spec["G"]), 32
    groups = int(spec["N"]) // g
    N = groups * G

    def spread(key):
        v = [float(t) for t in spec[key].split()]
        out = np.zeros(N)
        for c in range(groups):
            out[c * G:c * G + g] = v[c * g:(c + 1) * g]
        return out

    def spread_bytes(key):
        v = [int(t, 16) for t in spec[key].split()]
        out = np.zeros(N // 2, np.uint8)
        for c in range(groups):
            out[c * G // 2:c * G // 2 + g // 2] = v[c * g // 2:(c + 1) * g // 2]
        return out

    prm = _params(o, P, N, G, True, alpha=float(spec["alpha"]),
                  beta_fast=float(spec["beta_fast"]), beta_slow=float(spec["beta_slow"]))
    mf = np.zeros((P, N), np.float32)
    ms = np.zeros((P, N), np.float32)
    for call in (1, 2):
        x = np.stack([spread("x%d.%d" % (r, call)) for r in range(P)]).astype(np.float32)
        r = o.allreduce(prm, bf16_bits(x), mf, ms)
        assert np.array_equal(bits_to_f64(r.y), spread("y.%d" % call)), call
        assert np.array_equal(r.rcodes, spread_bytes("rcodes.%d" % call)), call
        for rr in range(P):
            assert np.array_equal(r.codes[rr], spread_bytes("codes%d.%d" % (rr, call)))
            for m, name in ((mf, "m_fast"), (ms, "m_slow")):
                want = spread("%s%d.%d" % (name, rr, call))
                assert np.array_equal(m[rr].astype(np.float64), want), (call, name, rr)
                assert not np.signbit(m[rr][want == 0]).any(), (call, name, rr)


def pin_golden_reduce_scatter(o):
    """A hand-worked reduce-scatter call with a sum that is not a bf16
    value, so the owner's residual is not zero
    (tests/golden/reduce_scatter_worked.txt)."""
    spec = {}
    for row in _read_golden("reduce_scatter_worked.txt"):
        key, val = [p.strip() for p in row.split("=", 1)]
        spec[key] = val

    def vec(key, conv=float):
        return [conv(t) for t in spec[key].split()]

    P, N, G = int(spec["P"]), int(spec["N"]), int(spec["G"])
    prm = _params(o, P, N, G, True, alpha=float(spec["alpha"]),
                  beta_fast=float(spec["beta_fast"]), beta_slow=float(spec["beta_slow"]))
    mf = np.zeros((P, N), np.float32)
    ms = np.zeros((P, N), np.float32)
    x = np.array([vec("x%d" % r) for r in range(P)], np.float32)
    r = o.reduce_scatter(prm, bf16_bits(x), mf, ms)
    assert r.s.tolist() == vec("s")
    assert bits_to_f64(r.y).tolist() == vec("y")
    assert r.e_req.tolist() == vec("e_req")
    for rr in range(P):
        assert r.codes[rr].tolist() == vec("codes%d" % rr, lambda t: int(t, 16)), rr
        assert r.scales[rr].tolist() == vec("scales%d" % rr), rr
        assert mf[rr].tolist() == vec("m_fast%d" % rr), rr
        assert ms[rr].tolist() == vec("m_slow%d" % rr), rr


# ---------------------------------------------------------------- invariants

def grid_exact_inputs(rng, P, N, G, L=7):
    """Inputs on the code grid whose sums stay on it (values k*2^e with
    every rank's group max |k| = L and |sum_r k_r| <= L, reaching L)."""
    assert G >= P
    x = np.zeros((P, N), np.float64)
    for c in range(N // G):
        e = int(rng.integers(-8, 8))
        pos = rng.permutation(G)
        special = pos[:P]
        k = np.zeros((P, G), np.int64)
        for j in pos[P:]:
            budget = L
            for r in rng.permutation(P):
                if budget == 0:
                    break
                v = int(rng.integers(-budget, budget + 1))
                k[r, j] = v
                budget -= abs(v)
        for r in range(P):
            k[r, special[r]] = L * int(rng.choice([-1, 1])) if r else L
        x[:, c * G:(c + 1) * G] = k * 2.0 ** e
    return x.astype(np.float32)


def pin_grid_exact(o):
    """Inputs on the int4 grid reduce exactly; errors and states stay 0."""
    rng = np.random.default_rng(13)
    for P, G in ((2, 32), (4, 32), (8, 64), (3, 16)):
        N = P * G * 3
        for comp in (True, False):
            prm = _params(o, P, N, G, comp)
            xs = [bf16_bits(grid_exact_inputs(rng, P, N, G)) for _ in range(4)]
            for x, (r, mf, ms) in zip(xs, _run_sequence(o, prm, xs)):
                exact = bits_to_f64(x).sum(axis=0)
                assert np.array_equal(bits_to_f64(r.y), exact)
                assert not r.e_in.any() and not r.e_req.any()
                if comp:
                    assert not mf.any() and not ms.any()


def pin_off_mode_composition(o):
    """Compensator off: y = bf16(deq(requant(sum_r deq(q(x_r))))) composed
    from the stand-alone group primitives."""
    rng = np.random.default_rng(14)
    P, G = 4, 32
    N = P * G * 2
    prm = _params(o, P, N, G, False)
    x = bf16_bits(rng.normal(0, 1, (P, N)))
    r = o.allreduce(prm, x, None, None)
    xf = o.bf16_to_f32(x)
    for c in range(N // G):
        sl = slice(c * G, (c + 1) * G)
        s = np.zeros(G, np.float32)
        for rr in range(P):
            k, sc = o.quantize_group(xf[rr, sl])
            s = (s + o.dequant(k, sc)).astype(np.float32)
        k2, sc2 = o.quantize_group(s)
        y = o.f32_to_bf16(o.dequant(k2, sc2))
        assert np.array_equal(y, r.y[sl])


def pin_two_quantizations(o):
    """Each value is quantized exactly twice per call for any P; at P=1 the
    requantization reproduces the entry codes."""
    rng = np.random.default_rng(15)
    for P in (1, 2, 3, 4, 8):
        G = 32
        N = P * G * 2
        prm = _params(o, P, N, G, True)
        x = bf16_bits(rng.normal(0, 1, (P, N)))
        mf = (rng.normal(0, 0.05, (P, N))).astype(np.float32)
        ms = mf.copy()
        r = o.allreduce(prm, x, mf, ms)
        assert (r.qcount == 2).all(), r.qcount
        if P == 1:
            assert np.array_equal(r.rcodes, r.codes[0])
            ulp = np.spacing(r.scales[0])
            assert (np.abs(r.rscales - r.scales[0]) <= ulp).all()


def pin_packed_ratio(o):
    """Transport bytes per bf16 byte: (1/2 + 4/G)/2 -- "nearly 4x" fewer."""
    for G, expect in ((32, 0.3125), (64, 0.28125), (128, 0.265625)):
        P, N = 2, 2 * G * 2
        prm = _params(o, P, N, G, False)
        r = o.allreduce(prm, np.zeros((P, N), np.uint16), None, None)
        ratio = (r.codes.nbytes + r.scales.nbytes) / (P * N * 2)
        assert ratio == expect and 0.25 < ratio < 0.32


def pin_residual_accounting(o):
    """Per call, the revealed errors add up to the call's output residual
    sum_r xt_r - y up to the fp32 rounding of the sum."""
    rng = np.random.default_rng(16)
    P, G = 4, 32
    N = P * G * 4
    prm = _params(o, P, N, G, True)
    mf = rng.normal(0, 0.05, (P, N)).astype(np.float32)
    ms = rng.normal(0, 0.05, (P, N)).astype(np.float32)
    x = bf16_bits(rng.normal(0, 1, (P, N)))
    r = o.allreduce(prm, x, mf, ms)
    own = _owner(prm, np.arange(N))
    revealed = r.e_in.astype(np.float64).sum(axis=0) + r.e_req
    resid = r.xt.astype(np.float64).sum(axis=0) - bits_to_f64(r.y)
    d = r.xt.astype(np.float64) - r.e_in  # dequantized entries (up to rounding)
    tol = 2.0 ** -23 * (P * np.abs(d).sum(axis=0) + np.abs(r.e_in).sum(axis=0)
                        + np.abs(r.e_req) + np.abs(r.xt).sum(axis=0))
    assert (np.abs(revealed - resid) <= tol + 1e-30).all()
    assert own.min() == 0 and own.max() == P - 1


def _sequence_inputs(rng, P, N, T, sigma=1.0):
    return [bf16_bits(rng.normal(0, sigma, (P, N))) for _ in range(T)]


def pin_telescoping(o):
    """Closed form of the dual-EMA compensator: with S_T the sum of the
    outputs and X_T the sum of all inputs over T calls,
    S_T - X_T = -sum_r [a*mf_r/(1-bf) + (1-a)*ms_r/(1-bs)], for every T."""
    rng = np.random.default_rng(17)
    cases = [(2, 32, DEFAULTS), (4, 32, DEFAULTS), (8, 64, DEFAULTS),
             (4, 32, dict(alpha=0.75, beta_fast=0.5, beta_slow=0.9)),
             (3, 16, dict(alpha=1.0, beta_fast=0.25, beta_slow=0.5))]
    for P, G, kw in cases:
        N = P * G * 2
        T = 20
        prm = _params(o, P, N, G, True, **kw)
        xs = _sequence_inputs(rng, P, N, T)
        a = np.float64(np.float32(kw["alpha"]))
        bf = np.float64(np.float32(kw["beta_fast"]))
        bs = np.float64(np.float32(kw["beta_slow"]))
        S = np.zeros(N)
        X = np.zeros(N)
        for t, (x, (r, mf, ms)) in enumerate(zip(xs, _run_sequence(o, prm, xs)), 1):
            S += bits_to_f64(r.y)
            X += bits_to_f64(x).sum(axis=0)
            rhs = -(a * mf.astype(np.float64) / (1 - bf)
                    + (1 - a) * ms.astype(np.float64) / (1 - bs)).sum(axis=0)
            tol = 64 * t * P * 2.0 ** -24 * (1 + np.abs(S))
            assert (np.abs((S - X) - rhs) <= tol).all(), np.abs((S - X) - rhs).max()
    # without compensation the same quantity is the plain sum of residuals,
    # which keeps growing
    P, G, N, T = 4, 32, 4 * 32 * 2, 20
    prm = _params(o, P, N, G, False)
    xs = _sequence_inputs(rng, P, N, T)
    S = np.zeros(N)
    X = np.zeros(N)
    mf = np.zeros((P, N), np.float32)
    for x in xs:
        r = o.allreduce(prm, x, None, None)
        S += bits_to_f64(r.y)
        X += bits_to_f64(x).sum(axis=0)
    assert np.sqrt(np.mean((S - X) ** 2)) > 0.1


def pin_classic_error_feedback(o):
    """beta=0, alpha=1 is textbook error feedback (state = last revealed
    error, correction = state); beta=1 freezes the states at 0 and the call
    is bit-identical to the uncompensated one."""
    rng = np.random.default_rng(18)
    P, G = 4, 32
    N = P * G * 2
    xs = _sequence_inputs(rng, P, N, 6)
    prm = _params(o, P, N, G, True, alpha=1.0, beta_fast=0.0, beta_slow=0.0)
    own = _owner(prm, np.arange(N))
    prev = np.zeros((P, N), np.float32)
    S = np.zeros(N)
    X = np.zeros(N)
    for x, (r, mf, ms) in zip(xs, _run_sequence(o, prm, xs)):
        xf = bits_to_f64(x)
        # the correction of this call is the previous state, unchanged
        assert np.array_equal(r.xt, xf.astype(np.float32) + prev)
        rho = r.e_in.astype(np.float64).copy()
        rho[own, np.arange(N)] += r.e_req
        assert np.array_equal(mf, rho.astype(np.float32))
        assert np.array_equal(mf, ms)
        prev = mf.copy()
        S += bits_to_f64(r.y)
        X += xf.sum(axis=0)
        assert np.allclose(S - X, -mf.astype(np.float64).sum(axis=0), atol=1e-4)
    prm1 = _params(o, P, N, G, True, alpha=0.5, beta_fast=1.0, beta_slow=1.0)
    prm0 = _params(o, P, N, G, False)
    for x, (r, mf, ms) in zip(xs, _run_sequence(o, prm1, xs)):
        r0 = o.allreduce(prm0, x, None, None)
        assert not mf.any() and not ms.any()
        assert np.array_equal(r.y, r0.y) and np.array_equal(r.codes, r0.codes)
        assert np.array_equal(r.rcodes, r0.rcodes)


def pin_ema_closed_form(o):
    """Per rank, m_T = sum_t (1-b)*b^(T-t)*rho_t, where rho is the entry
    error plus, for the owner of the chunk only, the requantization error."""
    rng = np.random.default_rng(19)
    for P, G, kw in ((4, 32, DEFAULTS), (2, 16, dict(alpha=0.25, beta_fast=0.75, beta_slow=0.9))):
        N = P * G * 2
        T = 10
        prm = _params(o, P, N, G, True, **kw)
        own = _owner(prm, np.arange(N))
        xs = _sequence_inputs(rng, P, N, T)
        bf = np.float64(np.float32(kw["beta_fast"]))
        bs = np.float64(np.float32(kw["beta_slow"]))
        rhos = []
        for x, (r, mf, ms) in zip(xs, _run_sequence(o, prm, xs)):
            rho = r.e_in.astype(np.float64).copy()
            rho[own, np.arange(N)] += r.e_req
            rhos.append(rho)
            Tn = len(rhos)
            cf = sum((1 - bf) * bf ** (Tn - 1 - t) * rhos[t] for t in range(Tn))
            cs = sum((1 - bs) * bs ** (Tn - 1 - t) * rhos[t] for t in range(Tn))
            scale = np.abs(np.stack(rhos)).max() + 1e-30
            assert np.allclose(mf, cf, rtol=1e-6, atol=1e-6 * scale), np.abs(mf - cf).max()
            assert np.allclose(ms, cs, rtol=1e-6, atol=1e-6 * scale), np.abs(ms - cs).max()


def pin_column_locality(o):
    """A call evaluated on a subset of group columns gives, byte for byte,
    the full call's values at those columns, across a sequence of calls."""
    rng = np.random.default_rng(20)
    P, G = 4, 32
    N = P * G * 6
    prm = _params(o, P, N, G, True)
    cols = np.array([0, 3, 7, 8, 13, 23], np.int64)
    idx = (cols[:, None] * G + np.arange(G)[None, :]).ravel()
    mf = np.zeros((P, N), np.float32)
    ms = np.zeros((P, N), np.float32)
    mfs = np.zeros((P, idx.size), np.float32)
    mss = np.zeros((P, idx.size), np.float32)
    for x in _sequence_inputs(rng, P, N, 5):
        full = o.allreduce(prm, x, mf, ms)
        sub = o.allreduce(prm, x[:, idx], mfs, mss, cols)
        assert np.array_equal(full.y[idx], sub.y)
        assert np.array_equal(full.e_req[idx], sub.e_req)
        assert np.array_equal(full.scales[:, cols], sub.scales)
        assert np.array_equal(full.rscales[cols], sub.rscales)
        cidx = (cols[:, None] * (G // 2) + np.arange(G // 2)[None, :]).ravel()
        assert np.array_equal(full.codes[:, cidx], sub.codes)
        assert np.array_equal(full.rcodes[cidx], sub.rcodes)
        assert np.array_equal(mf[:, idx], mfs) and np.array_equal(ms[:, idx], mss)


def pin_determinism(o):
    rng = np.random.default_rng(21)
    P, G = 3, 32
    N = P * G * 2
    prm = _params(o, P, N, G, True)
    xs = _sequence_inputs(rng, P, N, 3)
    a = _run_sequence(o, prm, xs)
    b = _run_sequence(o, prm, xs)
    for (ra, mfa, msa), (rb, mfb, msb) in zip(a, b):
        assert np.array_equal(ra.y, rb.y) and np.array_equal(ra.codes, rb.codes)
        assert np.array_equal(mfa, mfb) and np.array_equal(msa, msb)


# ---------------------------------------------------------------- 8-bit codes

def pin_quantize8_bruteforce(o):
    """8-bit codes: each code minimises |v - k*scale| over k in -127..127
    (exact arithmetic), exact midpoints go to the even code, the scale is the
    fp32 nearest to a/127, and the largest magnitude maps to +-127."""
    rng = np.random.default_rng(25)
    for trial in range(24):
        G = int(rng.choice([2, 4, 8]))
        kind = trial % 3
        if kind == 0:
            v = rng.normal(0, 1, G)
        elif kind == 1:
            e = int(rng.integers(-4, 4))
            v = (rng.integers(-127, 127, G) + 0.5) * 2.0 ** e
            v[rng.integers(0, G)] = 127.0 * 2.0 ** e
        else:
            v = rng.standard_t(3, G) * 100
        v = np.asarray(v, np.float32)
        k, scale = o.quantize_group_levels(v, 127)
        a = np.float32(np.max(np.abs(v)))
        _nearest_f32_check(Fraction(float(a)) / 127, scale)
        fs = Fraction(float(scale))
        for vj, kj in zip(v, k):
            errs = [(abs(Fraction(float(vj)) - c * fs), c) for c in range(-127, 128)]
            m = min(e for e, _ in errs)
            cands = [c for e, c in errs if e == m]
            q = Fraction(float(vj)) / fs
            near = abs(q - (q.__floor__() + Fraction(1, 2))) <= Fraction(1, 2**12)
            if len(cands) == 2:
                assert int(kj) == [c for c in cands if c % 2 == 0][0], (vj, kj, cands)
            elif not near:
                assert int(kj) == cands[0], (vj, kj, cands)
        assert abs(int(k[int(np.argmax(np.abs(v)))])) == 127


def pin_golden_quantize8(o):
    """Hand-worked 8-bit groups (tests/golden/quantize8_worked.txt)."""
    for row in _read_golden("quantize8_worked.txt"):
        vals, codes, scale, packed = [p.strip() for p in row.split("|")]
        v = np.array([float(t) for t in vals.split()], np.float32)
        k, sc = o.quantize_group_levels(v, 127)
        assert k.tolist() == [int(t) for t in codes.split()], (row, k)
        assert sc == np.float32(float.fromhex(scale)), (row, sc)
        assert k.view(np.uint8).tolist() == [int(t, 16) for t in packed.split()], row


def pin_8bit_calls(o):
    """8-bit plans: grid-exact inputs reduce exactly with zero states, each
    value is quantized twice, the transport is (1 + 4/G)/2 of bf16, codes
    are one byte each, and the telescoping identity holds."""
    rng = np.random.default_rng(26)
    for P, G in ((2, 32), (4, 64)):
        N = P * G * 2
        prm = _params(o, P, N, G, True, bits=8)
        xs = [bf16_bits(grid_exact_inputs(rng, P, N, G, L=127)) for _ in range(3)]
        for x, (r, mf, ms) in zip(xs, _run_sequence(o, prm, xs)):
            assert np.array_equal(bits_to_f64(r.y), bits_to_f64(x).sum(axis=0))
            assert not mf.any() and not ms.any()
            assert (r.qcount == 2).all()
            assert r.codes.shape == (P, N) and r.rcodes.shape == (N,)
            assert (r.codes.nbytes + r.scales.nbytes) / (P * N * 2) == (1 + 4 / G) / 2
    P, G = 4, 32
    N = P * G * 2
    prm = _params(o, P, N, G, True, bits=8)
    S = np.zeros(N)
    X = np.zeros(N)
    xs = _sequence_inputs(rng, P, N, 12)
    for t, (x, (r, mf, ms)) in enumerate(zip(xs, _run_sequence(o, prm, xs)), 1):
        S += bits_to_f64(r.y)
        X += bits_to_f64(x).sum(axis=0)
        rhs = -(0.5 * mf.astype(np.float64) / 0.5
                + 0.5 * ms.astype(np.float64) / (1 - np.float64(np.float32(0.95)))).sum(axis=0)
        assert (np.abs((S - X) - rhs) <= 64 * t * P * 2.0 ** -24 * (1 + np.abs(S))).all()
    # the transport bytes of a call are the quantizer's codes, one byte each
    prm0 = _params(o, P, N, G, False, bits=8)
    x0 = _sequence_inputs(rng, P, N, 1)[0]
    r0 = o.allreduce(prm0, x0, None, None)
    xf0 = o.bf16_to_f32(x0)
    for rank in range(P):
        for c in range(N // G):
            k, sc = o.quantize_group_levels(xf0[rank, c * G:(c + 1) * G], 127)
            assert np.array_equal(r0.codes[rank, c * G:(c + 1) * G], k.view(np.uint8))
            assert r0.scales[rank, c] == sc
    # 8-bit codes are finer than 4-bit ones: the output residual is smaller
    x = _sequence_inputs(rng, P, N, 1)[0]
    r4 = o.allreduce(_params(o, P, N, G, False), x, None, None)
    r8 = o.allreduce(_params(o, P, N, G, False, bits=8), x, None, None)
    ex = bits_to_f64(x).sum(axis=0)
    assert np.abs(bits_to_f64(r8.y) - ex).mean() < 0.2 * np.abs(bits_to_f64(r4.y) - ex).mean()


def pin_mixed_width_sequence(o):
    """One state across calls of both code widths (the serving policy's
    per-layer promotion): the telescoping identity and the EMA closed form
    hold over the mixed sequence, and every call's transport is that of its
    own width -- 8-bit calls reduce 8-bit grid-exact inputs exactly, 4-bit
    calls the 4-bit ones."""
    rng = np.random.default_rng(27)
    P, G = 4, 32
    N = P * G * 2
    widths = [8, 8, 8, 8, 4, 4, 4, 4, 8, 4, 8, 4, 8, 8, 4, 4]
    kw = DEFAULTS
    bf = np.float64(np.float32(kw["beta_fast"]))
    bs = np.float64(np.float32(kw["beta_slow"]))
    a = np.float64(np.float32(kw["alpha"]))
    own = _owner(_params(o, P, N, G, True), np.arange(N))
    mf = np.zeros((P, N), np.float32)
    ms = np.zeros((P, N), np.float32)
    S = np.zeros(N)
    X = np.zeros(N)
    rhos = []
    for t, bits in enumerate(widths, 1):
        prm = _params(o, P, N, G, True, bits=bits, **kw)
        x = _sequence_inputs(rng, P, N, 1)[0]
        r = o.allreduce(prm, x, mf, ms)
        assert r.codes.shape == (P, N * bits // 8) and (r.qcount == 2).all()
        S += bits_to_f64(r.y)
        X += bits_to_f64(x).sum(axis=0)
        rhs = -(a * mf.astype(np.float64) / (1 - bf)
                + (1 - a) * ms.astype(np.float64) / (1 - bs)).sum(axis=0)
        assert (np.abs((S - X) - rhs) <= 64 * t * P * 2.0 ** -24 * (1 + np.abs(S))).all()
        rho = r.e_in.astype(np.float64).copy()
        rho[own, np.arange(N)] += r.e_req
        rhos.append(rho)
        cf = sum((1 - bf) * bf ** (t - 1 - k) * rhos[k] for k in range(t))
        scale = np.abs(np.stack(rhos)).max() + 1e-30
        assert np.allclose(mf, cf, rtol=1e-6, atol=1e-6 * scale)
    for bits, L in ((8, 127), (4, 7)):
        prm = _params(o, P, N, G, True, bits=bits)
        x = bf16_bits(grid_exact_inputs(rng, P, N, G, L=L))
        z = np.zeros((P, N), np.float32)
        r = o.allreduce(prm, x, z, z.copy())
        assert np.array_equal(bits_to_f64(r.y), bits_to_f64(x).sum(axis=0))


# ---------------------------------------------------------------- reduce-scatter

def _run_rs_sequence(o, prm, xs):
    P, N = prm.P, prm.N
    mf = np.zeros((P, N), np.float32)
    ms = np.zeros((P, N), np.float32)
    out = []
    for x in xs:
        r = o.reduce_scatter(prm, x, mf, ms)
        out.append((r, mf.copy(), ms.copy()))
    return out


def pin_rs_quantized_once(o):
    """Reduce-scatter: each value is quantized once (at entry), and what the
    owner receives is its fp32 sum rounded to bf16 -- the all-reduce's sum
    for the same inputs and state."""
    rng = np.random.default_rng(22)
    for P in (1, 2, 4, 8):
        G = 32
        N = P * G * 2
        prm = _params(o, P, N, G, True)
        x = bf16_bits(rng.normal(0, 1, (P, N)))
        m0 = rng.normal(0, 0.05, (P, N)).astype(np.float32)
        a = o.allreduce(prm, x, m0.copy(), m0.copy())
        r = o.reduce_scatter(prm, x, m0.copy(), m0.copy())
        assert (r.qcount == 1).all()
        assert np.array_equal(r.codes, a.codes) and np.array_equal(r.scales, a.scales)
        assert np.array_equal(r.s.view(np.uint32), a.s.view(np.uint32))
        assert np.array_equal(r.y, bf16_bits(a.s))


def pin_rs_telescoping(o):
    """The telescoping identity holds for the reduce-scatter too, with y the
    values the owners receive and their bf16 rounding error as the revealed
    output residual."""
    rng = np.random.default_rng(23)
    for P, G, kw in ((4, 32, DEFAULTS), (2, 64, dict(alpha=0.75, beta_fast=0.5, beta_slow=0.9))):
        N = P * G * 2
        T = 16
        prm = _params(o, P, N, G, True, **kw)
        xs = _sequence_inputs(rng, P, N, T)
        a = np.float64(np.float32(kw["alpha"]))
        bf = np.float64(np.float32(kw["beta_fast"]))
        bs = np.float64(np.float32(kw["beta_slow"]))
        S = np.zeros(N)
        X = np.zeros(N)
        for t, (x, (r, mf, ms)) in enumerate(zip(xs, _run_rs_sequence(o, prm, xs)), 1):
            S += bits_to_f64(r.y)
            X += bits_to_f64(x).sum(axis=0)
            rhs = -(a * mf.astype(np.float64) / (1 - bf)
                    + (1 - a) * ms.astype(np.float64) / (1 - bs)).sum(axis=0)
            tol = 64 * t * P * 2.0 ** -24 * (1 + np.abs(S))
            assert (np.abs((S - X) - rhs) <= tol).all(), np.abs((S - X) - rhs).max()


def pin_rs_grid_exact(o):
    """Grid-exact inputs reduce-scatter exactly; the states stay 0."""
    rng = np.random.default_rng(24)
    for P, G in ((2, 32), (4, 64)):
        N = P * G * 3
        prm = _params(o, P, N, G, True)
        xs = [bf16_bits(grid_exact_inputs(rng, P, N, G)) for _ in range(3)]
        for x, (r, mf, ms) in zip(xs, _run_rs_sequence(o, prm, xs)):
            assert np.array_equal(bits_to_f64(r.y), bits_to_f64(x).sum(axis=0))
            assert not mf.any() and not ms.any()


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
