"""ctypes wrapper around the C oracle of Echo's all-reduce (echo_oracle.c).

TEST INFRASTRUCTURE ONLY: the oracle is what the CUDA path is checked
against.  Only the tests, the smoke check in ``__graft_entry__`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library
and its Python binding never import it.

Every function mirrors one step of the definition written in echo_oracle.c,
which cites the page passages it follows ("Echo: Error-Compensated 4-Bit
Tensor-Parallel Communication", ai4snews news summary "Interpretation"; the
arXiv abstract on the fugumt mirror).

``Oracle(path)`` binds one compiled copy of the C source; the module-level
functions use the default build next to this file.  The tests also compile
deliberately broken copies of the source to show that the pins catch them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "echo_oracle.c")
_LIB = os.path.join(_HERE, "libecho_oracle.so")

# Plain IEEE single precision: no contraction into FMA, no fast-math.
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c99", "-Wall",
          "-Wextra", "-fPIC", "-shared"]


def compile_source(src: str, out: str) -> str:
    """Compile a C source file of the oracle into a shared library."""
    tmp = out + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile echo_oracle.c into libecho_oracle.so next to it (gcc)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(SOURCE)):
        return _LIB
    return compile_source(SOURCE, _LIB)


class _Params(ctypes.Structure):
    _fields_ = [("P", ctypes.c_int32), ("G", ctypes.c_int32),
                ("N", ctypes.c_int64), ("compensate", ctypes.c_int32),
                ("alpha", ctypes.c_float), ("beta_fast", ctypes.c_float),
                ("beta_slow", ctypes.c_float), ("bits", ctypes.c_int32)]


@dataclass
class Params:
    """Parameters of one plan: P ranks, N elements per rank, group size G."""
    P: int
    N: int
    G: int
    compensate: bool = True
    alpha: float = 0.5
    beta_fast: float = 0.5
    beta_slow: float = 0.95
    bits: int = 4

    def c_struct(self) -> _Params:
        return _Params(self.P, self.G, self.N, int(bool(self.compensate)),
                       self.alpha, self.beta_fast, self.beta_slow, self.bits)


@dataclass
class CallResult:
    codes: np.ndarray    # [P, n/2] uint8, entry codes
    scales: np.ndarray   # [P, ncols] fp32, entry scales
    xt: np.ndarray       # [P, n] fp32, corrected input
    e_in: np.ndarray     # [P, n] fp32, entry error
    s: np.ndarray        # [n] fp32, reduce-scatter sum
    rcodes: np.ndarray   # [n/2] uint8, requantized sum
    rscales: np.ndarray  # [ncols] fp32
    e_req: np.ndarray    # [n] fp32, requantization error
    y: np.ndarray        # [n] uint16, bf16 bits every rank receives
    qcount: np.ndarray   # [n] int32, quantizations on each result's path


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """One compiled copy of the oracle's C source."""

    def __init__(self, path: str):
        self.path = path
        L = ctypes.CDLL(path)
        vp = ctypes.c_void_p
        L.eo_bf16_to_f32.restype = ctypes.c_float
        L.eo_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.eo_f32_to_bf16_rne.restype = ctypes.c_uint16
        L.eo_f32_to_bf16_rne.argtypes = [ctypes.c_float]
        L.eo_quantize_group.restype = None
        L.eo_quantize_group.argtypes = [vp, ctypes.c_int, vp, vp, vp]
        if hasattr(L, "eo_quantize_group_levels"):
            L.eo_quantize_group_levels.restype = None
            L.eo_quantize_group_levels.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, vp, vp]
        L.eo_dequant.restype = ctypes.c_float
        L.eo_dequant.argtypes = [ctypes.c_int8, ctypes.c_float]
        L.eo_pack.restype = None
        L.eo_pack.argtypes = [vp, ctypes.c_int64, vp]
        L.eo_unpack.restype = None
        L.eo_unpack.argtypes = [vp, ctypes.c_int64, vp]
        L.eo_allreduce.restype = ctypes.c_int
        L.eo_allreduce.argtypes = [ctypes.POINTER(_Params), ctypes.c_int64,
                                   vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                   vp, vp, vp, vp]
        self.has_rs = hasattr(L, "eo_reduce_scatter")
        if self.has_rs:
            L.eo_reduce_scatter.restype = ctypes.c_int
            L.eo_reduce_scatter.argtypes = [ctypes.POINTER(_Params), ctypes.c_int64,
                                            vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                            vp, vp]
        self.L = L

    # ------------------------------------------------------------ primitives
    def bf16_to_f32(self, bits) -> np.ndarray:
        """bf16 bit patterns (uint16) -> fp32, exact."""
        bits = np.asarray(bits, dtype=np.uint16)
        out = np.empty(bits.shape, np.float32)
        flat = out.reshape(-1)
        for i, b in enumerate(bits.reshape(-1)):
            flat[i] = self.L.eo_bf16_to_f32(int(b))
        return out

    def f32_to_bf16(self, x) -> np.ndarray:
        """fp32 -> bf16 bit patterns, round to nearest, ties to even."""
        x = np.asarray(x, dtype=np.float32)
        out = np.empty(x.shape, np.uint16)
        flat = out.reshape(-1)
        for i, v in enumerate(x.reshape(-1)):
            flat[i] = self.L.eo_f32_to_bf16_rne(float(v))
        return out

    def quantize_group(self, v, count=None):
        """Symmetric absmax int4 quantization of one group: (k, scale)."""
        v = np.ascontiguousarray(v, dtype=np.float32)
        k = np.zeros(v.size, dtype=np.int8)
        sc = np.zeros(1, dtype=np.float32)
        self.L.eo_quantize_group(_ptr(v), v.size, _ptr(k), _ptr(sc), _ptr(count))
        return k, np.float32(sc[0])

    def quantize_group_levels(self, v, levels: int, count=None):
        """Symmetric absmax quantization with `levels` levels per side."""
        v = np.ascontiguousarray(v, dtype=np.float32)
        k = np.zeros(v.size, dtype=np.int8)
        sc = np.zeros(1, dtype=np.float32)
        self.L.eo_quantize_group_levels(_ptr(v), v.size, levels, _ptr(k), _ptr(sc), _ptr(count))
        return k, np.float32(sc[0])

    def dequant(self, k, scale) -> np.ndarray:
        k = np.asarray(k, dtype=np.int8).ravel()
        return np.array([self.L.eo_dequant(int(c), float(scale)) for c in k],
                        dtype=np.float32)

    def pack(self, k) -> np.ndarray:
        k = np.ascontiguousarray(k, dtype=np.int8)
        assert k.size % 2 == 0
        out = np.zeros(k.size // 2, dtype=np.uint8)
        self.L.eo_pack(_ptr(k), k.size, _ptr(out))
        return out

    def unpack(self, b, n: int) -> np.ndarray:
        b = np.ascontiguousarray(b, dtype=np.uint8)
        assert b.size * 2 >= n and n % 2 == 0
        out = np.zeros(n, dtype=np.int8)
        self.L.eo_unpack(_ptr(b), n, _ptr(out))
        return out

    # ------------------------------------------------------------ one call
    def allreduce(self, prm: Params, x_bits: np.ndarray, m_fast, m_slow,
                  cols=None) -> CallResult:
        """One call on all group columns (cols=None) or on a list of them.

        x_bits: [P, n] uint16 bf16 bits, n = len(cols)*G (or N).  m_fast,
        m_slow: [P, n] float32 arrays, updated in place (ignored when the
        compensator is off).  Returns every intermediate of the call.
        """
        P, G = prm.P, prm.G
        if cols is None:
            ncols, cptr = prm.N // G, None
        else:
            cols = np.ascontiguousarray(cols, dtype=np.int64)
            ncols, cptr = cols.size, _ptr(cols)
        n = ncols * G
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        assert x_bits.shape == (P, n), (x_bits.shape, (P, n))
        if prm.compensate:
            for m in (m_fast, m_slow):
                assert m is not None and m.dtype == np.float32 and m.shape == (P, n)
                assert m.flags.c_contiguous
        cb = n * prm.bits // 8
        res = CallResult(
            codes=np.zeros((P, cb), np.uint8),
            scales=np.zeros((P, ncols), np.float32),
            xt=np.zeros((P, n), np.float32), e_in=np.zeros((P, n), np.float32),
            s=np.zeros(n, np.float32), rcodes=np.zeros(cb, np.uint8),
            rscales=np.zeros(ncols, np.float32), e_req=np.zeros(n, np.float32),
            y=np.zeros(n, np.uint16), qcount=np.zeros(n, np.int32))
        st = prm.c_struct()
        rc = self.L.eo_allreduce(
            ctypes.byref(st), ncols, cptr, _ptr(x_bits),
            _ptr(m_fast) if prm.compensate else None,
            _ptr(m_slow) if prm.compensate else None,
            _ptr(res.codes), _ptr(res.scales), _ptr(res.xt), _ptr(res.e_in),
            _ptr(res.s), _ptr(res.rcodes), _ptr(res.rscales), _ptr(res.e_req),
            _ptr(res.y), _ptr(res.qcount))
        if rc != 0:
            raise ValueError("oracle rejected the arguments (P=%d N=%d G=%d)"
                             % (P, prm.N, G))
        return res


    def reduce_scatter(self, prm: Params, x_bits: np.ndarray, m_fast, m_slow,
                       cols=None) -> CallResult:
        """One reduce-scatter call: y[i] (bf16 bits) is what the owner of
        element i's chunk receives; e_req holds the owner's output residual;
        rcodes and rscales are empty."""
        P, G = prm.P, prm.G
        if cols is None:
            ncols, cptr = prm.N // G, None
        else:
            cols = np.ascontiguousarray(cols, dtype=np.int64)
            ncols, cptr = cols.size, _ptr(cols)
        n = ncols * G
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        assert x_bits.shape == (P, n), (x_bits.shape, (P, n))
        if prm.compensate:
            for m in (m_fast, m_slow):
                assert m is not None and m.dtype == np.float32 and m.shape == (P, n)
                assert m.flags.c_contiguous
        res = CallResult(
            codes=np.zeros((P, n * prm.bits // 8), np.uint8),
            scales=np.zeros((P, ncols), np.float32),
            xt=np.zeros((P, n), np.float32), e_in=np.zeros((P, n), np.float32),
            s=np.zeros(n, np.float32), rcodes=np.zeros(0, np.uint8),
            rscales=np.zeros(0, np.float32), e_req=np.zeros(n, np.float32),
            y=np.zeros(n, np.uint16), qcount=np.zeros(n, np.int32))
        st = prm.c_struct()
        rc = self.L.eo_reduce_scatter(
            ctypes.byref(st), ncols, cptr, _ptr(x_bits),
            _ptr(m_fast) if prm.compensate else None,
            _ptr(m_slow) if prm.compensate else None,
            _ptr(res.codes), _ptr(res.scales), _ptr(res.xt), _ptr(res.e_in),
            _ptr(res.s), _ptr(res.e_req), _ptr(res.y), _ptr(res.qcount))
        if rc != 0:
            raise ValueError("oracle rejected the arguments (P=%d N=%d G=%d)"
                             % (P, prm.N, G))
        return res


def owner_of_columns(prm: Params, cols) -> np.ndarray:
    """Owner rank of each group column: floor(col*G / (N/P))."""
    return (np.asarray(cols, np.int64) * prm.G) // (prm.N // prm.P)


_default: Oracle | None = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def bf16_to_f32(bits):
    return default().bf16_to_f32(bits)


def f32_to_bf16(x):
    return default().f32_to_bf16(x)


def quantize_group(v, count=None):
    return default().quantize_group(v, count)


def dequant(k, scale):
    return default().dequant(k, scale)


def pack(k):
    return default().pack(k)


def unpack(b, n):
    return default().unpack(b, n)


def allreduce(prm, x_bits, m_fast, m_slow, cols=None):
    return default().allreduce(prm, x_bits, m_fast, m_slow, cols)


def reduce_scatter(prm, x_bits, m_fast, m_slow, cols=None):
    return default().reduce_scatter(prm, x_bits, m_fast, m_slow, cols)
