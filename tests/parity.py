"""GPU-vs-oracle comparison of whole calls and call sequences.

The CUDA path runs a call on the full tensors; the oracle runs the same
call on the same input bytes, on every group column or on a sample of
them (every quantity at an element depends only on its group column across
the ranks and on earlier calls at that column, so a sampled oracle run with
its own carried states is exact).  Every intermediate the library exposes
is compared: entry codes and scales, the requantized codes and scales, the
bf16 output of every rank, e_req and both EMA states.

Acceptance: integer/byte outputs (codes) and the fp32 scales bit-exact;
outputs, e_req and states are compared bit-exactly too, since both sides
evaluate the same fp32 operations in the same order.  On a mismatch the
message also says whether the looser acceptance (fp32 within 1e-6
relative, bf16 within 1 ulp) still holds.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from bit_error_compensated_echo_b200 import workloads
from bit_error_compensated_echo_b200.api import EchoPlan


def _bits_u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _f32(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().numpy()


def _u8(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().numpy()


def assert_same(name: str, got: np.ndarray, want: np.ndarray, kind: str, call: int):
    if got.shape != want.shape:
        raise AssertionError("%s (call %d): shape %s vs %s" % (name, call, got.shape, want.shape))
    if kind == "f32":
        same = np.array_equal(got.view(np.uint32), want.view(np.uint32)) or np.array_equal(got, want)
    else:
        same = np.array_equal(got, want)
    if same:
        return
    bad = np.argwhere(got != want)
    msg = "%s (call %d): %d of %d differ; first at %s: got %r want %r" % (
        name, call, len(bad), got.size, tuple(bad[0]), got[tuple(bad[0])], want[tuple(bad[0])])
    if kind == "f32":
        rel = np.abs(got.astype(np.float64) - want) / np.maximum(np.abs(want), 1e-30)
        msg += "; max rel diff %.3g" % rel.max()
    if kind == "bf16":
        ulps = np.abs(got.astype(np.int64) - want.astype(np.int64))
        msg += "; max bf16 ulp diff %d" % ulps.max()
    raise AssertionError(msg)


class SequenceChecker:
    """Runs calls on a GPU plan and on the oracle, comparing every call."""

    def __init__(self, plan: EchoPlan, prm: oracle.Params, cols=None):
        self.plan, self.prm = plan, prm
        P, N, G = prm.P, prm.N, prm.G
        if cols is None:
            self.cols = None
            self.idx = np.arange(N)
            self.gidx = np.arange(N // G)
        else:
            self.cols = np.asarray(cols, np.int64)
            self.idx = workloads.column_elements(self.cols, G)
            self.gidx = self.cols
        n = self.idx.size
        self.mf = np.zeros((P, n), np.float32)
        self.ms = np.zeros((P, n), np.float32)
        self.t_idx = torch.from_numpy(self.idx).to(plan.device)
        self.t_gidx = torch.from_numpy(self.gidx).to(plan.device)
        self._t_cidx = {}
        self.calls = 0

    def cidx(self, bits: int) -> torch.Tensor:
        """Byte indices of the sampled columns in a code row of this width."""
        if bits not in self._t_cidx:
            cb = self.prm.G * bits // 8          # code bytes per group
            if self.cols is None:
                c = np.arange(self.prm.N // self.prm.G * cb)
            else:
                c = workloads.column_elements(self.cols, cb)
            self._t_cidx[bits] = torch.from_numpy(c).to(self.plan.device)
        return self._t_cidx[bits]

    def _prm(self) -> oracle.Params:
        """The oracle's parameters for the plan's current code width."""
        if self.prm.bits == self.plan.bits:
            return self.prm
        import dataclasses
        return dataclasses.replace(self.prm, bits=self.plan.bits)

    def gather(self, t: torch.Tensor, which: str) -> torch.Tensor:
        ix = {"e": self.t_idx, "c": self.cidx(self.plan.bits), "g": self.t_gidx}[which]
        if self.cols is None:
            return t
        return t.index_select(t.dim() - 1, ix)

    def step(self, x: torch.Tensor, out: torch.Tensor | None = None, side_stream=None,
             check_states: bool = True, bits: int | None = None):
        """One call on x ([P, N] bf16 on the plan's device) and its check
        (bits: the call's code width, None for the plan's current one)."""
        out = self.plan.allreduce(x, out=out, side_stream=side_stream, bits=bits)
        return out, self.verify(x, out, check_states=check_states)

    def verify(self, x: torch.Tensor, out: torch.Tensor, check_states: bool = True):
        """Check an all-reduce call that was already made on the plan, on
        inputs x and outputs out ([P, N] bf16 on the plan's device), at the
        plan's current code width; the oracle's carried states advance by
        this call.  Returns the oracle's CallResult."""
        plan = self.plan
        prm = self._prm()
        torch.cuda.synchronize()
        call = self.calls
        self.calls += 1
        xb = _bits_u16(self.gather(x, "e"))
        ref = oracle.allreduce(prm, xb, self.mf, self.ms, self.cols)
        dv = plan.debug_view()
        assert_same("entry codes", _u8(self.gather(dv["codes"], "c")), ref.codes, "u8", call)
        assert_same("entry scales", _f32(self.gather(dv["scales"], "g")), ref.scales, "f32", call)
        assert_same("reduced codes", _u8(self.gather(dv["rcodes"], "c")), ref.rcodes, "u8", call)
        assert_same("reduced scales", _f32(self.gather(dv["rscales"], "g")), ref.rscales, "f32", call)
        ob = _bits_u16(self.gather(out, "e"))
        assert_same("outputs", ob, np.broadcast_to(ref.y, ob.shape), "bf16", call)
        if prm.compensate:
            if plan.fixup != "exit":   # in exit mode e_req is folded in the reduce, not stored
                assert_same("e_req", _f32(self.gather(dv["e_req"], "e")), ref.e_req, "f32",
                            call)
            if check_states:
                if dv["fixup_pending"]:
                    mf, ms = plan.get_state()
                else:
                    mf, ms = dv["m_fast"], dv["m_slow"]
                assert_same("m_fast", _f32(self.gather(mf, "e")), self.mf, "f32", call)
                assert_same("m_slow", _f32(self.gather(ms, "e")), self.ms, "f32", call)
                del mf, ms
        return ref


def oracle_params(plan: EchoPlan) -> oracle.Params:
    c = plan.cfg
    return oracle.Params(P=c.P, N=c.N, G=c.G, compensate=bool(c.compensate), alpha=c.alpha,
                         beta_fast=c.beta_fast, beta_slow=c.beta_slow, bits=c.bits)


class RSChecker(SequenceChecker):
    """The same comparison for reduce-scatter calls (and, through
    step_allreduce, all-reduce calls on the same plan and state)."""

    def step_rs(self, x: torch.Tensor, side_stream=None, bits: int | None = None):
        plan = self.plan
        out = plan.reduce_scatter(x, side_stream=side_stream, bits=bits)
        prm = self._prm()
        torch.cuda.synchronize()
        call = self.calls
        self.calls += 1
        xb = _bits_u16(self.gather(x, "e"))
        ref = oracle.reduce_scatter(prm, xb, self.mf, self.ms, self.cols)
        dv = plan.debug_view()
        assert_same("entry codes", _u8(self.gather(dv["codes"], "c")), ref.codes, "u8", call)
        assert_same("entry scales", _f32(self.gather(dv["scales"], "g")), ref.scales, "f32", call)
        C = prm.N // prm.P
        owner = torch.from_numpy(self.idx // C).to(plan.device)
        local = torch.from_numpy(self.idx % C).to(plan.device)
        got = out[owner, local]
        assert_same("owner outputs", _bits_u16(got), ref.y, "bf16", call)
        if prm.compensate:
            if plan.fixup != "exit":
                assert_same("output residual", _f32(self.gather(dv["e_req"], "e")), ref.e_req,
                            "f32", call)
            mf, ms = plan.get_state()
            assert_same("m_fast", _f32(self.gather(mf, "e")), self.mf, "f32", call)
            assert_same("m_slow", _f32(self.gather(ms, "e")), self.ms, "f32", call)
        return out, ref
