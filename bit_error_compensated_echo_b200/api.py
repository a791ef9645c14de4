"""Torch-facing wrapper over the C ABI: checks tensors and passes pointers.

PyTorch supplies device memory and streams only; every step of the
all-reduce runs in the library's CUDA kernels (``abi`` forwards to them).
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import abi


class _DeviceArray:
    """Zero-copy view of plan-owned device memory for torch.as_tensor."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {
            "shape": tuple(shape), "typestr": typestr, "data": (ptr, False),
            "version": 3, "strides": None}


def _stream_handle(stream: Optional[torch.cuda.Stream], device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream)


def make_config(P: int, N: int, G: int, compensate: bool, alpha: float, beta_fast: float,
                beta_slow: float, device: int, fixup: str, bits: int) -> abi.echo_config:
    """The echo_config of include/echo.h for these parameters."""
    cfg = abi.echo_config_default()
    cfg.P, cfg.N, cfg.G = int(P), int(N), int(G)
    cfg.compensate = int(bool(compensate))
    cfg.alpha, cfg.beta_fast, cfg.beta_slow = alpha, beta_fast, beta_slow
    cfg.device = int(device)
    if fixup not in abi.FIXUP_MODES:
        raise ValueError("fixup must be one of %s" % sorted(abi.FIXUP_MODES))
    cfg.fixup = abi.FIXUP_MODES[fixup]
    cfg.bits = int(bits)
    return cfg


class EchoPlan:
    """A plan for P virtual ranks of N bf16 elements each, group size G.

    Owns the compensator state (two fp32 EMAs per rank) and the workspace;
    ``allreduce`` runs one call of the error-compensated 4-bit all-reduce.
    """

    def __init__(self, P: int, N: int, G: int = 128, compensate: bool = True,
                 alpha: float = 0.5, beta_fast: float = 0.5, beta_slow: float = 0.95,
                 device: Optional[int] = None, fixup: str = "exit", bits: int = 4):
        if device is None:
            device = torch.cuda.current_device()
        cfg = make_config(P, N, G, compensate, alpha, beta_fast, beta_slow, device, fixup, bits)
        self.cfg = cfg
        self.max_bits = int(bits)   # the transport is sized for this width
        self.bits = int(bits)       # width of the following calls
        self.P, self.N, self.G = int(P), int(N), int(G)
        self.compensate = bool(compensate)
        self.fixup = fixup
        self.device = torch.device("cuda", int(device))
        self.handle = abi.echo_plan_create(cfg)

    # ------------------------------------------------------------ lifetime
    def close(self) -> None:
        if getattr(self, "handle", None):
            abi.echo_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # ------------------------------------------------------------ checks
    def _rank_tensors(self, xs, what: str) -> Sequence[torch.Tensor]:
        if isinstance(xs, torch.Tensor):
            if xs.dim() < 1 or xs.shape[0] != self.P:
                raise ValueError("%s: expected leading dim P=%d" % (what, self.P))
            xs = list(xs.unbind(0))
        if len(xs) != self.P:
            raise ValueError("%s: expected %d tensors" % (what, self.P))
        for t in xs:
            if t.dtype != torch.bfloat16 or t.numel() != self.N or not t.is_contiguous():
                raise ValueError("%s: each rank needs a contiguous bf16 tensor of %d elements"
                                 % (what, self.N))
        return xs

    # ------------------------------------------------------------ calls
    def set_bits(self, bits: int) -> None:
        """Code width of the following calls (4, or 8 if the plan was made
        with bits=8); every width shares the plan's one state."""
        abi.echo_plan_set_bits(self.handle, bits)
        self.bits = int(bits)

    def _width(self, bits: Optional[int]) -> None:
        if bits is not None and int(bits) != self.bits:
            self.set_bits(bits)

    def allreduce(self, xs, out=None, stream: Optional[torch.cuda.Stream] = None,
                  side_stream: Optional[torch.cuda.Stream] = None, bits: Optional[int] = None):
        """One call.  xs: [P, N] bf16 tensor or P tensors on the plan's
        device.  out: same form (allocated if None; may be xs for in place).
        bits: code width of this call and the following ones (None: keep).
        Returns out."""
        self._width(bits)
        xs_l = self._rank_tensors(xs, "inputs")
        if out is None:
            out = torch.empty((self.P, self.N), dtype=torch.bfloat16, device=self.device)
        out_l = self._rank_tensors(out, "outputs")
        for t in list(xs_l) + list(out_l):
            if t.device != self.device:
                raise ValueError("tensors must live on %s" % self.device)
        side = int(side_stream.cuda_stream) if side_stream is not None else 0
        abi.echo_allreduce(self.handle, [t.data_ptr() for t in xs_l],
                           [t.data_ptr() for t in out_l],
                           _stream_handle(stream, self.device), side)
        return out

    def reduce_scatter(self, xs, out=None, stream: Optional[torch.cuda.Stream] = None,
                       side_stream: Optional[torch.cuda.Stream] = None,
                       bits: Optional[int] = None):
        """One reduce-scatter call.  xs: [P, N] bf16 (or P tensors); out:
        [P, N/P] bf16 (allocated if None), row r = rank r's own chunk of the
        sum.  Returns out."""
        self._width(bits)
        xs_l = self._rank_tensors(xs, "inputs")
        C = self.N // self.P
        if out is None:
            out = torch.empty((self.P, C), dtype=torch.bfloat16, device=self.device)
        out_l = list(out.unbind(0)) if isinstance(out, torch.Tensor) else list(out)
        if len(out_l) != self.P or any(t.dtype != torch.bfloat16 or t.numel() != C
                                       or not t.is_contiguous() or t.device != self.device
                                       for t in out_l):
            raise ValueError("outputs: P contiguous bf16 tensors of N/P elements on the device")
        for t in xs_l:
            if t.device != self.device:
                raise ValueError("tensors must live on %s" % self.device)
        side = int(side_stream.cuda_stream) if side_stream is not None else 0
        abi.echo_reduce_scatter(self.handle, [t.data_ptr() for t in xs_l],
                                [t.data_ptr() for t in out_l],
                                _stream_handle(stream, self.device), side)
        return out

    def allreduce_host(self, xs_host, out_host=None, stream: Optional[torch.cuda.Stream] = None,
                       bits: Optional[int] = None):
        """The same call on host tensors (pinned for asynchronous copies);
        the caller synchronizes the stream before reading out_host."""
        self._width(bits)
        xs_l = self._rank_tensors(xs_host, "host inputs")
        if out_host is None:
            out_host = torch.empty((self.P, self.N), dtype=torch.bfloat16, pin_memory=True)
        out_l = self._rank_tensors(out_host, "host outputs")
        for t in list(xs_l) + list(out_l):
            if t.device.type != "cpu":
                raise ValueError("allreduce_host takes host tensors")
        abi.echo_allreduce_host(self.handle, [t.data_ptr() for t in xs_l],
                                [t.data_ptr() for t in out_l],
                                _stream_handle(stream, self.device))
        return out_host

    def reset_state(self, stream=None) -> None:
        abi.echo_reset_state(self.handle, _stream_handle(stream, self.device))

    def get_state(self, stream=None):
        """(m_fast, m_slow) as new [P, N] fp32 tensors (pending fix-up applied;
        in deferred mode e_req is -0, a no-op, when none is pending)."""
        mf = torch.empty((self.P, self.N), dtype=torch.float32, device=self.device)
        ms = torch.empty_like(mf)
        abi.echo_get_state(self.handle, mf.data_ptr(), ms.data_ptr(),
                           _stream_handle(stream, self.device))
        return mf, ms

    def set_state(self, m_fast: torch.Tensor, m_slow: torch.Tensor, stream=None) -> None:
        for m in (m_fast, m_slow):
            if (m.dtype != torch.float32 or m.numel() != self.P * self.N
                    or not m.is_contiguous() or m.device != self.device):
                raise ValueError("state must be a contiguous fp32 [P, N] tensor on the device")
        abi.echo_set_state(self.handle, m_fast.data_ptr(), m_slow.data_ptr(),
                           _stream_handle(stream, self.device))

    def debug_view(self) -> dict:
        """Zero-copy tensors over the plan's workspace (valid while the plan
        lives; contents as left by the last call)."""
        v = abi.echo_debug_view_get(self.handle)
        P, N, G, bits = self.P, self.N, self.G, v.bits

        def t(ptr, shape, typestr):
            if not ptr:
                return None
            return torch.as_tensor(_DeviceArray(ptr, shape, typestr), device=self.device)

        return {
            "m_fast": t(v.m_fast, (P, N), "<f4"), "m_slow": t(v.m_slow, (P, N), "<f4"),
            "codes": t(v.codes, (P, N * bits // 8), "|u1"),
            "scales": t(v.scales, (P, N // G), "<f4"),
            "rcodes": t(v.rcodes, (N * bits // 8,), "|u1"),
            "rscales": t(v.rscales, (N // G,), "<f4"),
            "e_req": t(v.e_req, (N,), "<f4"), "fixup_pending": bool(v.fixup_pending),
            "guard": t(v.guard, (int(v.guard_bytes),), "|u1"),
        }

    def profile_enable(self, on: bool = True) -> None:
        abi.echo_profile_enable(self.handle, on)

    def profile_read(self, reset: bool = False) -> dict:
        p = abi.echo_profile_read(self.handle, reset)
        return {k: getattr(p, k) for k, _ in abi.echo_profile._fields_}

    def launches_per_call(self) -> int:
        return abi.echo_launches_per_call(self.handle)

    def workspace_bytes(self) -> int:
        return abi.echo_workspace_bytes(self.cfg)
