"""One rank of an Echo group spread over processes, one GPU each.

The pages' setting is a tensor-parallel group of GPUs whose all-reduce moves
4-bit integers and sums them in high precision (ai4snews news summary,
"Interpretation"; arXiv abstract).  ``EchoRankPlan`` runs this rank's part
of it: the library's kernels (include/echo_rank.h) do every arithmetic
step, and the two exchange steps between them -- an all-to-all of the packed
entry chunks and an all-gather of the owners' reduced chunks -- go through a
transport, by default ``torch.distributed`` (NCCL between GPUs).  Only
packed codes and fp32 group scales cross between ranks: C*bits/8 + 4*C/G
bytes per chunk of C = N/P elements, against 2*C for a bf16 all-reduce.

Run by every rank of a group with the same parameters, a call gives every
rank the output that ``EchoPlan.allreduce`` gives P virtual ranks on one
GPU, and leaves each rank the state of its virtual counterpart, bit for bit.
"""
from __future__ import annotations

import datetime
import os
from typing import List, Optional, Sequence

import torch
import torch.distributed as dist

from . import abi
from .api import _stream_handle, make_config


def process_group_options(backend: str, local_rank: int) -> dict:
    """Extra keyword arguments of torch.distributed.init_process_group for a
    process driving GPU ``local_rank``: an NCCL group is bound to that GPU
    (device_id), so that NCCL never guesses the device from the global rank
    -- a guess that is wrong whenever ranks and GPUs are numbered
    differently, and then hangs the group's first collective."""
    if backend == "nccl":
        return {"device_id": torch.device("cuda", int(local_rank))}
    return {}


def init_process_group(backend: Optional[str] = None, timeout_s: float = 120.0, **kw) -> int:
    """Join the process group of the launch (RANK, WORLD_SIZE, MASTER_* and
    LOCAL_RANK from the environment, or rank/world_size in kw) with a short
    timeout; with NCCL the process first makes its GPU, LOCAL_RANK, current
    and binds the group to it.  Returns the local rank."""
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    if backend == "nccl":
        torch.cuda.set_device(local)
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s),
                            **process_group_options(backend, local), **kw)
    return local


class TorchDistTransport:
    """The two exchange steps over a torch.distributed process group.

    all_to_all(recv, send): equal splits -- part o of ``send`` goes to rank o
    and part r of ``recv`` comes from rank r.  all_gather(out, inp): part o
    of ``out`` is rank o's ``inp``.  Both are ordered with the current CUDA
    stream by torch.distributed (the collectives wait for the work queued on
    it, and later work on it waits for them)."""

    def __init__(self, group=None):
        self.group = group

    def all_to_all(self, recv: torch.Tensor, send: torch.Tensor) -> None:
        dist.all_to_all_single(recv, send, group=self.group)

    def all_gather(self, out: torch.Tensor, inp: torch.Tensor) -> None:
        dist.all_gather_into_tensor(out, inp, group=self.group)


class ExchangeBuffers:
    """The exchange buffers of one rank (layouts: include/echo_rank.h).

    With cb code bytes and cs scales per chunk:
      send_codes [P*cb] u8, send_scales [P*cs] f32 : chunk o for rank o
      recv_codes [P*cb] u8, recv_scales [P*cs] f32 : rank r's copy of this chunk
      red_codes  [cb] u8,   red_scales  [cs] f32   : this rank's reduced chunk
      all_codes  [P*cb] u8, all_scales  [P*cs] f32 : owner o's reduced chunk

    The code buffers are allocated for ``chunk_code_bytes`` (the widest
    width) and viewed at the width in force (``set_code_bytes``).
    """

    def __init__(self, P: int, chunk_code_bytes: int, chunk_scale_bytes: int, device):
        cb, cs = int(chunk_code_bytes), int(chunk_scale_bytes) // 4
        u8, f32 = torch.uint8, torch.float32
        self.P, self.cb_max, self.cs = int(P), cb, cs
        self._codes = {k: torch.empty(P * cb if k != "red" else cb, dtype=u8, device=device)
                       for k in ("send", "recv", "red", "all")}
        self.send_scales = torch.empty(P * cs, dtype=f32, device=device)
        self.recv_scales = torch.empty(P * cs, dtype=f32, device=device)
        self.red_scales = torch.empty(cs, dtype=f32, device=device)
        self.all_scales = torch.empty(P * cs, dtype=f32, device=device)
        self.set_code_bytes(cb)

    def set_code_bytes(self, cb: int) -> None:
        """View the code buffers for chunks of cb bytes (cb <= the allocated
        size): chunk o then starts at o*cb."""
        if cb > self.cb_max:
            raise ValueError("chunk of %d code bytes exceeds the %d allocated" % (cb, self.cb_max))
        P, self.cb = self.P, int(cb)
        self.send_codes = self._codes["send"][:P * cb]
        self.recv_codes = self._codes["recv"][:P * cb]
        self.red_codes = self._codes["red"][:cb]
        self.all_codes = self._codes["all"][:P * cb]

    def wire_bytes(self) -> int:
        """Bytes this rank sends per all-reduce: (P-1) chunks in the
        all-to-all and its reduced chunk to P-1 ranks in the all-gather."""
        chunk = self.cb + 4 * self.cs
        return 2 * (self.P - 1) * chunk


class TorchDistBarrier:
    """The stream-ordered barrier of the fused transport: a one-element
    all-reduce on the current stream, which completes on a rank only after
    every rank's earlier work on its stream."""

    def __init__(self, device, group=None):
        self.group = group
        self.flag = torch.zeros(1, dtype=torch.int32, device=device)

    def __call__(self) -> None:
        dist.all_reduce(self.flag, group=self.group)


def _offsets(layout: dict) -> dict:
    return {k: v for k, v in layout.items() if k != "base"}


class PeerWindows:
    """Every rank's window as mapped in this process (include/echo_rank.h,
    "Fused transport over peer memory").

    bases[o] is the base address of rank o's window here (this rank's own
    allocation for o == rank); the byte offsets of the four buffers are the
    same on every rank of a group (same config).  The pointer tables of the
    fused stage calls follow from the two.

    Teardown, on every rank: synchronize the stream, barrier the group,
    ``close()`` (unmaps the peers' windows), barrier again, and only then
    destroy the plan (which frees this rank's window): no rank may still
    read a window that is unmapped or freed."""

    def __init__(self, plan: "EchoRankPlan", bases: Sequence[int], layout: dict,
                 opened: Sequence[int] = ()):
        if len(bases) != plan.P:
            raise ValueError("one window base per rank")
        self.rank, self.P, self.device = plan.rank, plan.P, plan.device
        self.bases = [int(b) for b in bases]
        self.layout = dict(layout)
        self._opened = list(opened)

    def _at(self, key: str) -> List[int]:
        off = self.layout[key]
        return [b + off for b in self.bases]

    # tables over the P ranks, and this rank's own buffers
    def recv_codes_peers(self) -> List[int]:
        return self._at("recv_codes")

    def recv_scales_peers(self) -> List[int]:
        return self._at("recv_scales")

    def red_codes_peers(self) -> List[int]:
        return self._at("red_codes")

    def red_scales_peers(self) -> List[int]:
        return self._at("red_scales")

    def own(self, key: str) -> int:
        return self.bases[self.rank] + self.layout[key]

    @classmethod
    def exchange(cls, plan: "EchoRankPlan", group=None) -> "PeerWindows":
        """Run by every rank of the group: share the windows' CUDA IPC
        handles and map the other ranks' windows into this process."""
        layout = abi.echo_rank_window(plan.handle)
        mine = (plan.rank, abi.echo_ipc_handle_get(layout["base"]), layout)
        got = [None] * plan.P
        dist.all_gather_object(got, mine, group=group)
        bases, opened = [], []
        try:
            for o, (r, handle, lay) in enumerate(got):
                if r != o or _offsets(lay) != _offsets(layout):
                    raise RuntimeError("rank %d: window layouts differ across the group" % o)
                if o == plan.rank:
                    bases.append(layout["base"])
                else:
                    b = abi.echo_ipc_open(handle, plan.device.index)
                    opened.append(b)
                    bases.append(b)
        except Exception:
            for b in opened:
                abi.echo_ipc_close(b, plan.device.index)
            raise
        return cls(plan, bases, layout, opened)

    @classmethod
    def in_process(cls, plans: Sequence["EchoRankPlan"]) -> List["PeerWindows"]:
        """Every rank's plan in this one process (one device): each rank's
        tables point straight at the other plans' windows, no IPC."""
        layouts = [abi.echo_rank_window(p.handle) for p in plans]
        bases = [lay["base"] for lay in layouts]
        return [cls(p, bases, layouts[0]) for p in plans]

    def close(self) -> None:
        """Unmap the peers' windows (this rank's own stays with its plan)."""
        opened, self._opened = self._opened, []
        for b in opened:
            abi.echo_ipc_close(b, self.device.index)


def exchange(bufs: ExchangeBuffers, transport) -> None:
    """The reduce-scatter exchange: every rank's chunk o to rank o."""
    transport.all_to_all(bufs.recv_codes, bufs.send_codes)
    transport.all_to_all(bufs.recv_scales, bufs.send_scales)


def gather(bufs: ExchangeBuffers, transport) -> None:
    """The all-gather exchange: every owner's reduced chunk to every rank."""
    transport.all_gather(bufs.all_codes, bufs.red_codes)
    transport.all_gather(bufs.all_scales, bufs.red_scales)


class EchoRankPlan:
    """Rank ``rank`` of a group of P ranks, N bf16 elements per rank.

    Owns this rank's compensator state (two fp32 EMAs of N elements) and
    its exchange buffers.  The stage methods (entry, reduce, exit,
    reduce_scatter_finish) are the library calls; ``allreduce`` and
    ``reduce_scatter`` put the transport's exchanges between them.
    """

    def __init__(self, P: int, rank: int, N: int, G: int = 128, compensate: bool = True,
                 alpha: float = 0.5, beta_fast: float = 0.5, beta_slow: float = 0.95,
                 device: Optional[int] = None, fixup: str = "deferred", bits: int = 4):
        if device is None:
            device = torch.cuda.current_device()
        self.cfg = make_config(P, N, G, compensate, alpha, beta_fast, beta_slow, device, fixup,
                               bits)
        self.P, self.rank, self.N, self.G, self.bits = int(P), int(rank), int(N), int(G), int(bits)
        self.max_bits = int(bits)
        self.compensate = bool(compensate)
        self.fixup = fixup
        self.device = torch.device("cuda", int(device))
        cb, sb = abi.echo_rank_exchange_bytes(self.cfg)
        self.handle = abi.echo_rank_plan_create(self.cfg, self.rank)
        self.bufs = ExchangeBuffers(self.P, cb, sb, self.device)

    # ------------------------------------------------------------ lifetime
    def close(self) -> None:
        if getattr(self, "handle", None):
            abi.echo_rank_plan_destroy(self.handle)
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

    def set_bits(self, bits: int) -> None:
        """Code width of the following calls (4, or 8 if the plan was made
        with bits=8), one state for every width.  Every rank of the group
        must use the same width for a call."""
        abi.echo_rank_plan_set_bits(self.handle, bits)
        self.bits = int(bits)
        self.bufs.set_code_bytes(self.N // self.P * self.bits // 8)

    # ------------------------------------------------------------ checks
    def _check_bf16(self, t: torch.Tensor, n: int, what: str) -> None:
        if (t.dtype != torch.bfloat16 or t.numel() != n or not t.is_contiguous()
                or t.device != self.device):
            raise ValueError("%s: a contiguous bf16 tensor of %d elements on %s"
                             % (what, n, self.device))

    def _st(self, stream) -> int:
        return _stream_handle(stream, self.device)

    # ------------------------------------------------------------ stages
    def entry(self, x: torch.Tensor, stream=None) -> None:
        """Correction, quantization of every chunk, partial EMA update:
        writes bufs.send_codes / bufs.send_scales."""
        self._check_bf16(x, self.N, "input")
        b = self.bufs
        abi.echo_rank_entry(self.handle, x.data_ptr(), b.send_codes.data_ptr(),
                            b.send_scales.data_ptr(), self._st(stream))

    def reduce(self, stream=None, side_stream=None) -> None:
        """Sum of the received chunks, requantization: writes
        bufs.red_codes / bufs.red_scales (and the owner fix-up by mode)."""
        b = self.bufs
        side = int(side_stream.cuda_stream) if side_stream is not None else 0
        abi.echo_rank_reduce(self.handle, b.recv_codes.data_ptr(), b.recv_scales.data_ptr(),
                             b.red_codes.data_ptr(), b.red_scales.data_ptr(), self._st(stream),
                             side)

    def exit(self, out: torch.Tensor, stream=None) -> None:
        """Dequantization of the gathered chunks into out (N bf16)."""
        self._check_bf16(out, self.N, "output")
        b = self.bufs
        abi.echo_rank_exit(self.handle, b.all_codes.data_ptr(), b.all_scales.data_ptr(),
                           out.data_ptr(), self._st(stream))

    def reduce_scatter_finish(self, out: torch.Tensor, stream=None, side_stream=None) -> None:
        """bf16 sum of this rank's chunk from the received chunks into out."""
        self._check_bf16(out, self.N // self.P, "output")
        b = self.bufs
        side = int(side_stream.cuda_stream) if side_stream is not None else 0
        abi.echo_rank_reduce_scatter(self.handle, b.recv_codes.data_ptr(),
                                     b.recv_scales.data_ptr(), out.data_ptr(),
                                     self._st(stream), side)

    # ------------------------------------------------------------ calls
    def allreduce(self, x: torch.Tensor, transport=None, out: Optional[torch.Tensor] = None,
                  side_stream=None, bits: Optional[int] = None) -> torch.Tensor:
        """One compensated all-reduce of this rank's x ([N] bf16) with the
        other ranks of the group, on the current stream.  out may be x.
        bits: code width of this call and the following ones (None: keep)."""
        if bits is not None and int(bits) != self.bits:
            self.set_bits(bits)
        transport = transport if transport is not None else TorchDistTransport()
        if out is None:
            out = torch.empty(self.N, dtype=torch.bfloat16, device=self.device)
        self.entry(x)
        exchange(self.bufs, transport)
        self.reduce(side_stream=side_stream)
        gather(self.bufs, transport)
        self.exit(out)
        return out

    def reduce_scatter(self, x: torch.Tensor, transport=None, out: Optional[torch.Tensor] = None,
                       side_stream=None, bits: Optional[int] = None) -> torch.Tensor:
        """The reduce-scatter of sequence parallelism: returns this rank's
        chunk (N/P bf16) of the sum."""
        if bits is not None and int(bits) != self.bits:
            self.set_bits(bits)
        transport = transport if transport is not None else TorchDistTransport()
        if out is None:
            out = torch.empty(self.N // self.P, dtype=torch.bfloat16, device=self.device)
        self.entry(x)
        exchange(self.bufs, transport)
        self.reduce_scatter_finish(out, side_stream=side_stream)
        return out

    # ------------------------------------------------------------ fused transport
    def _check_win(self, win: PeerWindows) -> None:
        if win.rank != self.rank or win.P != self.P or win.device != self.device:
            raise ValueError("the windows were mapped for rank %d of %d on %s, not for this "
                             "plan (rank %d of %d on %s)" % (win.rank, win.P, win.device,
                                                             self.rank, self.P, self.device))

    def entry_peers(self, x: torch.Tensor, win: PeerWindows, stream=None) -> None:
        """Steps 1-3, chunk o stored straight into rank o's receive buffers."""
        self._check_win(win)
        self._check_bf16(x, self.N, "input")
        abi.echo_rank_entry_peers(self.handle, x.data_ptr(), win.recv_codes_peers(),
                                  win.recv_scales_peers(), self._st(stream))

    def reduce_window(self, win: PeerWindows, stream=None, side_stream=None) -> None:
        """Steps 4-5 from this rank's receive buffers into its reduced
        buffers (both in its window)."""
        self._check_win(win)
        side = int(side_stream.cuda_stream) if side_stream is not None else 0
        abi.echo_rank_reduce(self.handle, win.own("recv_codes"), win.own("recv_scales"),
                             win.own("red_codes"), win.own("red_scales"), self._st(stream), side)

    def exit_peers(self, win: PeerWindows, out: torch.Tensor, stream=None) -> None:
        """Step 6, owner o's reduced chunk loaded straight from owner o."""
        self._check_win(win)
        self._check_bf16(out, self.N, "output")
        abi.echo_rank_exit_peers(self.handle, win.red_codes_peers(), win.red_scales_peers(),
                                 out.data_ptr(), self._st(stream))

    def allreduce_peers(self, x: torch.Tensor, win: PeerWindows, barrier,
                        out: Optional[torch.Tensor] = None, side_stream=None,
                        bits: Optional[int] = None) -> torch.Tensor:
        """The all-reduce over the fused transport: entry_peers, barrier,
        reduce, barrier, exit_peers (include/echo_rank.h).  barrier: a
        stream-ordered barrier of the group (TorchDistBarrier)."""
        if bits is not None and int(bits) != self.bits:
            self.set_bits(bits)
        if out is None:
            out = torch.empty(self.N, dtype=torch.bfloat16, device=self.device)
        self.entry_peers(x, win)
        barrier()
        self.reduce_window(win, side_stream=side_stream)
        barrier()
        self.exit_peers(win, out)
        return out

    def reduce_scatter_peers(self, x: torch.Tensor, win: PeerWindows, barrier,
                             out: Optional[torch.Tensor] = None, side_stream=None,
                             bits: Optional[int] = None) -> torch.Tensor:
        """The reduce-scatter over the fused transport: entry_peers, barrier,
        the owner's bf16 sum from its receive buffers, barrier."""
        if bits is not None and int(bits) != self.bits:
            self.set_bits(bits)
        if out is None:
            out = torch.empty(self.N // self.P, dtype=torch.bfloat16, device=self.device)
        self.entry_peers(x, win)
        barrier()
        self.reduce_scatter_peers_finish(win, out, side_stream=side_stream)
        barrier()
        return out

    def reduce_scatter_peers_finish(self, win: PeerWindows, out: torch.Tensor, stream=None,
                                    side_stream=None) -> None:
        """bf16 sum of this rank's chunk from its receive buffers into out."""
        self._check_win(win)
        self._check_bf16(out, self.N // self.P, "output")
        side = int(side_stream.cuda_stream) if side_stream is not None else 0
        abi.echo_rank_reduce_scatter(self.handle, win.own("recv_codes"), win.own("recv_scales"),
                                     out.data_ptr(), self._st(stream), side)

    # ------------------------------------------------------------ state
    def reset_state(self, stream=None) -> None:
        abi.echo_rank_reset_state(self.handle, self._st(stream))

    def get_state(self, stream=None):
        """(m_fast, m_slow) of this rank as new [N] fp32 tensors."""
        mf = torch.empty(self.N, dtype=torch.float32, device=self.device)
        ms = torch.empty_like(mf)
        abi.echo_rank_get_state(self.handle, mf.data_ptr(), ms.data_ptr(), self._st(stream))
        return mf, ms

    def set_state(self, m_fast: torch.Tensor, m_slow: torch.Tensor, stream=None) -> None:
        for m in (m_fast, m_slow):
            if (m.dtype != torch.float32 or m.numel() != self.N or not m.is_contiguous()
                    or m.device != self.device):
                raise ValueError("state: a contiguous fp32 tensor of N elements on the device")
        abi.echo_rank_set_state(self.handle, m_fast.data_ptr(), m_slow.data_ptr(),
                                self._st(stream))

    def launches_per_call(self) -> int:
        return abi.echo_rank_launches_per_call(self.handle)

    def workspace_bytes(self) -> int:
        return abi.echo_rank_workspace_bytes(self.cfg)
