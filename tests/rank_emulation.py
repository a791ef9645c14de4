"""P rank plans driven in lockstep inside one process (one GPU).

The two exchanges of a group are done here with plain tensor copies that
restate the buffer layouts of include/echo_rank.h: after the all-to-all,
rank o's recv part r is rank r's send part o; after the all-gather, every
rank's all part o is owner o's reduced chunk.  No kernel waits on another:
each stage runs for every rank before the next stage starts.
"""
from __future__ import annotations

from typing import List, Optional

import torch

from bit_error_compensated_echo_b200.rank import EchoRankPlan, PeerWindows


def _part(t: torch.Tensor, i: int, size: int) -> torch.Tensor:
    return t[i * size:(i + 1) * size]


def all_to_all(plans: List[EchoRankPlan]) -> None:
    P = len(plans)
    cb, cs = plans[0].bufs.cb, plans[0].bufs.cs
    for o in range(P):
        for r in range(P):
            _part(plans[o].bufs.recv_codes, r, cb).copy_(_part(plans[r].bufs.send_codes, o, cb))
            _part(plans[o].bufs.recv_scales, r, cs).copy_(_part(plans[r].bufs.send_scales, o, cs))


def all_gather(plans: List[EchoRankPlan]) -> None:
    P = len(plans)
    cb, cs = plans[0].bufs.cb, plans[0].bufs.cs
    for r in range(P):
        for o in range(P):
            _part(plans[r].bufs.all_codes, o, cb).copy_(plans[o].bufs.red_codes)
            _part(plans[r].bufs.all_scales, o, cs).copy_(plans[o].bufs.red_scales)


class EmulatedGroup:
    """P EchoRankPlan objects (ranks 0..P-1) on one device."""

    def __init__(self, P: int, N: int, G: int, device: int = 0, **kw):
        self.P, self.N, self.G = P, N, G
        self.plans = [EchoRankPlan(P, r, N, G, device=device, **kw) for r in range(P)]

    def close(self):
        for p in self.plans:
            p.close()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def allreduce(self, xs: torch.Tensor, side_stream: Optional[torch.cuda.Stream] = None):
        """xs: [P, N] bf16; returns [P, N] bf16, row r = rank r's output."""
        out = torch.empty_like(xs)
        for r, p in enumerate(self.plans):
            p.entry(xs[r])
        all_to_all(self.plans)
        for p in self.plans:
            p.reduce(side_stream=side_stream)
        all_gather(self.plans)
        for r, p in enumerate(self.plans):
            p.exit(out[r])
        return out

    def reduce_scatter(self, xs: torch.Tensor, side_stream: Optional[torch.cuda.Stream] = None):
        """xs: [P, N] bf16; returns [P, N/P] bf16, row r = rank r's chunk."""
        out = torch.empty((self.P, self.N // self.P), dtype=xs.dtype, device=xs.device)
        for r, p in enumerate(self.plans):
            p.entry(xs[r])
        all_to_all(self.plans)
        for r, p in enumerate(self.plans):
            p.reduce_scatter_finish(out[r], side_stream=side_stream)
        return out

    def get_state(self):
        """(m_fast, m_slow) as [P, N] fp32, row r = rank r's state."""
        mf, ms = zip(*(p.get_state() for p in self.plans))
        return torch.stack(mf), torch.stack(ms)


class EmulatedPeerGroup(EmulatedGroup):
    """The same P rank plans on the fused transport: each rank's entry
    stores into the other plans' windows and its exit loads from them
    (PeerWindows.in_process).  The stages still run rank by rank, each stage
    for every rank before the next, so the barrier of a real group is the
    stream order here and no kernel waits on another."""

    def __init__(self, P: int, N: int, G: int, device: int = 0, **kw):
        super().__init__(P, N, G, device=device, **kw)
        self.wins = PeerWindows.in_process(self.plans)

    def allreduce(self, xs: torch.Tensor, side_stream: Optional[torch.cuda.Stream] = None):
        out = torch.empty_like(xs)
        for r, (p, w) in enumerate(zip(self.plans, self.wins)):
            p.entry_peers(xs[r], w)
        for p, w in zip(self.plans, self.wins):
            p.reduce_window(w, side_stream=side_stream)
        for r, (p, w) in enumerate(zip(self.plans, self.wins)):
            p.exit_peers(w, out[r])
        return out

    def reduce_scatter(self, xs: torch.Tensor, side_stream: Optional[torch.cuda.Stream] = None):
        out = torch.empty((self.P, self.N // self.P), dtype=xs.dtype, device=xs.device)
        for r, (p, w) in enumerate(zip(self.plans, self.wins)):
            p.entry_peers(xs[r], w)
        for r, (p, w) in enumerate(zip(self.plans, self.wins)):
            p.reduce_scatter_peers_finish(w, out[r], side_stream=side_stream)
        return out
