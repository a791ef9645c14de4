"""Host logic of the rank path's fused transport on the CPU (no CUDA).

1. ``PeerWindows.exchange`` over gloo ranks (2 and 3 processes), with the
   library's window and IPC calls replaced by fakes that record what they
   are given: every rank maps every other rank's window from that rank's
   own handle, never opens its own, builds its pointer tables from the
   bases and the shared offsets, and ``close`` unmaps exactly what it
   mapped.  A group whose window layouts differ is refused on every rank,
   with nothing left mapped.
2. ``allreduce_peers`` and ``reduce_scatter_peers`` put the stages and the
   barriers in the order include/echo_rank.h requires.
"""
import os
import socket

import pytest
import torch

from bit_error_compensated_echo_b200 import rank as rank_mod
from bit_error_compensated_echo_b200.rank import EchoRankPlan, PeerWindows

OFFS = {"recv_codes": 0, "recv_scales": 4096, "red_codes": 8192, "red_scales": 12288}
MAPPED = 1 << 44                # where the fake IPC maps a peer's window


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _base_of(rank):
    return (rank + 1) << 32


class _FakePlan:
    def __init__(self, P, rank):
        self.P, self.rank, self.handle = P, rank, 1000 + rank
        self.device = torch.device("cuda", 0)


def _install_fakes(rank, bad_layout, log):
    lay = dict(OFFS, base=_base_of(rank), bytes=16384)
    if bad_layout and rank == 1:
        lay["red_scales"] += 256

    def window(handle):
        assert handle == 1000 + rank
        return dict(lay)

    def handle_get(ptr):
        assert ptr == _base_of(rank)
        return ptr.to_bytes(8, "little") + bytes(56)

    def ipc_open(handle, device):
        base = int.from_bytes(handle[:8], "little")
        assert base != _base_of(rank), "a rank opened its own window"
        log.append(("open", base))
        return MAPPED + base

    def ipc_close(ptr, device):
        log.append(("close", ptr))

    rank_mod.abi.echo_rank_window = window
    rank_mod.abi.echo_ipc_handle_get = handle_get
    rank_mod.abi.echo_ipc_open = ipc_open
    rank_mod.abi.echo_ipc_close = ipc_close


def _exchange_main(rank, ws, port, bad_layout, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    log = []
    try:
        _install_fakes(rank, bad_layout, log)
        try:
            win = PeerWindows.exchange(_FakePlan(ws, rank))
        except RuntimeError as e:
            q.put((rank, "refused", str(e), list(log)))
            return
        tables = (win.bases, win.recv_codes_peers(), win.recv_scales_peers(),
                  win.red_codes_peers(), win.red_scales_peers(), win.own("recv_codes"))
        opened = list(log)
        win.close()
        win.close()                                    # a second close unmaps nothing
        q.put((rank, "ok", tables, opened, log[len(opened):]))
    finally:
        dist.destroy_process_group()


def _run(ws, bad_layout):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_exchange_main, args=(r, ws, port, bad_layout, q))
             for r in range(ws)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(ws):
        item = q.get(timeout=120)
        got[item[0]] = item[1:]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    return got


@pytest.mark.parametrize("ws", [2, 3])
def test_exchange_maps_every_peer_window(ws):
    got = _run(ws, bad_layout=False)
    for r in range(ws):
        status, tables, opened, closed = got[r]
        assert status == "ok"
        bases, rc, rs, dc, ds, own = tables
        want = [_base_of(o) if o == r else MAPPED + _base_of(o) for o in range(ws)]
        assert bases == want, r
        assert rc == [b + OFFS["recv_codes"] for b in want]
        assert rs == [b + OFFS["recv_scales"] for b in want]
        assert dc == [b + OFFS["red_codes"] for b in want]
        assert ds == [b + OFFS["red_scales"] for b in want]
        assert own == _base_of(r) + OFFS["recv_codes"]
        assert opened == [("open", _base_of(o)) for o in range(ws) if o != r]
        assert sorted(closed) == sorted(("close", MAPPED + _base_of(o))
                                        for o in range(ws) if o != r)


def test_exchange_refuses_differing_layouts():
    got = _run(3, bad_layout=True)
    for r in range(3):
        status, msg, log = got[r]
        assert status == "refused" and "layouts differ" in msg, r
        opened = [b for op, b in log if op == "open"]
        closed = [b - MAPPED for op, b in log if op == "close"]
        assert sorted(opened) == sorted(closed), r   # nothing left mapped


class _OrderPlan(EchoRankPlan):
    """EchoRankPlan whose stages only record their order."""

    def __init__(self, log):
        self.log, self.P, self.N, self.bits = log, 2, 64, 4
        self.device = torch.device("cpu")
        self.handle = None

    def entry_peers(self, x, win, stream=None):
        self.log.append("entry_peers")

    def reduce_window(self, win, stream=None, side_stream=None):
        self.log.append("reduce")

    def exit_peers(self, win, out, stream=None):
        self.log.append("exit_peers")

    def reduce_scatter_peers_finish(self, win, out, stream=None, side_stream=None):
        self.log.append("reduce_scatter")


def test_fused_calls_order_stages_and_barriers():
    log = []
    plan = _OrderPlan(log)
    x = torch.zeros(64, dtype=torch.bfloat16)
    plan.allreduce_peers(x, None, lambda: log.append("barrier"),
                         out=torch.empty(64, dtype=torch.bfloat16))
    assert log == ["entry_peers", "barrier", "reduce", "barrier", "exit_peers"]
    log.clear()
    plan.reduce_scatter_peers(x, None, lambda: log.append("barrier"),
                              out=torch.empty(32, dtype=torch.bfloat16))
    assert log == ["entry_peers", "barrier", "reduce_scatter", "barrier"]
