"""The rank path's exchanges on the CPU, with gloo ranks (2 and 3 processes).

1. The transport: after ``exchange`` and ``gather`` over torch.distributed,
   every rank's receive buffers hold what the layout of include/echo_rank.h
   says (part r of recv = rank r's send part o at rank o; part o of all =
   owner o's reduced chunk), compared with the lockstep copies the GPU
   tests use for their single-process group.
2. The orchestration: ``EchoRankPlan.allreduce`` and ``reduce_scatter``
   with the library stages replaced by byte-level stand-ins (no CUDA) put
   the exchanges between the right stages: the stand-ins make the call an
   exact all-reduce of bytes modulo 256, which the test checks.
"""
import os
import socket

import pytest
import torch

from bit_error_compensated_echo_b200.rank import (EchoRankPlan, ExchangeBuffers,
                                                  TorchDistTransport, exchange, gather)

CB, CS = 48, 3          # code bytes and scales per chunk in these tests


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _send_for(rank, P):
    g = torch.Generator().manual_seed(1000 + rank)
    codes = torch.randint(0, 256, (P * CB,), generator=g, dtype=torch.uint8)
    scales = torch.randn(P * CS, generator=g)
    red_codes = torch.randint(0, 256, (CB,), generator=g, dtype=torch.uint8)
    red_scales = torch.randn(CS, generator=g)
    return codes, scales, red_codes, red_scales


def _transport_main(rank, ws, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        b = ExchangeBuffers(ws, CB, 4 * CS, "cpu")
        codes, scales, rc, rs = _send_for(rank, ws)
        b.send_codes.copy_(codes)
        b.send_scales.copy_(scales)
        b.red_codes.copy_(rc)
        b.red_scales.copy_(rs)
        t = TorchDistTransport()
        exchange(b, t)
        gather(b, t)
        # numpy copies travel by value: a tensor would be fetched from this
        # process, which may have exited by the time the parent reads it
        q.put((rank, b.recv_codes.numpy().copy(), b.recv_scales.numpy().copy(),
               b.all_codes.numpy().copy(), b.all_scales.numpy().copy()))
    finally:
        dist.destroy_process_group()


class _Bufs:
    """Stand-in for a rank plan, holding only exchange buffers, for the
    lockstep copies of tests/rank_emulation.py."""

    def __init__(self, b):
        self.bufs = b


@pytest.mark.parametrize("ws", [2, 3])
def test_transport_matches_the_buffer_layout(ws):
    import torch.multiprocessing as mp

    import rank_emulation
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_transport_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(ws):
        r, *bufs = q.get(timeout=120)
        got[r] = [torch.from_numpy(a) for a in bufs]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0

    # the same exchanges as lockstep copies
    emul = []
    for r in range(ws):
        b = ExchangeBuffers(ws, CB, 4 * CS, "cpu")
        codes, scales, rc, rs = _send_for(r, ws)
        b.send_codes.copy_(codes)
        b.send_scales.copy_(scales)
        b.red_codes.copy_(rc)
        b.red_scales.copy_(rs)
        emul.append(_Bufs(b))
    rank_emulation.all_to_all(emul)
    rank_emulation.all_gather(emul)
    for r in range(ws):
        want = emul[r].bufs
        for g, w in zip(got[r], (want.recv_codes, want.recv_scales, want.all_codes,
                                 want.all_scales)):
            assert torch.equal(g, w), r
    # and spelled out for one part: rank 1's part 0 of recv is rank 0's part 1 of send
    assert torch.equal(got[1][0][:CB], _send_for(0, ws)[0][CB:2 * CB])


class ByteStagePlan(EchoRankPlan):
    """EchoRankPlan whose stages are byte-level stand-ins on CPU buffers:
    entry copies chunk o of x (uint8) into send part o; reduce sums the P
    received parts modulo 256; exit concatenates the gathered parts.  The
    scales carry the rank index through the same exchanges."""

    def __init__(self, P, rank, C):
        self.P, self.rank, self.N = P, rank, P * C
        self.bufs = ExchangeBuffers(P, C, 4, "cpu")
        self.handle = None

    def entry(self, x, stream=None):
        self.bufs.send_codes.copy_(x)
        self.bufs.send_scales.fill_(float(self.rank))

    def reduce(self, stream=None, side_stream=None):
        b = self.bufs
        parts = b.recv_codes.view(self.P, b.cb).to(torch.int64)
        b.red_codes.copy_((parts.sum(0) % 256).to(torch.uint8))
        b.red_scales.copy_(b.recv_scales.sum().reshape(1))

    def exit(self, out, stream=None):
        out.copy_(self.bufs.all_codes)

    def reduce_scatter_finish(self, out, stream=None, side_stream=None):
        parts = self.bufs.recv_codes.view(self.P, self.bufs.cb).to(torch.int64)
        out.copy_((parts.sum(0) % 256).to(torch.uint8))


def _x_for(rank, N):
    g = torch.Generator().manual_seed(77 + rank)
    return torch.randint(0, 256, (N,), generator=g, dtype=torch.uint8)


def _orchestration_main(rank, ws, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        C = 40
        plan = ByteStagePlan(ws, rank, C)
        x = _x_for(rank, ws * C)
        y = plan.allreduce(x, TorchDistTransport(), out=torch.empty(ws * C, dtype=torch.uint8))
        scales = plan.bufs.all_scales.clone()
        z = plan.reduce_scatter(x, TorchDistTransport(), out=torch.empty(C, dtype=torch.uint8))
        q.put((rank, y.numpy().copy(), scales.numpy().copy(), z.numpy().copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws", [2, 3])
def test_allreduce_orchestration_with_byte_stages(ws):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_orchestration_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(ws):
        r, y, scales, z = q.get(timeout=120)
        got[r] = (torch.from_numpy(y), torch.from_numpy(scales), torch.from_numpy(z))
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    C = 40
    total = sum(_x_for(r, ws * C).to(torch.int64) for r in range(ws)) % 256
    rank_sum = float(sum(range(ws)))
    for r in range(ws):
        y, scales, z = got[r]
        assert torch.equal(y.to(torch.int64), total), r
        assert torch.equal(scales, torch.full((ws,), rank_sum)), r
        assert torch.equal(z.to(torch.int64), total[r * C:(r + 1) * C]), r


def _bind_main(rank, ws, port, q):
    import torch.distributed as dist

    import bench
    from bit_error_compensated_echo_b200 import rank as rank_mod
    # ranks and local ranks numbered differently: rank r drives GPU ws-1-r
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(ws - 1 - rank))
    got_ws, got_rank, local = bench.dist_setup()
    try:
        opts = rank_mod.process_group_options("nccl", local)
        locals_ = [None] * ws
        dist.all_gather_object(locals_, local)
        q.put((rank, got_ws, got_rank, local, str(opts["device_id"]), locals_,
               dist.get_backend()))
    finally:
        dist.destroy_process_group()


def test_process_group_binds_each_rank_to_its_local_device():
    """World size 2 over gloo, launched as the bench's ranks are (RANK,
    WORLD_SIZE, LOCAL_RANK from the environment), with ranks and GPUs
    numbered differently: each rank joins as its RANK, keeps its LOCAL_RANK,
    and an NCCL group would be bound to cuda:LOCAL_RANK, not cuda:RANK."""
    import torch.multiprocessing as mp
    ws = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bind_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(ws):
        item = q.get(timeout=120)
        got[item[0]] = item[1:]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    for r in range(ws):
        got_ws, got_rank, local, dev, locals_, backend = got[r]
        assert (got_ws, got_rank, local) == (ws, r, ws - 1 - r)
        assert dev == "cuda:%d" % (ws - 1 - r)
        assert locals_ == [ws - 1 - q_ for q_ in range(ws)]
        assert backend == "gloo"


def test_nccl_group_is_bound_to_the_local_gpu(monkeypatch):
    """The NCCL path of init_process_group, with fakes for the two calls it
    makes: the process's GPU (LOCAL_RANK) is made current and passed as
    device_id."""
    from bit_error_compensated_echo_b200 import rank as rank_mod
    seen = {}
    monkeypatch.setenv("LOCAL_RANK", "3")
    monkeypatch.setattr(rank_mod.torch.cuda, "set_device", lambda d: seen.setdefault("dev", d))
    monkeypatch.setattr(rank_mod.dist, "init_process_group",
                        lambda **kw: seen.setdefault("kw", kw))
    assert rank_mod.init_process_group("nccl", timeout_s=5.0) == 3
    assert seen["dev"] == 3
    assert seen["kw"]["backend"] == "nccl"
    assert seen["kw"]["device_id"] == torch.device("cuda", 3)
    assert seen["kw"]["timeout"].total_seconds() == 5.0
    assert rank_mod.process_group_options("gloo", 3) == {}
