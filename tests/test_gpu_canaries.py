"""Guard canaries around every caller buffer, and after the plan's own
workspace (the stand-in for a memory checker, which is closed here).

Each buffer the library reads or writes on the caller's side -- inputs,
outputs, the caller-owned state of the allocation-free call, host buffers of
the pipelined call, the rank path's exchange buffers -- is carved out of one
allocation between guard zones of at least 4 KiB filled with a byte
pattern.  After calls of every kind on ragged shapes (owner chunks that end
in a partial block), the guards must be intact, inputs unchanged (unless the
call runs in place), and the results equal to the same calls on plain
buffers."""
import pytest
import torch

from bit_error_compensated_echo_b200 import abi
from bit_error_compensated_echo_b200 import workloads as W
from bit_error_compensated_echo_b200.api import EchoPlan, make_config
from bit_error_compensated_echo_b200.rank import EchoRankPlan
from rank_emulation import EmulatedGroup

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
GUARD = 4096
PATTERN = 0xA5


class Guarded:
    """Buffers of the given byte sizes in one allocation, each 256-byte
    aligned, with >= GUARD pattern bytes before, between and after them."""

    def __init__(self, sizes, device=DEV, pin=False):
        self.spans = []
        off = GUARD
        for n in sizes:
            self.spans.append((off, n))
            off += (n + 255) // 256 * 256 + GUARD
        if device == "cpu":
            self.mem = torch.full((off,), PATTERN, dtype=torch.uint8, pin_memory=pin)
        else:
            self.mem = torch.full((off,), PATTERN, dtype=torch.uint8, device=device)

    def view(self, i, dtype, shape):
        off, n = self.spans[i]
        t = self.mem[off:off + n].view(dtype)
        return t.view(shape)

    def check(self, what):
        torch.cuda.synchronize()
        mask = torch.ones(self.mem.numel(), dtype=torch.bool, device=self.mem.device)
        for off, n in self.spans:
            mask[off:off + n] = False
        bad = (self.mem[mask] != PATTERN).nonzero()
        assert bad.numel() == 0, "%s: %d guard bytes changed" % (what, bad.numel())


def _bits(t):
    return t.contiguous().view(torch.uint8)


def _plan_guard_intact(plan: EchoPlan, what: str):
    """The guard zone after the plan's own workspace (include/echo.h)."""
    torch.cuda.synchronize()
    g = plan.debug_view()["guard"]
    assert g.numel() == 4096
    assert bool((g == PATTERN).all()), "%s: the plan's workspace guard changed" % what


CASES = [(2, 32, 37, 4), (3, 64, 5, 4), (8, 128, 3, 4), (4, 32, 11, 8), (8, 128, 2, 8)]


@pytest.mark.parametrize("P,G,k,bits", CASES, ids=lambda v: str(v))
@pytest.mark.parametrize("comp,fixup", [(True, "exit"), (True, "deferred"), (True, "side"),
                                        (False, "exit")])
def test_device_calls_keep_guards(P, G, k, bits, comp, fixup):
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    C = N // P
    side = torch.cuda.Stream() if fixup == "side" else None
    kw = dict(compensate=comp, fixup=fixup, bits=bits, device=0)
    g = Guarded([2 * N] * P + [2 * N] * P + [2 * C] * P)
    xs = [g.view(r, torch.bfloat16, (N,)) for r in range(P)]
    ys = [g.view(P + r, torch.bfloat16, (N,)) for r in range(P)]
    zs = [g.view(2 * P + r, torch.bfloat16, (C,)) for r in range(P)]
    with EchoPlan(P, N, G, **kw) as gp, EchoPlan(P, N, G, **kw) as ref:
        for t, op in enumerate("AARAI"):
            x = W.generate(w, t, DEV)
            for r in range(P):
                xs[r].copy_(x[r])
            if op == "A":
                gp.allreduce(xs, out=ys, side_stream=side)
                want, got = ref.allreduce(x, side_stream=side), torch.stack(ys)
            elif op == "R":
                gp.reduce_scatter(xs, out=zs, side_stream=side)
                want, got = ref.reduce_scatter(x, side_stream=side), torch.stack(zs)
            else:                                            # in place
                gp.allreduce(xs, out=xs, side_stream=side)
                want, got = ref.allreduce(x, side_stream=side), torch.stack(xs)
            g.check("call %d (%s)" % (t, op))
            _plan_guard_intact(gp, "call %d (%s)" % (t, op))
            assert torch.equal(_bits(got), _bits(want)), t
            if op != "I":
                assert torch.equal(_bits(torch.stack(xs)), _bits(x)), "input changed"


@pytest.mark.parametrize("fixup", ["exit", "deferred"])
def test_host_call_keeps_guards(fixup):
    P, G, k = 4, 64, 9
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    g = Guarded([2 * N] * (2 * P), device="cpu", pin=True)
    xs = [g.view(r, torch.bfloat16, (N,)) for r in range(P)]
    ys = [g.view(P + r, torch.bfloat16, (N,)) for r in range(P)]
    with EchoPlan(P, N, G, fixup=fixup, device=0) as gp, \
            EchoPlan(P, N, G, fixup=fixup, device=0) as ref:
        for t in range(3):
            x = W.generate(w, t, DEV)
            xc = x.cpu()
            for r in range(P):
                xs[r].copy_(xc[r])
            gp.allreduce_host(xs, ys)
            want = ref.allreduce(x).cpu()
            torch.cuda.synchronize()
            g.check("host call %d" % t)
            _plan_guard_intact(gp, "host call %d" % t)
            assert torch.equal(_bits(torch.stack(ys)), _bits(want)), t
            assert torch.equal(_bits(torch.stack(xs)), _bits(xc)), "input changed"


@pytest.mark.parametrize("P,G,k", [(2, 32, 37), (8, 128, 3), (5, 64, 7)], ids=lambda v: str(v))
def test_noalloc_call_keeps_guards(P, G, k):
    """The allocation-free call writes only the outputs and the caller's
    states."""
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    g = Guarded([2 * N] * (2 * P) + [4 * P * N] * 2)
    xs = [g.view(r, torch.bfloat16, (N,)) for r in range(P)]
    ys = [g.view(P + r, torch.bfloat16, (N,)) for r in range(P)]
    mf = g.view(2 * P, torch.float32, (P, N))
    ms = g.view(2 * P + 1, torch.float32, (P, N))
    mf.zero_()
    ms.zero_()
    cfg = make_config(P, N, G, True, 0.5, 0.5, 0.95, 0, "exit", 4)
    with EchoPlan(P, N, G, fixup="exit", device=0) as ref:
        for t in range(3):
            x = W.generate(w, t, DEV)
            for r in range(P):
                xs[r].copy_(x[r])
            abi.echo_allreduce_noalloc(cfg, [t_.data_ptr() for t_ in xs],
                                       [t_.data_ptr() for t_ in ys], mf.data_ptr(), ms.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
            want = ref.allreduce(x)
            g.check("noalloc call %d" % t)
            assert torch.equal(_bits(torch.stack(ys)), _bits(want)), t
            rf, rs = ref.get_state()
            assert torch.equal(_bits(mf), _bits(rf)) and torch.equal(_bits(ms), _bits(rs)), t


@pytest.mark.parametrize("fixup", ["exit", "deferred"])
def test_rank_stages_keep_guards(fixup):
    """The rank path's stages read and write only their exchange buffers and
    the caller's input and output."""
    P, G, k, bits = 4, 32, 13, 4
    N = P * G * k
    C = N // P
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    cb, cs = C * bits // 8, C // G
    with EchoRankPlan(P, 1, N, G, device=0, fixup=fixup) as p, \
            EmulatedGroup(P, N, G, fixup=fixup) as ref:
        sizes = [2 * N, P * cb, 4 * P * cs, P * cb, 4 * P * cs, cb, 4 * cs, P * cb, 4 * P * cs,
                 2 * N, 2 * C]
        g = Guarded(sizes)
        x = g.view(0, torch.bfloat16, (N,))
        send_c, send_s = g.view(1, torch.uint8, (P * cb,)), g.view(2, torch.float32, (P * cs,))
        recv_c, recv_s = g.view(3, torch.uint8, (P * cb,)), g.view(4, torch.float32, (P * cs,))
        red_c, red_s = g.view(5, torch.uint8, (cb,)), g.view(6, torch.float32, (cs,))
        all_c, all_s = g.view(7, torch.uint8, (P * cb,)), g.view(8, torch.float32, (P * cs,))
        out, out_rs = g.view(9, torch.bfloat16, (N,)), g.view(10, torch.bfloat16, (C,))
        st = torch.cuda.current_stream().cuda_stream
        h = p.handle
        for t in range(3):
            xx = W.generate(w, t, DEV)
            x.copy_(xx[1])
            y_ref = ref.allreduce(xx)
            abi.echo_rank_entry(h, x.data_ptr(), send_c.data_ptr(), send_s.data_ptr(), st)
            # the exchanges, from the reference group's buffers (rank 1's view)
            recv_c.copy_(ref.plans[1].bufs.recv_codes)
            recv_s.copy_(ref.plans[1].bufs.recv_scales)
            abi.echo_rank_reduce(h, recv_c.data_ptr(), recv_s.data_ptr(), red_c.data_ptr(),
                                 red_s.data_ptr(), st, 0)
            all_c.copy_(ref.plans[1].bufs.all_codes)
            all_s.copy_(ref.plans[1].bufs.all_scales)
            abi.echo_rank_exit(h, all_c.data_ptr(), all_s.data_ptr(), out.data_ptr(), st)
            g.check("rank call %d" % t)
            assert torch.equal(_bits(send_c), _bits(ref.plans[1].bufs.send_codes)), t
            assert torch.equal(_bits(red_c), _bits(ref.plans[1].bufs.red_codes)), t
            assert torch.equal(_bits(out), _bits(y_ref[1])), t
        xx = W.generate(w, 9, DEV)
        x.copy_(xx[1])
        z_ref = ref.reduce_scatter(xx)
        abi.echo_rank_entry(h, x.data_ptr(), send_c.data_ptr(), send_s.data_ptr(), st)
        recv_c.copy_(ref.plans[1].bufs.recv_codes)
        recv_s.copy_(ref.plans[1].bufs.recv_scales)
        abi.echo_rank_reduce_scatter(h, recv_c.data_ptr(), recv_s.data_ptr(), out_rs.data_ptr(),
                                     st, 0)
        g.check("rank reduce-scatter")
        assert torch.equal(_bits(out_rs), _bits(z_ref[1]))
