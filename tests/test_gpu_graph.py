"""CUDA-graph capture of the calls (include/echo.h, "Stream capture").

A graph captured at any point of a plan's life -- on a fresh plan or after
earlier calls, replayed across state resets and restores -- gives bit for
bit what the same eager calls give on a second plan: outputs and both EMA
states, for the all-reduce and the reduce-scatter, in the fix-up modes that
run on one stream (exit, deferred, side without a side stream), compensated
and not; the same for a whole rank-path call with its exchanges.  Captures
that a replay could not honour are refused with UNSUPPORTED."""
import pytest
import torch

from bit_error_compensated_echo_b200 import abi
from bit_error_compensated_echo_b200 import workloads as W
from bit_error_compensated_echo_b200.api import EchoPlan
from rank_emulation import EmulatedGroup

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _bits(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def _eq(a: torch.Tensor, b: torch.Tensor, what: str, call: int) -> None:
    assert torch.equal(_bits(a), _bits(b)), "%s differs at call %d" % (what, call)


def _call(plan: EchoPlan, op: str, x: torch.Tensor, out: torch.Tensor) -> None:
    if op == "allreduce":
        plan.allreduce(x, out=out)
    else:
        plan.reduce_scatter(x, out=out)


@pytest.mark.parametrize("capture_at", [0, 2])
@pytest.mark.parametrize("op", ["allreduce", "reduce_scatter"])
@pytest.mark.parametrize("fixup,comp", [("deferred", True), ("exit", True), ("side", True),
                                        ("deferred", False)])
def test_graph_replay_equals_eager(fixup, comp, op, capture_at):
    """One call captured after `capture_at` eager calls (0: a fresh plan,
    nothing pending), replayed 6 times on new inputs, with a state reset
    before the fourth replay and a restore before the sixth."""
    P, G, k = 4, 64, 6
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    oshape = (P, N) if op == "allreduce" else (P, N // P)
    kw = dict(compensate=comp, fixup=fixup, device=0)
    with EchoPlan(P, N, G, **kw) as gp, EchoPlan(P, N, G, **kw) as ep:
        xs = torch.zeros((P, N), dtype=torch.bfloat16, device=DEV)
        ys = torch.empty(oshape, dtype=torch.bfloat16, device=DEV)
        ye = torch.empty_like(ys)
        for t in range(capture_at):
            x = W.generate(w, t, DEV)
            _call(gp, op, x, ys)
            _call(ep, op, x, ye)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            _call(gp, op, xs, ys)
        saved = None
        for t in range(capture_at, capture_at + 6):
            if comp and t == capture_at + 3:
                gp.reset_state()
                ep.reset_state()
            if comp and t == capture_at + 5:
                gp.set_state(*saved)
                ep.set_state(*saved)
            x = W.generate(w, t, DEV)
            xs.copy_(x)
            g.replay()
            _call(ep, op, x, ye)
            torch.cuda.synchronize()
            _eq(ys, ye, "outputs", t)
            if comp:
                (gf, gs), (ef, es) = gp.get_state(), ep.get_state()
                _eq(gf, ef, "m_fast", t)
                _eq(gs, es, "m_slow", t)
                if t == capture_at + 1:
                    saved = (ef.clone(), es.clone())
        del g


@pytest.mark.parametrize("fixup", ["deferred", "exit"])
def test_graph_of_mixed_calls(fixup):
    """A graph of three calls on one plan (all-reduce at 8 bits, then a
    reduce-scatter and an all-reduce at 4 bits), captured on a fresh plan and
    replayed 4 times, equals the same eager sequence."""
    P, G, k = 8, 128, 3
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    kw = dict(fixup=fixup, bits=8, device=0)
    with EchoPlan(P, N, G, **kw) as gp, EchoPlan(P, N, G, **kw) as ep:
        xs = [torch.zeros((P, N), dtype=torch.bfloat16, device=DEV) for _ in range(3)]
        ys = [torch.empty((P, N), dtype=torch.bfloat16, device=DEV),
              torch.empty((P, N // P), dtype=torch.bfloat16, device=DEV),
              torch.empty((P, N), dtype=torch.bfloat16, device=DEV)]
        ye = [torch.empty_like(y) for y in ys]
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            gp.allreduce(xs[0], out=ys[0], bits=8)
            gp.reduce_scatter(xs[1], out=ys[1], bits=4)
            gp.allreduce(xs[2], out=ys[2], bits=4)
        for rep in range(4):
            x = [W.generate(w, 3 * rep + i, DEV) for i in range(3)]
            for a, b in zip(xs, x):
                a.copy_(b)
            g.replay()
            ep.allreduce(x[0], out=ye[0], bits=8)
            ep.reduce_scatter(x[1], out=ye[1], bits=4)
            ep.allreduce(x[2], out=ye[2], bits=4)
            torch.cuda.synchronize()
            for i in range(3):
                _eq(ys[i], ye[i], "output %d" % i, rep)
            for a, b in zip(gp.get_state(), ep.get_state()):
                _eq(a, b, "state", rep)
        del g


@pytest.mark.parametrize("fixup", ["deferred", "exit"])
def test_graph_of_rank_group_call(fixup):
    """A whole rank-path all-reduce of 4 emulated ranks -- entries, the
    exchange copies, reduces, exits -- captured on fresh rank plans, replays
    bit for bit like the virtual-rank plan's eager calls."""
    P, G, k = 4, 32, 9
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    with EmulatedGroup(P, N, G, fixup=fixup) as grp, \
            EchoPlan(P, N, G, device=0, fixup=fixup) as plan:
        xs = torch.zeros((P, N), dtype=torch.bfloat16, device=DEV)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            ys = grp.allreduce(xs)
        for t in range(5):
            x = W.generate(w, t, DEV)
            xs.copy_(x)
            g.replay()
            ye = plan.allreduce(x)
            torch.cuda.synchronize()
            _eq(ys, ye, "outputs", t)
            mf, ms = grp.get_state()
            ef, es = plan.get_state()
            _eq(mf, ef, "m_fast", t)
            _eq(ms, es, "m_slow", t)
        del g


def _refused_under_capture(fn) -> None:
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        with pytest.raises(abi.EchoError) as e:
            fn()
    assert e.value.status == abi.ECHO_ERR_UNSUPPORTED
    del g


@pytest.mark.filterwarnings("ignore:The CUDA Graph is empty")   # the refused calls queue nothing
def test_refused_captures():
    """Under capture: a side-stream fix-up, profiling and the host-buffer
    call return UNSUPPORTED before queueing anything; eager calls on the same
    plans still work and agree afterwards."""
    P, G, N = 2, 32, 2 * 32 * 4
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    x = W.generate(w, 0, DEV)
    out = torch.empty_like(x)
    side = torch.cuda.Stream()
    with EchoPlan(P, N, G, device=0, fixup="side") as sp, \
            EchoPlan(P, N, G, device=0, fixup="side") as ref:
        _refused_under_capture(lambda: sp.allreduce(x, out=out, side_stream=side))
        _refused_under_capture(lambda: sp.reduce_scatter(x, side_stream=side))
        ya = sp.allreduce(x, side_stream=side)
        yb = ref.allreduce(x)
        torch.cuda.synchronize()
        _eq(ya, yb, "outputs after refusal", 0)
    with EchoPlan(P, N, G, device=0) as pp:
        pp.profile_enable(True)
        _refused_under_capture(lambda: pp.allreduce(x, out=out))
        pp.profile_enable(False)
        xh = x.cpu().pin_memory()
        yh = torch.empty_like(xh).pin_memory()
        _refused_under_capture(lambda: pp.allreduce_host(xh, yh))


@pytest.mark.filterwarnings("ignore:The CUDA Graph is empty")   # the refused calls queue nothing
def test_rank_side_fixup_refused_under_capture():
    """The rank path's reduce and reduce-scatter with a side-stream fix-up
    return UNSUPPORTED while the stream is capturing; the plan then runs
    eagerly as if the refused calls had not been made."""
    from bit_error_compensated_echo_b200.rank import EchoRankPlan
    P, G, N = 2, 32, 2 * 32 * 4
    side = torch.cuda.Stream()
    x = torch.zeros(N, dtype=torch.bfloat16, device=DEV)
    with EchoRankPlan(P, 0, N, G, device=0, fixup="side") as p:
        p.entry(x)
        _refused_under_capture(lambda: p.reduce(side_stream=side))
        _refused_under_capture(
            lambda: p.reduce_scatter_finish(torch.empty(N // P, dtype=torch.bfloat16,
                                                        device=DEV), side_stream=side))
        p.reduce(side_stream=side)          # the entry is still waiting for its reduce
        torch.cuda.synchronize()
