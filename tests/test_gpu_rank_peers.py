"""The fused transport of the rank path (include/echo_rank.h, "Fused
transport over peer memory"): P rank plans on one GPU whose entries store
each chunk straight into the owner's window and whose exits load the owners'
reduced chunks straight from theirs, against the oracle and against the plan
of P virtual ranks, call by call, bit for bit -- outputs, the bytes in every
window (each rank's receive buffers and each owner's reduced chunk) and
every rank's two EMA states."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle

from bit_error_compensated_echo_b200 import abi
from bit_error_compensated_echo_b200 import workloads as W
from bit_error_compensated_echo_b200.api import EchoPlan, _DeviceArray
from bit_error_compensated_echo_b200.rank import EchoRankPlan, PeerWindows
from parity import _bits_u16, _f32, assert_same
from rank_emulation import EmulatedGroup, EmulatedPeerGroup

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _same(name, a: torch.Tensor, b: torch.Tensor, call: int):
    a, b = a.contiguous().cpu(), b.contiguous().cpu()
    if a.dtype == torch.bfloat16:
        assert_same(name, _bits_u16(a), _bits_u16(b), "bf16", call)
    elif a.dtype == torch.float32:
        assert_same(name, _f32(a), _f32(b), "f32", call)
    else:
        assert_same(name, a.numpy(), b.numpy(), "u8", call)


def _window_bytes(win: PeerWindows, key: str, n: int, dtype) -> torch.Tensor:
    """A host copy of n elements of this rank's window buffer `key`."""
    typestr = {torch.uint8: "|u1", torch.float32: "<f4"}[dtype]
    view = torch.as_tensor(_DeviceArray(win.own(key), (n,), typestr), device=DEV)
    return view.cpu()


def _compare_windows(grp: EmulatedPeerGroup, plan: EchoPlan, call: int):
    """Rank o's receive part r is row r, chunk o of the virtual entry
    transport; owner o's reduced chunk is chunk o of the reduced transport."""
    dv = plan.debug_view()
    P, N, G = plan.P, plan.N, plan.G
    C = N // P
    cb, cs = C * plan.bits // 8, C // G
    codes = dv["codes"].reshape(P, P, cb)          # [row r][chunk o]
    scales = dv["scales"].reshape(P, P, cs)
    rcodes = dv["rcodes"].reshape(P, cb)
    rscales = dv["rscales"].reshape(P, cs)
    for o, w in enumerate(grp.wins):
        guard = _window_bytes(w, "guard", w.layout["guard_bytes"], torch.uint8)
        assert bool((guard == 0xA5).all()), "call %d: window guard of rank %d changed" % (call, o)
        rc = _window_bytes(w, "recv_codes", P * cb, torch.uint8).reshape(P, cb)
        rs = _window_bytes(w, "recv_scales", P * cs, torch.float32).reshape(P, cs)
        _same("recv codes of rank %d" % o, rc, codes[:, o], call)
        _same("recv scales of rank %d" % o, rs, scales[:, o], call)
        _same("red codes of owner %d" % o, _window_bytes(w, "red_codes", cb, torch.uint8),
              rcodes[o], call)
        _same("red scales of owner %d" % o, _window_bytes(w, "red_scales", cs, torch.float32),
              rscales[o], call)


def _windows_against_oracle(grp: EmulatedPeerGroup, ref, bits: int, call: int,
                            reduced: bool = True):
    """Rank o's receive part r holds rank r's chunk o of the oracle's entry
    codes and scales; owner o's reduced chunk is chunk o of the oracle's
    requantized codes and scales (all-reduce calls only)."""
    P, N, G = grp.P, grp.N, grp.G
    C = N // P
    cb, cs = C * bits // 8, C // G
    for o, w in enumerate(grp.wins):
        rc = _window_bytes(w, "recv_codes", P * cb, torch.uint8).reshape(P, cb)
        rs = _window_bytes(w, "recv_scales", P * cs, torch.float32).reshape(P, cs)
        assert_same("recv codes of rank %d" % o, rc.numpy(), ref.codes[:, o * cb:(o + 1) * cb],
                    "u8", call)
        assert_same("recv scales of rank %d" % o, rs.numpy(),
                    ref.scales[:, o * cs:(o + 1) * cs], "f32", call)
        if reduced:
            assert_same("red codes of owner %d" % o,
                        _window_bytes(w, "red_codes", cb, torch.uint8).numpy(),
                        ref.rcodes[o * cb:(o + 1) * cb], "u8", call)
            assert_same("red scales of owner %d" % o,
                        _window_bytes(w, "red_scales", cs, torch.float32).numpy(),
                        ref.rscales[o * cs:(o + 1) * cs], "f32", call)


@pytest.mark.parametrize("comp,fixup", [(True, "exit"), (True, "side"), (True, "deferred"),
                                        (False, "deferred")])
def test_peer_group_against_oracle(comp, fixup):
    """The tiny workload's 16-call sequence on the fused transport, every
    rank against the oracle: outputs, every window, both states."""
    w = W.TINY
    side = torch.cuda.Stream() if fixup == "side" else None
    prm = oracle.Params(P=w.P, N=w.N, G=w.G, compensate=comp)
    mf = np.zeros((w.P, w.N), np.float32)
    ms = np.zeros((w.P, w.N), np.float32)
    with EmulatedPeerGroup(w.P, w.N, w.G, compensate=comp, fixup=fixup) as grp:
        for t in range(w.calls):
            x = W.generate(w, t, DEV)
            y = grp.allreduce(x, side_stream=side)
            torch.cuda.synchronize()
            ref = oracle.allreduce(prm, _bits_u16(x), mf, ms)
            yb = _bits_u16(y)
            assert_same("outputs", yb, np.broadcast_to(ref.y, yb.shape), "bf16", t)
            _windows_against_oracle(grp, ref, 4, t)
            if comp:
                gmf, gms = grp.get_state()
                assert_same("m_fast", _f32(gmf), mf, "f32", t)
                assert_same("m_slow", _f32(gms), ms, "f32", t)


@pytest.mark.parametrize("P,G,k", [(3, 64, 7), (8, 128, 5), (8, 32, 3), (5, 32, 11)],
                         ids=lambda v: str(v))
@pytest.mark.parametrize("fixup", ["exit", "side", "deferred"])
def test_peer_group_mixed_ops_against_oracle(P, G, k, fixup):
    """All-reduces and reduce-scatters at 8 and 4 bits on one state of a
    bits=8 group, on the fused transport, against the oracle call by call
    (ragged chunks: k groups per owner)."""
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    side = torch.cuda.Stream() if fixup == "side" else None
    prm = oracle.Params(P=P, N=N, G=G, compensate=True)
    mf = np.zeros((P, N), np.float32)
    ms = np.zeros((P, N), np.float32)
    C = N // P
    with EmulatedPeerGroup(P, N, G, fixup=fixup, bits=8) as grp:
        for t, (op, bits) in enumerate([("A", 8), ("R", 8), ("A", 4), ("R", 4), ("A", 4),
                                        ("A", 8), ("R", 4), ("A", 4)]):
            for p in grp.plans:
                p.set_bits(bits)
            x = W.generate(w, t, DEV)
            cp = dataclasses.replace(prm, bits=bits)
            if op == "A":
                y = grp.allreduce(x, side)
                torch.cuda.synchronize()
                ref = oracle.allreduce(cp, _bits_u16(x), mf, ms)
                yb = _bits_u16(y)
                assert_same("outputs", yb, np.broadcast_to(ref.y, yb.shape), "bf16", t)
            else:
                y = grp.reduce_scatter(x, side)
                torch.cuda.synchronize()
                ref = oracle.reduce_scatter(cp, _bits_u16(x), mf, ms)
                assert_same("owner outputs", _bits_u16(y), ref.y.reshape(P, C), "bf16", t)
            _windows_against_oracle(grp, ref, bits, t, reduced=(op == "A"))
            gmf, gms = grp.get_state()
            assert_same("m_fast", _f32(gmf), mf, "f32", t)
            assert_same("m_slow", _f32(gms), ms, "f32", t)


def test_peer_group_llama_shape_against_oracle():
    """P=8, 2048 x 4096 bf16 per rank, G=128, deferred fix-up, 4 calls on
    the fused transport: outputs and both states against the oracle on 258
    sampled group columns."""
    wl = W.LLAMA
    cols = W.column_sample(wl, 256, seed=99)
    idx = torch.from_numpy(W.column_elements(cols, wl.G)).to(DEV)
    prm = oracle.Params(P=wl.P, N=wl.N, G=wl.G, compensate=True)
    mf = np.zeros((wl.P, idx.numel()), np.float32)
    ms = np.zeros_like(mf)
    with EmulatedPeerGroup(wl.P, wl.N, wl.G, fixup="deferred") as grp:
        for t in range(4):
            x = W.generate(wl, t, DEV)
            y = grp.allreduce(x)
            torch.cuda.synchronize()
            ref = oracle.allreduce(prm, _bits_u16(x.index_select(1, idx)), mf, ms, cols)
            yb = _bits_u16(y.index_select(1, idx))
            assert_same("outputs", yb, np.broadcast_to(ref.y, yb.shape), "bf16", t)
            gmf, gms = grp.get_state()
            assert_same("m_fast", _f32(gmf.index_select(1, idx)), mf, "f32", t)
            assert_same("m_slow", _f32(gms.index_select(1, idx)), ms, "f32", t)
            del gmf, gms


CASES = [  # P, G, groups per chunk, bits
    (1, 32, 5, 4), (2, 32, 64, 4), (3, 64, 7, 4), (4, 128, 3, 4), (5, 32, 11, 4),
    (8, 128, 16, 4), (8, 32, 1, 4), (2, 64, 9, 8), (4, 32, 13, 8), (8, 128, 4, 8)]


@pytest.mark.parametrize("P,G,k,bits", CASES, ids=lambda v: str(v))
@pytest.mark.parametrize("comp,fixup", [(True, "exit"), (True, "side"), (True, "deferred"),
                                        (False, "deferred")])
def test_peer_group_equals_virtual_plan(P, G, k, bits, comp, fixup):
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    side = torch.cuda.Stream() if fixup == "side" else None
    kw = dict(compensate=comp, fixup=fixup, bits=bits)
    with EmulatedPeerGroup(P, N, G, **kw) as grp, EchoPlan(P, N, G, device=0, **kw) as plan:
        for t in range(4):
            x = W.generate(w, t, DEV)
            y_rank = grp.allreduce(x, side_stream=side)
            y_virt = plan.allreduce(x, side_stream=side)
            torch.cuda.synchronize()
            _same("outputs", y_rank, y_virt, t)
            _compare_windows(grp, plan, t)
            if comp:
                for a, b in zip(grp.get_state(), plan.get_state()):
                    _same("state", a, b, t)


@pytest.mark.parametrize("fixup", ["exit", "side", "deferred"])
def test_peer_group_mixed_ops_and_widths(fixup):
    """All-reduces and reduce-scatters at 8 and 4 bits on one state, the
    fused group against the exchange-buffer group and the virtual plan."""
    P, G, k = 4, 64, 7
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    side = torch.cuda.Stream() if fixup == "side" else None
    kw = dict(fixup=fixup, bits=8)
    with EmulatedPeerGroup(P, N, G, **kw) as fused, EmulatedGroup(P, N, G, **kw) as copies, \
            EchoPlan(P, N, G, device=0, **kw) as plan:
        for t, (op, bits) in enumerate([("A", 8), ("R", 8), ("A", 4), ("R", 4), ("A", 4),
                                        ("A", 8), ("R", 4)]):
            for p in fused.plans + copies.plans:
                p.set_bits(bits)
            plan.set_bits(bits)
            x = W.generate(w, t, DEV)
            if op == "A":
                ys = [fused.allreduce(x, side), copies.allreduce(x, side),
                      plan.allreduce(x, side_stream=side)]
            else:
                ys = [fused.reduce_scatter(x, side), copies.reduce_scatter(x, side),
                      plan.reduce_scatter(x, side_stream=side)]
            torch.cuda.synchronize()
            _same("fused vs copies (%s)" % op, ys[0], ys[1], t)
            _same("fused vs virtual (%s)" % op, ys[0], ys[2], t)
            for a, b in zip(fused.get_state(), plan.get_state()):
                _same("state", a, b, t)


def test_peer_group_llama_shape():
    """P=8, 2048 x 4096 bf16 per rank, G=128, deferred fix-up: 4 calls."""
    wl = W.LLAMA
    with EmulatedPeerGroup(wl.P, wl.N, wl.G, fixup="deferred") as grp, \
            EchoPlan(wl.P, wl.N, wl.G, device=0, fixup="deferred") as plan:
        for t in range(4):
            x = W.generate(wl, t, DEV)
            y_rank = grp.allreduce(x)
            y_virt = plan.allreduce(x)
            torch.cuda.synchronize()
            assert torch.equal(y_rank.view(torch.int16), y_virt.view(torch.int16)), t
        for a, b in zip(grp.get_state(), plan.get_state()):
            assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_peer_calls_arguments():
    P, G, N = 2, 32, 2 * 32 * 4
    with EchoRankPlan(P, 0, N, G, device=0) as p:
        lay = abi.echo_rank_window(p.handle)
        assert lay["base"] and lay["base"] % 256 == 0
        assert lay == abi.echo_rank_window(p.handle)          # allocated once
        C = N // P
        assert lay["red_codes"] >= lay["recv_scales"] + P * (C // G) * 4
        assert lay["guard"] >= lay["red_scales"] + (C // G) * 4
        assert lay["guard_bytes"] == 4096 and lay["bytes"] == lay["guard"] + 4096
        x = torch.zeros(N, dtype=torch.bfloat16, device=DEV)
        codes = [lay["base"] + lay["recv_codes"]] * P
        scales = [lay["base"] + lay["recv_scales"]] * P
        with pytest.raises(abi.EchoError) as e:
            abi.echo_rank_entry_peers(p.handle, x.data_ptr(), [codes[0], 0], scales)
        assert e.value.status == abi.ECHO_ERR_INVALID_ARG
        with pytest.raises(abi.EchoError) as e:
            abi.echo_rank_entry_peers(p.handle, x.data_ptr(), [codes[0], codes[1] + 8], scales)
        assert e.value.status == abi.ECHO_ERR_ALIGNMENT
        with pytest.raises(abi.EchoError) as e:
            abi.echo_rank_exit_peers(p.handle, [lay["base"] + lay["red_codes"]] * P,
                                     [lay["base"] + lay["red_scales"] + 2] * P, x.data_ptr())
        assert e.value.status == abi.ECHO_ERR_ALIGNMENT


@pytest.mark.parametrize("fixup", ["deferred", "exit"])
def test_graph_of_peer_group_call(fixup):
    """A whole fused-transport all-reduce of 4 emulated ranks captured into
    a CUDA graph on fresh plans replays like the virtual plan's eager calls."""
    P, G, k = 4, 32, 9
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    with EmulatedPeerGroup(P, N, G, fixup=fixup) as grp, \
            EchoPlan(P, N, G, device=0, fixup=fixup) as plan:
        xs = torch.zeros((P, N), dtype=torch.bfloat16, device=DEV)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            ys = grp.allreduce(xs)
        for t in range(4):
            x = W.generate(w, t, DEV)
            xs.copy_(x)
            g.replay()
            ye = plan.allreduce(x)
            torch.cuda.synchronize()
            _same("outputs", ys, ye, t)
            for a, b in zip(grp.get_state(), plan.get_state()):
                _same("state", a, b, t)
        del g
