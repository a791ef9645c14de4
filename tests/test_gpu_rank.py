"""The rank path (include/echo_rank.h): P rank plans on one GPU, driven in
lockstep with the exchanges done by copies, against the oracle and against
the plan of P virtual ranks, call by call, bit for bit -- outputs, the
packed codes and scales on both wires, and every rank's two EMA states."""
import numpy as np
import pytest
import torch

import oracle
from bit_error_compensated_echo_b200 import abi
from bit_error_compensated_echo_b200 import workloads as W
from bit_error_compensated_echo_b200.api import EchoPlan
from bit_error_compensated_echo_b200.rank import EchoRankPlan
from parity import _bits_u16, _f32, assert_same
from rank_emulation import EmulatedGroup

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


def _compare_wires(grp: EmulatedGroup, plan: EchoPlan, call: int):
    """Rank r's send buffers are row r of the virtual entry transport;
    the gathered reduced chunks are the virtual reduced transport."""
    dv = plan.debug_view()
    for r, p in enumerate(grp.plans):
        _same("send codes r%d" % r, p.bufs.send_codes, dv["codes"][r], call)
        _same("send scales r%d" % r, p.bufs.send_scales, dv["scales"][r], call)
        _same("gathered codes r%d" % r, p.bufs.all_codes, dv["rcodes"], call)
        _same("gathered scales r%d" % r, p.bufs.all_scales, dv["rscales"], call)


CASES = [  # P, G, groups per chunk, bits
    (1, 32, 5, 4), (2, 32, 64, 4), (3, 64, 7, 4), (4, 128, 3, 4), (5, 32, 11, 4),
    (8, 128, 16, 4), (8, 32, 1, 4), (2, 64, 9, 8), (4, 32, 13, 8), (8, 128, 4, 8)]


@pytest.mark.parametrize("P,G,k,bits", CASES, ids=lambda v: str(v))
@pytest.mark.parametrize("comp,fixup", [(True, "exit"), (True, "side"), (True, "deferred"),
                                        (False, "deferred")])
def test_rank_group_equals_virtual_plan(P, G, k, bits, comp, fixup):
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    side = torch.cuda.Stream() if fixup == "side" else None
    kw = dict(compensate=comp, fixup=fixup, bits=bits)
    with EmulatedGroup(P, N, G, **kw) as grp, EchoPlan(P, N, G, device=0, **kw) as plan:
        for t in range(4):
            x = W.generate(w, t, DEV)
            y_rank = grp.allreduce(x, side_stream=side)
            y_virt = plan.allreduce(x, side_stream=side)
            torch.cuda.synchronize()
            _same("outputs", y_rank, y_virt, t)
            _compare_wires(grp, plan, t)
            if comp:
                mf_r, ms_r = grp.get_state()
                mf_v, ms_v = plan.get_state()
                _same("m_fast", mf_r, mf_v, t)
                _same("m_slow", ms_r, ms_v, t)


@pytest.mark.parametrize("fixup", ["exit", "side", "deferred"])
def test_rank_group_against_oracle(fixup):
    """The tiny workload's 16-call sequence, every rank against the oracle."""
    w = W.TINY
    side = torch.cuda.Stream() if fixup == "side" else None
    prm = oracle.Params(P=w.P, N=w.N, G=w.G, compensate=True)
    mf = np.zeros((w.P, w.N), np.float32)
    ms = np.zeros((w.P, w.N), np.float32)
    with EmulatedGroup(w.P, w.N, w.G, fixup=fixup) as grp:
        for t in range(w.calls):
            x = W.generate(w, t, DEV)
            y = grp.allreduce(x, side_stream=side)
            torch.cuda.synchronize()
            ref = oracle.allreduce(prm, _bits_u16(x), mf, ms)
            yb = _bits_u16(y)
            assert_same("outputs", yb, np.broadcast_to(ref.y, yb.shape), "bf16", t)
            for r, p in enumerate(grp.plans):
                assert_same("send codes r%d" % r, p.bufs.send_codes.cpu().numpy(), ref.codes[r],
                            "u8", t)
                assert_same("gathered codes r%d" % r, p.bufs.all_codes.cpu().numpy(),
                            ref.rcodes, "u8", t)
            gmf, gms = grp.get_state()
            assert_same("m_fast", _f32(gmf), mf, "f32", t)
            assert_same("m_slow", _f32(gms), ms, "f32", t)


@pytest.mark.parametrize("fixup", ["exit", "side", "deferred"])
@pytest.mark.parametrize("P,G,k,bits", [(2, 32, 8, 4), (4, 64, 5, 4), (8, 128, 3, 4),
                                        (4, 32, 6, 8)], ids=lambda v: str(v))
def test_rank_reduce_scatter_equals_virtual_plan(P, G, k, bits, fixup):
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    side = torch.cuda.Stream() if fixup == "side" else None
    kw = dict(fixup=fixup, bits=bits)
    with EmulatedGroup(P, N, G, **kw) as grp, EchoPlan(P, N, G, device=0, **kw) as plan:
        for t, op in enumerate("RRARAR"):
            x = W.generate(w, t, DEV)
            if op == "R":
                a, b = grp.reduce_scatter(x, side_stream=side), plan.reduce_scatter(
                    x, side_stream=side)
            else:
                a, b = grp.allreduce(x, side_stream=side), plan.allreduce(x, side_stream=side)
            torch.cuda.synchronize()
            _same("outputs (%s)" % op, a, b, t)
            mf_r, ms_r = grp.get_state()
            mf_v, ms_v = plan.get_state()
            _same("m_fast", mf_r, mf_v, t)
            _same("m_slow", ms_r, ms_v, t)


def test_rank_llama_shape_equals_virtual_plan():
    """P=8, 2048 x 4096 bf16 per rank, G=128, deferred fix-up: 6 calls."""
    w = W.LLAMA
    with EmulatedGroup(w.P, w.N, w.G, fixup="deferred") as grp, \
            EchoPlan(w.P, w.N, w.G, device=0, fixup="deferred") as plan:
        for t in range(6):
            x = W.generate(w, t, DEV)
            y_rank = grp.allreduce(x)
            y_virt = plan.allreduce(x)
            torch.cuda.synchronize()
            assert torch.equal(y_rank.view(torch.int16), y_virt.view(torch.int16)), t
        mf_r, ms_r = grp.get_state()
        mf_v, ms_v = plan.get_state()
        assert torch.equal(mf_r.view(torch.int32), mf_v.view(torch.int32))
        assert torch.equal(ms_r.view(torch.int32), ms_v.view(torch.int32))


def test_rank_state_calls():
    """set_state / get_state / reset_state of a rank plan, with a pending
    deferred fix-up, agree with the virtual plan's."""
    P, G, N = 4, 64, 4 * 64 * 6
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    g = torch.Generator(device=DEV).manual_seed(7)
    mf0 = torch.randn((P, N), generator=g, device=DEV) * 0.01
    ms0 = torch.randn((P, N), generator=g, device=DEV) * 0.01
    with EmulatedGroup(P, N, G, fixup="deferred") as grp, \
            EchoPlan(P, N, G, device=0, fixup="deferred") as plan:
        for r, p in enumerate(grp.plans):
            p.set_state(mf0[r].contiguous(), ms0[r].contiguous())
        plan.set_state(mf0.contiguous(), ms0.contiguous())
        for t in range(3):
            x = W.generate(w, t, DEV)
            _same("outputs", grp.allreduce(x), plan.allreduce(x), t)
            for a, b in zip(grp.get_state(), plan.get_state()):
                _same("state", a, b, t)
        for p in grp.plans:
            p.reset_state()
        plan.reset_state()
        x = W.generate(w, 9, DEV)
        _same("outputs after reset", grp.allreduce(x), plan.allreduce(x), 9)


def test_rank_stage_order_and_arguments():
    P, G, N = 2, 32, 2 * 32 * 4
    with EchoRankPlan(P, 1, N, G, device=0, fixup="exit") as p:
        with pytest.raises(abi.EchoError) as e:
            p.reduce()                         # no entry yet
        assert e.value.status == abi.ECHO_ERR_INVALID_ARG
        x = torch.zeros(N, dtype=torch.bfloat16, device=DEV)
        p.entry(x)
        p.reduce()
        with pytest.raises(abi.EchoError):
            p.reduce()                         # a second reduce needs a new entry
        with pytest.raises(abi.EchoError) as e:
            abi.echo_rank_entry(p.handle, x.data_ptr() + 2, p.bufs.send_codes.data_ptr(),
                                p.bufs.send_scales.data_ptr())
        assert e.value.status == abi.ECHO_ERR_ALIGNMENT
        assert p.launches_per_call() == 3     # the EXIT fix-up runs in the reduce
    cfg = abi.echo_config_default()
    cfg.P, cfg.N, cfg.G = P, N, G
    with pytest.raises(abi.EchoError) as e:
        abi.echo_rank_plan_create(cfg, 2)      # rank outside the group
    assert e.value.status == abi.ECHO_ERR_INVALID_ARG


def test_rank_group_mixed_widths():
    """Rank plans made with bits=8 follow a per-call width schedule on one
    state, bit-identical to the virtual-rank plan."""
    P, G, N = 4, 64, 4 * 64 * 7
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    with EmulatedGroup(P, N, G, fixup="deferred", bits=8) as grp, \
            EchoPlan(P, N, G, device=0, fixup="deferred", bits=8) as plan:
        for t, bits in enumerate([8, 8, 4, 4, 8, 4, 4, 8]):
            for p in grp.plans:
                p.set_bits(bits)
            plan.set_bits(bits)
            x = W.generate(w, t, DEV)
            _same("outputs", grp.allreduce(x), plan.allreduce(x), t)
            _compare_wires(grp, plan, t)
            for a, b in zip(grp.get_state(), plan.get_state()):
                _same("state", a, b, t)


@pytest.mark.parametrize("transport", ["copies", "peers"])
def test_rank_reduce_scatter_staged_size_against_oracle(transport):
    """P=8 ranks of 2048 x 4096 (owner chunks of 2^20 elements, where the
    reduce-scatter kernel stages the received code tiles in shared memory):
    three reduce-scatter calls of the rank group, deferred fix-up, against
    the oracle on 258 sampled group columns -- every rank's chunk of the
    sum and both states."""
    from rank_emulation import EmulatedPeerGroup
    wl = W.LLAMA
    P, N, G = wl.P, wl.N, wl.G
    cols = W.column_sample(wl, 256, seed=5)
    idx = torch.from_numpy(W.column_elements(cols, G)).to(DEV)
    prm = oracle.Params(P=P, N=N, G=G, compensate=True)
    mf = np.zeros((P, idx.numel()), np.float32)
    ms = np.zeros_like(mf)
    C = N // P
    group = EmulatedGroup if transport == "copies" else EmulatedPeerGroup
    with group(P, N, G, fixup="deferred") as grp:
        for t in range(3):
            x = W.generate(wl, t, DEV)
            y = grp.reduce_scatter(x)           # [P, C]: row r = rank r's chunk
            torch.cuda.synchronize()
            ref = oracle.reduce_scatter(prm, _bits_u16(x.index_select(1, idx)), mf, ms, cols)
            got = y.reshape(-1).index_select(0, idx)   # element i of the sum at [i // C][i % C]
            assert_same("owner outputs", _bits_u16(got), ref.y, "bf16", t)
            gmf, gms = grp.get_state()
            assert_same("m_fast", _f32(gmf.index_select(1, idx)), mf, "f32", t)
            assert_same("m_slow", _f32(gms.index_select(1, idx)), ms, "f32", t)
            del gmf, gms
    assert C >= 1 << 20


@pytest.mark.parametrize("transport,fixup,bits", [("copies", "exit", 4), ("peers", "exit", 4),
                                                  ("copies", "deferred", 4),
                                                  ("peers", "deferred", 4),
                                                  ("copies", "deferred", 8),
                                                  ("peers", "exit", 8)])
def test_rank_run_exit_every_element_ragged(transport, fixup, bits):
    """The all-gather kernel with a thread per 16-element run (owner chunks of
    at least 2^22 elements): P=2 ranks, owner chunks of 2^22 + 128
    elements, so each owner's last block of 256 runs is partial (8 runs);
    the fix-up in the reduce (32-byte state accesses) or deferred; 4- and
    8-bit codes; two all-reduce calls of the rank group, every element of
    every rank's output and both states against the oracle."""
    from rank_emulation import EmulatedPeerGroup
    P, G = 2, 128
    C = (1 << 22) + G
    N = P * C
    assert (C // 16) % 256 == 8
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    prm = oracle.Params(P=P, N=N, G=G, compensate=True, bits=bits)
    mf = np.zeros((P, N), np.float32)
    ms = np.zeros_like(mf)
    group = EmulatedGroup if transport == "copies" else EmulatedPeerGroup
    with group(P, N, G, fixup=fixup, bits=bits) as grp:
        for t in range(2):
            x = W.generate(w, t, DEV)
            y = grp.allreduce(x)
            torch.cuda.synchronize()
            ref = oracle.allreduce(prm, _bits_u16(x), mf, ms)
            yb = _bits_u16(y)
            assert_same("outputs", yb, np.broadcast_to(ref.y, yb.shape), "bf16", t)
            gmf, gms = grp.get_state()
            assert_same("m_fast", _f32(gmf), mf, "f32", t)
            assert_same("m_slow", _f32(gms), ms, "f32", t)
            del gmf, gms
