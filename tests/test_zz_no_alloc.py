"""The allocation-free entry point, echo_allreduce_noalloc, called through
the C ABI, gives the same results as the plan-based echo_allreduce.

echo_allreduce_noalloc is for callers that cannot allocate device memory
on their call path (a serving process whose memory manager owns the whole
GPU, code that cannot take the synchronization of cudaMalloc/cudaFree, a
plugin host that hands over only buffers and a stream): its scratch lives
in a fixed device array inside the library and the caller owns the
compensator state.  Two calls in a row are compared, so the second one
also checks the state carried by the caller and that the shared scratch
array, left as the first call wrote it, does not leak into the next call.
Further tests: the largest size that fits the array, the free device
memory unchanged across calls, and, in a fresh process, the set-up refused
while a stream captures and redone in a second CUDA context.
This file is collected last on purpose; it passes alone or after the
other tests.
"""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from bit_error_compensated_echo_b200 import abi
from bit_error_compensated_echo_b200 import workloads as W
from bit_error_compensated_echo_b200.api import EchoPlan

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _check_same(got_bits, want_bits, what):
    # the acceptance the parity tests use: identical bits (which is within
    # 1 bf16 ulp for outputs and 1e-6 relative for fp32 state)
    assert np.array_equal(got_bits, want_bits), what


def _cfg(P, G, N, comp):
    cfg = abi.echo_config_default()
    cfg.P, cfg.G, cfg.N, cfg.compensate, cfg.device = P, G, N, int(comp), 0
    return cfg


def scratch_bytes(P, N, G, comp):
    """The array bytes a call needs: each part rounded up to 256 bytes."""
    def r(b):
        return (b + 255) // 256 * 256
    need = r(P * N // 2) + r(P * (N // G) * 4) + r(N // 2) + r((N // G) * 4)
    return need + (r(N * 4) if comp else 0)


# small and large N per rank, all four code paths of the reduce (with and
# without the compensator and the fix-up); the last case (8 ranks of
# 2048 x 4096, G = 32) needs 77 MiB of the 80 MiB
@pytest.mark.parametrize("P,G,k,comp", [(8, 128, 70, True), (3, 32, 41, True),
                                        (4, 64, 33, False), (8, 128, 600, True),
                                        (8, 32, 32768, True)])
def test_noalloc_matches_plan_two_calls(P, G, k, comp):
    N = P * G * k
    assert scratch_bytes(P, N, G, comp) <= abi.ECHO_NOALLOC_MAX_SCRATCH_BYTES
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    cfg = _cfg(P, G, N, comp)
    stream = torch.cuda.current_stream().cuda_stream
    mf = torch.zeros((P, N), dtype=torch.float32, device=DEV)
    ms = torch.zeros_like(mf)
    with EchoPlan(P, N, G, compensate=comp, fixup="exit", device=0) as plan:
        for t in range(2):
            x = W.generate(w, t, DEV)
            want = plan.allreduce(x)
            got = torch.empty_like(x)
            abi.echo_allreduce_noalloc(cfg, [x[r].data_ptr() for r in range(P)],
                                       [got[r].data_ptr() for r in range(P)],
                                       mf.data_ptr() if comp else 0,
                                       ms.data_ptr() if comp else 0, stream)
            torch.cuda.synchronize()
            _check_same(_bits(got), _bits(want), "outputs, call %d" % t)
            if comp:
                pmf, pms = plan.get_state()
                torch.cuda.synchronize()
                _check_same(mf.cpu().numpy().view(np.uint32), pmf.cpu().numpy().view(np.uint32),
                            "m_fast, call %d" % t)
                _check_same(ms.cpu().numpy().view(np.uint32), pms.cpu().numpy().view(np.uint32),
                            "m_slow, call %d" % t)


@pytest.mark.parametrize("P,G,k", [(8, 128, 600), (3, 32, 41)])
def test_noalloc_state_and_outputs_aligned_to_16_bytes_only(P, G, k):
    """The caller's states and outputs 16 bytes past a 32-byte boundary
    (the ABI asks for 16-byte alignment): the owner fix-up in the reduce
    and the output stores take their 16-byte form and give the same bits
    as the plan, two calls; a large and a small N."""
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    cfg = _cfg(P, G, N, True)
    stream = torch.cuda.current_stream().cuda_stream
    s2 = (4 + P * N + 7) // 8 * 8 + 4             # floats: 16 bytes past a 32-byte boundary
    sbuf = torch.zeros(s2 + P * N, dtype=torch.float32, device=DEV)
    mf = sbuf[4:4 + P * N].view(P, N)
    ms = sbuf[s2:s2 + P * N].view(P, N)
    obuf = torch.empty(P * (N + 16) + 8, dtype=torch.bfloat16, device=DEV)
    outs = [obuf[8 + r * (N + 16):8 + r * (N + 16) + N] for r in range(P)]
    assert mf.data_ptr() % 32 == 16 and ms.data_ptr() % 32 == 16
    assert all(t.data_ptr() % 32 == 16 for t in outs)
    with EchoPlan(P, N, G, compensate=True, fixup="exit", device=0) as plan:
        for t in range(2):
            x = W.generate(w, t, DEV)
            want = plan.allreduce(x)
            abi.echo_allreduce_noalloc(cfg, [x[r].data_ptr() for r in range(P)],
                                       [o.data_ptr() for o in outs], mf.data_ptr(),
                                       ms.data_ptr(), stream)
            torch.cuda.synchronize()
            _check_same(_bits(torch.stack(outs)), _bits(want), "outputs, call %d" % t)
            pmf, pms = plan.get_state()
            torch.cuda.synchronize()
            _check_same(mf.cpu().numpy().view(np.uint32), pmf.cpu().numpy().view(np.uint32),
                        "m_fast, call %d" % t)
            _check_same(ms.cpu().numpy().view(np.uint32), pms.cpu().numpy().view(np.uint32),
                        "m_slow, call %d" % t)


def test_noalloc_largest_supported_and_rejected_sizes():
    """8 ranks of 2048 x 4096 with the compensator fit the fixed scratch at
    every group size; 1 GiB per rank does not and is refused before anything
    is launched."""
    for G in (32, 64, 128):
        assert scratch_bytes(8, 2048 * 4096, G, True) <= abi.ECHO_NOALLOC_MAX_SCRATCH_BYTES
    small = _cfg(8, 128, 2048 * 4096, True)
    big = _cfg(8, 128, 1 << 29, True)
    assert scratch_bytes(8, 1 << 29, 128, True) > abi.ECHO_NOALLOC_MAX_SCRATCH_BYTES
    buf = torch.empty(64, dtype=torch.bfloat16, device=DEV)
    st = torch.empty(64, dtype=torch.float32, device=DEV)
    with pytest.raises(abi.EchoError) as e:
        abi.echo_allreduce_noalloc(big, [buf.data_ptr()] * 8, [buf.data_ptr()] * 8,
                                   st.data_ptr(), st.data_ptr(), 0)
    assert e.value.status == abi.ECHO_ERR_UNSUPPORTED
    with pytest.raises(abi.EchoError) as e:  # missing state with the compensator on
        abi.echo_allreduce_noalloc(small, [buf.data_ptr()] * 8, [buf.data_ptr()] * 8, 0, 0, 0)
    assert e.value.status == abi.ECHO_ERR_INVALID_ARG


def test_noalloc_free_device_memory_unchanged():
    """After a first call (the set-up), further calls leave the device's
    free memory exactly as it was: nothing is allocated on the call path."""
    P, G, k = 8, 128, 600
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    cfg = _cfg(P, G, N, True)
    xs = [W.generate(w, t, DEV) for t in range(3)]
    out = torch.empty_like(xs[0])
    mf = torch.zeros((P, N), dtype=torch.float32, device=DEV)
    ms = torch.zeros_like(mf)
    stream = torch.cuda.current_stream().cuda_stream

    def call(x):
        abi.echo_allreduce_noalloc(cfg, [x[r].data_ptr() for r in range(P)],
                                   [out[r].data_ptr() for r in range(P)],
                                   mf.data_ptr(), ms.data_ptr(), stream)

    call(xs[0])
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for x in xs[1:]:
        call(x)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)


def _child():
    """Run in a fresh process: the set-up refused on a capturing stream, then
    calls in the primary context and in a second context made with the
    driver API, each against the plan's results."""
    P, G, k = 4, 64, 33
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    cfg = _cfg(P, G, N, True)
    xs = [W.generate(w, t, DEV) for t in range(2)]
    want = []
    with EchoPlan(P, N, G, compensate=True, fixup="exit", device=0) as plan:
        for x in xs:
            y = plan.allreduce(x)
            pmf, pms = plan.get_state()
            want.append((_bits(y), pmf.cpu().numpy(), pms.cpu().numpy()))
    torch.cuda.synchronize()
    out = torch.full((P, N), 7.0, dtype=torch.bfloat16, device=DEV)
    mf = torch.zeros((P, N), dtype=torch.float32, device=DEV)
    ms = torch.zeros_like(mf)

    def call(x, st):
        abi.echo_allreduce_noalloc(cfg, [x[r].data_ptr() for r in range(P)],
                                   [out[r].data_ptr() for r in range(P)],
                                   mf.data_ptr(), ms.data_ptr(), st)

    # (a) the first call of the process, on a capturing stream: refused
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    status = None
    with torch.cuda.graph(g, stream=s):
        try:
            call(xs[0], s.cuda_stream)
        except abi.EchoError as e:
            status = e.status
    torch.cuda.synchronize()
    assert status == abi.ECHO_ERR_UNSUPPORTED, status
    assert not mf.any() and bool((out == 7.0).all()), "a refused call launched work"
    del g

    # (b) the primary context (torch's): call 0
    call(xs[0], torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    _check_same(_bits(out), want[0][0], "outputs, call 0")
    _check_same(mf.cpu().numpy(), want[0][1], "m_fast, call 0")
    mf0, ms0 = mf.cpu().numpy(), ms.cpu().numpy()

    # (c) call 1 in a second context on the same device (driver API)
    cu = ctypes.CDLL("libcuda.so.1")
    u64, vp, sz = ctypes.c_uint64, ctypes.c_void_p, ctypes.c_size_t
    cu.cuMemAlloc_v2.argtypes = [ctypes.POINTER(u64), sz]
    cu.cuMemcpyHtoD_v2.argtypes = [u64, vp, sz]
    cu.cuMemcpyDtoH_v2.argtypes = [vp, u64, sz]
    cu.cuMemFree_v2.argtypes = [u64]
    cu.cuCtxCreate_v2.argtypes = [ctypes.POINTER(vp), ctypes.c_uint, ctypes.c_int]
    cu.cuCtxDestroy_v2.argtypes = [vp]

    def ok(rc, what):
        assert rc == 0, "%s returned %d" % (what, rc)

    dev = ctypes.c_int()
    ok(cu.cuDeviceGet(ctypes.byref(dev), 0), "cuDeviceGet")
    ctx = vp()
    ok(cu.cuCtxCreate_v2(ctypes.byref(ctx), 0, dev), "cuCtxCreate")   # now current
    held = []
    try:
        def alloc(nbytes):
            p = u64()
            ok(cu.cuMemAlloc_v2(ctypes.byref(p), nbytes), "cuMemAlloc")
            held.append(p.value)
            return p.value

        x1 = np.ascontiguousarray(_bits(xs[1]))
        xin = [alloc(2 * N) for _ in range(P)]
        yout = [alloc(2 * N) for _ in range(P)]
        dmf, dms = alloc(4 * P * N), alloc(4 * P * N)
        for r in range(P):
            ok(cu.cuMemcpyHtoD_v2(xin[r], x1[r].ctypes.data, 2 * N), "cuMemcpyHtoD")
        ok(cu.cuMemcpyHtoD_v2(dmf, mf0.ctypes.data, 4 * P * N), "cuMemcpyHtoD")
        ok(cu.cuMemcpyHtoD_v2(dms, ms0.ctypes.data, 4 * P * N), "cuMemcpyHtoD")
        abi.echo_allreduce_noalloc(cfg, xin, yout, dmf, dms, 0)
        ok(cu.cuCtxSynchronize(), "cuCtxSynchronize")
        y1 = np.empty((P, N), np.uint16)
        gmf = np.empty((P, N), np.float32)
        for r in range(P):
            ok(cu.cuMemcpyDtoH_v2(y1[r].ctypes.data, yout[r], 2 * N), "cuMemcpyDtoH")
        ok(cu.cuMemcpyDtoH_v2(gmf.ctypes.data, dmf, 4 * P * N), "cuMemcpyDtoH")
        _check_same(y1, want[1][0], "outputs, call 1, second context")
        _check_same(gmf, want[1][1], "m_fast, call 1, second context")
    finally:
        for p in held:
            cu.cuMemFree_v2(p)
        ok(cu.cuCtxDestroy_v2(ctx), "cuCtxDestroy")   # the primary context is current again

    # (d) call 1 again in the primary context, from the state after call 0
    mf.copy_(torch.from_numpy(mf0))
    ms.copy_(torch.from_numpy(ms0))
    call(xs[1], torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    _check_same(_bits(out), want[1][0], "outputs, call 1, primary context")
    _check_same(ms.cpu().numpy(), want[1][2], "m_slow, call 1, primary context")
    print("noalloc child ok")


def test_noalloc_setup_per_context_and_not_under_capture():
    """In a fresh process: the first call, made while its stream captures,
    is refused with ECHO_ERR_UNSUPPORTED and launches nothing; the next
    call does the set-up; a call in a second CUDA context on the device
    does the set-up again for that context; back in the first context the
    results are still the plan's."""
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ)
    env["PYTHONPATH"] = os.pathsep.join([os.path.dirname(here), here,
                                         env.get("PYTHONPATH", "")])
    r = subprocess.run([sys.executable, os.path.abspath(__file__), "--child"], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "noalloc child ok" in r.stdout, r.stdout + r.stderr


if __name__ == "__main__" and "--child" in sys.argv:
    _child()
