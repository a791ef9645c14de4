"""Host-side checks of the C-ABI library (no GPU needed).

The library loads, exports every entry point that include/echo.h declares,
and rejects invalid configurations on the host before any CUDA call.  The
benchmark's byte counts and cross-rank aggregation are checked here too,
the latter with two gloo ranks on the CPU.
"""
import ctypes
import os
import re
import socket

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def abi():
    from bit_error_compensated_echo_b200 import build
    build.build()
    from bit_error_compensated_echo_b200 import abi as a
    return a


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(echo_\w+)\s*\(", text)
    return sorted(set(names))


def test_exports_every_declared_symbol(abi):
    names = declared_functions()
    assert "echo_allreduce" in names and "echo_plan_create" in names
    for n in names:
        assert hasattr(abi.lib, n), n


def test_status_strings(abi):
    for code, name in abi.STATUS.items():
        assert abi.echo_status_string(code) == name


def _cfg(abi, **kw):
    c = abi.echo_config_default()
    c.P, c.G, c.N = 8, 128, 8 * 128 * 4
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("kw,status", [
    (dict(P=0), "ECHO_ERR_UNSUPPORTED"), (dict(P=9), "ECHO_ERR_UNSUPPORTED"),
    (dict(G=16), "ECHO_ERR_UNSUPPORTED"), (dict(G=96), "ECHO_ERR_UNSUPPORTED"),
    (dict(N=0), "ECHO_ERR_SHAPE"), (dict(N=-1024), "ECHO_ERR_SHAPE"),
    (dict(N=8 * 128 * 4 + 128), "ECHO_ERR_SHAPE"),
    (dict(alpha=1.5), "ECHO_ERR_INVALID_ARG"), (dict(beta_fast=-0.1), "ECHO_ERR_INVALID_ARG"),
    (dict(beta_slow=float("nan")), "ECHO_ERR_INVALID_ARG"),
    (dict(fixup=3), "ECHO_ERR_INVALID_ARG"), (dict(compensate=2), "ECHO_ERR_INVALID_ARG"),
    (dict(device=-1), "ECHO_ERR_INVALID_ARG"),
    (dict(bits=6), "ECHO_ERR_UNSUPPORTED"), (dict(bits=0), "ECHO_ERR_UNSUPPORTED"),
])
def test_invalid_configs_rejected_on_host(abi, kw, status):
    cfg = _cfg(abi, **kw)
    assert abi.echo_workspace_bytes(cfg) == 0
    with pytest.raises(abi.EchoError) as e:
        abi.echo_plan_create(cfg)
    assert abi.STATUS[e.value.status] == status


def test_null_arguments(abi):
    import ctypes
    assert abi.lib.echo_plan_create(None, None) == abi.ECHO_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert abi.lib.echo_plan_create(ctypes.byref(h), None) == abi.ECHO_ERR_INVALID_ARG
    assert abi.lib.echo_allreduce(None, None, None, None, None) == abi.ECHO_ERR_INVALID_ARG
    assert abi.lib.echo_reset_state(None, None) == abi.ECHO_ERR_INVALID_ARG
    assert abi.lib.echo_plan_destroy(None) == abi.ECHO_OK
    assert abi.lib.echo_launches_per_call(None) == 0


def test_workspace_bytes_closed_form(abi):
    def al(b):
        return (b + 255) // 256 * 256
    for P, G, k, comp, bits in ((8, 128, 64, 1, 4), (2, 32, 3, 0, 4), (5, 64, 7, 1, 4),
                                (4, 32, 5, 1, 8), (3, 128, 2, 0, 8)):
        N = P * G * k
        c = _cfg(abi, P=P, G=G, N=N, compensate=comp, bits=bits)
        # codes, scales, reduced codes and scales
        want = (al(P * N * bits // 8) + al(P * (N // G) * 4) + al(N * bits // 8)
                + al((N // G) * 4))
        if comp:
            want += 2 * al(P * N * 4) + al(N * 4)
        want += 4096                        # the guard zone after the sub-buffers
        assert abi.echo_workspace_bytes(c) == want


def test_rank_plan_sizes_and_host_checks(abi):
    """The rank path (include/echo_rank.h): chunk sizes and workspace in
    closed form, and invalid arguments rejected before any CUDA call."""
    def al(b):
        return (b + 255) // 256 * 256
    for P, G, k, comp, bits in ((8, 128, 64, 1, 4), (2, 32, 3, 0, 4), (4, 32, 5, 1, 8)):
        N = P * G * k
        c = _cfg(abi, P=P, G=G, N=N, compensate=comp, bits=bits)
        C = N // P
        assert abi.echo_rank_exchange_bytes(c) == (C * bits // 8, C // G * 4)
        want = (2 * al(N * 4) + al(C * 4)) if comp else 0
        assert abi.echo_rank_workspace_bytes(c) == want
    c = _cfg(abi)
    for rank in (-1, 8):
        with pytest.raises(abi.EchoError) as e:
            abi.echo_rank_plan_create(c, rank)
        assert e.value.status == abi.ECHO_ERR_INVALID_ARG
    with pytest.raises(abi.EchoError) as e:
        abi.echo_rank_plan_create(_cfg(abi, G=48), 0)
    assert e.value.status == abi.ECHO_ERR_UNSUPPORTED
    with pytest.raises(abi.EchoError) as e:
        abi.echo_rank_exchange_bytes(_cfg(abi, N=100))
    assert e.value.status == abi.ECHO_ERR_SHAPE
    L = abi.lib
    assert L.echo_rank_entry(None, None, None, None, None) == abi.ECHO_ERR_INVALID_ARG
    assert L.echo_rank_reduce(None, None, None, None, None, None, None) == \
        abi.ECHO_ERR_INVALID_ARG
    assert L.echo_rank_exit(None, None, None, None, None) == abi.ECHO_ERR_INVALID_ARG
    assert L.echo_rank_plan_destroy(None) == abi.ECHO_OK
    assert L.echo_rank_launches_per_call(None) == 0
    # the fused transport and the IPC layer (include/echo_rank.h)
    assert L.echo_rank_window(None, None) == abi.ECHO_ERR_INVALID_ARG
    assert L.echo_rank_entry_peers(None, None, None, None, None) == abi.ECHO_ERR_INVALID_ARG
    assert L.echo_rank_exit_peers(None, None, None, None, None) == abi.ECHO_ERR_INVALID_ARG
    assert L.echo_ipc_handle_get(None, None) == abi.ECHO_ERR_INVALID_ARG
    assert L.echo_ipc_open(None, 0, None) == abi.ECHO_ERR_INVALID_ARG
    assert L.echo_ipc_close(None, 0) == abi.ECHO_ERR_INVALID_ARG
    h = abi.echo_ipc_handle()
    out = ctypes.c_void_p()
    assert L.echo_ipc_open(ctypes.byref(h), -1, ctypes.byref(out)) == abi.ECHO_ERR_INVALID_ARG


def test_bench_byte_counts():
    import bench
    # 1 GiB per rank, P=8, G=128: 95.33 GB with the compensator, 22.31 GB off
    N = 1 << 29
    assert abs(bench.call_min_bytes(8, N, 128, True) / 1e9 - 95.33) < 0.01
    assert abs(bench.call_min_bytes(8, N, 128, False) / 1e9 - 22.31) < 0.01
    # tiny case: 211,968 and 48,128 bytes
    assert bench.call_min_bytes(2, 4096, 32, True) == 211968
    assert bench.call_min_bytes(2, 4096, 32, False) == 48128
    for G, q in ((32, 0.625), (64, 0.5625), (128, 0.53125)):
        assert bench.transport_bytes_per_elem(G) == q


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, ws, port, q):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        ms = [3.0, 5.0][rank]
        bytes_ = [100.0, 300.0][rank]
        t = bench.max_over_ranks(ms, ws, torch.device("cpu"))
        b = bench.sum_over_ranks(bytes_, ws, torch.device("cpu"))
        q.put((rank, t, b))
    finally:
        dist.destroy_process_group()


def test_cross_rank_aggregation_gloo():
    """Two gloo ranks: the step time is the max over ranks and the bytes are
    summed, so the whole-job value is total bytes / slowest rank."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert [g[1] for g in got] == [5.0, 5.0]
    assert [g[2] for g in got] == [400.0, 400.0]
    import bench
    v, t = bench.aggregate([3.0, 5.0], [100.0, 300.0])
    assert t == 5.0 and abs(v - 400.0 / 5e-3 / 1e9) < 1e-12


def test_bench_kernel_rooflines():
    """Per-kernel roofline fractions of the bench line: the algorithmic bytes
    of each kernel over its average launch time; the reduce writes the
    outputs (there is no exit launch on one GPU) and counts them."""
    import bench
    P, N, G = 8, 1 << 29, 128
    prof = {"calls": 10, "entry_ms": 117.0, "reduce_ms": 20.0, "exit_ms": 0.0028, "fixup_ms": 0.0}
    r = bench.kernel_rooflines(prof, P, N, G, True, "deferred", 4, 6543.4)
    q = 0.5 + 4 / 128
    assert set(r) == {"echo_entry", "echo_reduce"}
    assert r["echo_entry"]["bytes"] == P * N * (18 + q) + 4 * N
    assert r["echo_reduce"]["bytes"] == P * N * q + N * q + 4 * N + 2 * P * N
    for k in r.values():
        assert abs(k["achieved"] - k["bytes"] / (k["avg_launch_ms"] / 1e3) / 1e9) < 0.1
        assert abs(k["frac"] - k["achieved"] / 6543.4) < 1e-3
    off = dict(prof, exit_ms=0.0028)   # the profile's events around no exit launch
    r = bench.kernel_rooflines(off, P, N, G, False, "deferred", 4, 6543.4)
    assert "echo_exit" not in r
    assert r["echo_reduce"]["bytes"] == P * N * q + N * q + 2 * P * N
    small = bench.kernel_rooflines(off, P, 1 << 19, G, True, "exit", 4, 6543.4)
    assert small["echo_reduce"]["bytes"] == P * (1 << 19) * (q + 2) + (1 << 19) * (q + 16)
    rs = bench.kernel_rooflines(dict(prof, exit_ms=0.0028), P, N, G, True, "deferred", 4,
                                6543.4, rs=True)
    assert set(rs) == {"echo_entry", "echo_rs"}
    assert rs["echo_rs"]["bytes"] == P * N * q + 2 * N + 4 * N
