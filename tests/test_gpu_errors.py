"""Failure paths on the GPU that fault nothing: a plan whose workspace
cannot be allocated returns ECHO_ERR_OOM (the CUDA error is cleared, not
left sticky), a kernel wait that runs out is reported as ECHO_ERR_TIMEOUT
through the device error word, and the context stays usable for the next
plan and call."""
import ctypes

import pytest
import torch

from bit_error_compensated_echo_b200 import abi
from bit_error_compensated_echo_b200 import workloads as W
from bit_error_compensated_echo_b200.api import EchoPlan
from bit_error_compensated_echo_b200.rank import EchoRankPlan

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _small_call_works():
    w = W.TINY
    with EchoPlan(w.P, w.N, w.G, device=0) as plan:
        x = W.generate(w, 0, DEV)
        y = plan.allreduce(x)
        torch.cuda.synchronize()
        assert torch.equal(y[0].view(torch.int16), y[1].view(torch.int16))


def test_plan_larger_than_the_gpu_returns_oom():
    N = 1 << 34                      # states alone: 2 x 8 x 2^34 x 4 B = 1 TiB
    cfg = abi.echo_config_default()
    cfg.P, cfg.N, cfg.G = 8, N, 128
    assert abi.echo_workspace_bytes(cfg) > 1 << 40
    with pytest.raises(abi.EchoError) as e:
        EchoPlan(8, N, 128, device=0)
    assert e.value.status == abi.ECHO_ERR_OOM
    _small_call_works()


def test_rank_plan_larger_than_the_gpu_returns_oom():
    N = 1 << 37                      # this rank's states: 2 x 2^37 x 4 B = 1 TiB
    with pytest.raises(abi.EchoError) as e:
        EchoRankPlan(8, 0, N, 128, device=0)
    assert e.value.status == abi.ECHO_ERR_OOM
    _small_call_works()


def test_many_plans_created_and_destroyed():
    """Plans release everything they take: 50 create/call/destroy cycles
    leave the device's free memory where it was."""
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    w = W.with_size(W.TINY, P=4, rows=1, hidden=4 * 128 * 64, G=128)
    x = W.generate(w, 0, DEV)
    for i in range(50):
        with EchoPlan(w.P, w.N, w.G, device=0, fixup=("exit", "side", "deferred")[i % 3]) as p:
            p.allreduce(x, side_stream=torch.cuda.current_stream())
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 >= free0 - (8 << 20), (free0, free1)


def test_bounded_wait_runs_out_and_reports():
    """A wait that nothing completes gives up after its limit (about one
    second, not forever), sets ECHO_DEVERR_WAIT_TIMEOUT in the device error
    word, and leaves the context usable."""
    import time
    abi.echo_device_error_get(0, clear=True)
    assert abi.echo_device_error_get(0) == 0
    t0 = time.monotonic()
    abi.echo_selftest_wait_limit(0)
    took = time.monotonic() - t0
    assert 0.9 <= took < 30.0, took
    flags = ctypes.c_int32()
    # the C call reports the run-out wait as ECHO_ERR_TIMEOUT
    assert abi.lib.echo_device_error_get(0, ctypes.byref(flags), 0) == abi.ECHO_ERR_TIMEOUT
    assert flags.value == abi.ECHO_DEVERR_WAIT_TIMEOUT
    assert abi.echo_device_error_get(0, clear=True) == abi.ECHO_DEVERR_WAIT_TIMEOUT
    assert abi.lib.echo_device_error_get(0, ctypes.byref(flags), 0) == abi.ECHO_OK
    assert abi.echo_device_error_get(0) == 0
    _small_call_works()
