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
This file is collected last on purpose; it passes alone or after the
other tests.
"""
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


# N above and below 2^19 per rank: the call with and without the exit pass
@pytest.mark.parametrize("P,G,k,comp", [(8, 128, 70, True), (3, 32, 41, True),
                                        (4, 64, 33, False), (8, 128, 600, True)])
def test_noalloc_matches_plan_two_calls(P, G, k, comp):
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    cfg = abi.echo_config_default()
    cfg.P, cfg.G, cfg.N, cfg.compensate, cfg.device = P, G, N, int(comp), 0
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


def test_noalloc_largest_supported_and_rejected_sizes():
    """8 ranks of 2048 x 4096 with the compensator fit the fixed scratch;
    1 GiB per rank does not and is refused before anything is launched."""
    small = abi.echo_config_default()
    small.P, small.G, small.N = 8, 128, 2048 * 4096
    q = 0.5 + 4 / 128
    need = 8 * small.N * q + small.N * q + 4 * small.N
    assert need <= abi.ECHO_NOALLOC_MAX_SCRATCH_BYTES
    big = abi.echo_config_default()
    big.P, big.G, big.N = 8, 128, 1 << 29
    buf = torch.empty(64, dtype=torch.bfloat16, device=DEV)
    st = torch.empty(64, dtype=torch.float32, device=DEV)
    with pytest.raises(abi.EchoError) as e:
        abi.echo_allreduce_noalloc(big, [buf.data_ptr()] * 8, [buf.data_ptr()] * 8,
                                   st.data_ptr(), st.data_ptr(), 0)
    assert e.value.status == abi.ECHO_ERR_UNSUPPORTED
    with pytest.raises(abi.EchoError) as e:  # missing state with the compensator on
        abi.echo_allreduce_noalloc(small, [buf.data_ptr()] * 8, [buf.data_ptr()] * 8, 0, 0, 0)
    assert e.value.status == abi.ECHO_ERR_INVALID_ARG
