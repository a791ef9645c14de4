"""One rank of a real group over NCCL (run under torch.distributed.run):
EchoRankPlan.allreduce / reduce_scatter through TorchDistTransport, and
allreduce_peers / reduce_scatter_peers over the fused transport (windows
mapped with CUDA IPC, a one-element NCCL all-reduce as the barrier), against
the plan of P virtual ranks that every rank also runs on the whole group's
input.  Exits non-zero on the first difference.  Usable with any number of
GPUs, one rank each; the single-GPU test suite runs it with one rank."""
import os
import sys

import torch
import torch.distributed as dist

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from bit_error_compensated_echo_b200 import workloads as W  # noqa: E402
from bit_error_compensated_echo_b200.api import EchoPlan  # noqa: E402
from bit_error_compensated_echo_b200.rank import (EchoRankPlan, PeerWindows,  # noqa: E402
                                                  TorchDistBarrier, TorchDistTransport,
                                                  init_process_group)


def bits_equal(a, b):
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


def run_case(transport, P, rank, local, dev, G, k, fixup, bits, bad):
    N = P * G * k
    w = W.with_size(W.TINY, P=P, rows=1, hidden=N, G=G)
    side = torch.cuda.Stream(dev) if fixup == "side" else None
    t_port = TorchDistTransport()
    with EchoRankPlan(P, rank, N, G, device=local, fixup=fixup, bits=bits) as plan, \
            EchoPlan(P, N, G, device=local, fixup=fixup, bits=bits) as virt:
        win = PeerWindows.exchange(plan) if transport == "peers" else None
        barrier = TorchDistBarrier(dev)
        try:
            for t, op in enumerate("AARAR"):
                x = W.generate(w, t, dev)
                xr = x[rank].contiguous()
                if op == "A" and win is not None:
                    y = plan.allreduce_peers(xr, win, barrier, side_stream=side)
                elif op == "A":
                    y = plan.allreduce(xr, t_port, side_stream=side)
                elif win is not None:
                    y = plan.reduce_scatter_peers(xr, win, barrier, side_stream=side)
                else:
                    y = plan.reduce_scatter(xr, t_port, side_stream=side)
                yv = (virt.allreduce(x, side_stream=side) if op == "A"
                      else virt.reduce_scatter(x, side_stream=side))[rank]
                mf, ms = plan.get_state()
                mfv, msv = virt.get_state()
                torch.cuda.synchronize(dev)
                for name, a, b in (("output", y, yv), ("m_fast", mf, mfv[rank]),
                                   ("m_slow", ms, msv[rank])):
                    if not bits_equal(a, b):
                        bad.append("%s G=%d %s bits=%d call %d (%s): %s differs"
                                   % (transport, G, fixup, bits, t, op, name))
        finally:
            if win is not None:
                # no rank unmaps, and no owner frees, a window a peer still reads
                torch.cuda.synchronize(dev)
                dist.barrier()
                win.close()
                dist.barrier()


def main():
    local = init_process_group("nccl", timeout_s=120.0)
    rank, P = dist.get_rank(), dist.get_world_size()
    dev = torch.device("cuda", local)
    bad = []
    try:
        for transport in ("copies", "peers"):
            for G, k, fixup, bits in ((64, 24, "deferred", 4), (32, 40, "exit", 4),
                                      (128, 8, "side", 8)):
                run_case(transport, P, rank, local, dev, G, k, fixup, bits, bad)
        dist.barrier()
    finally:
        dist.destroy_process_group()
    if bad:
        print("rank %d: %s" % (rank, "; ".join(bad[:5])), file=sys.stderr)
        sys.exit(1)
    print("rank %d of %d: all calls equal" % (rank, P))


if __name__ == "__main__":
    main()
