"""The rank path through NCCL: tests/rank_nccl_worker.py under
torch.distributed.run, one rank per visible GPU (one on a one-GPU machine,
where the exchanges are NCCL's single-rank all-to-all and all-gather)."""
import os
import socket
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_rank_group_over_nccl():
    n = max(1, min(torch.cuda.device_count(), 8))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node=%d" % n, "--master-addr", "127.0.0.1",
           "--master-port", str(_free_port()), os.path.join(HERE, "rank_nccl_worker.py")]
    env = dict(os.environ, NCCL_NVLS_ENABLE="0")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert r.stdout.count("all calls equal") == n
