"""Seeded synthetic inputs for the five workloads, shared by the tests, the
benchmark and the oracle checks.  This module holds no arithmetic of the
method: it only draws bf16 tensors.

Shapes and distributions follow the settings on the pages (ai4snews news
summary, "Perspective": Llama-3-8B and Qwen3-8B served at TP=8, Qwen3-0.6B
pretrained at TP=8; "Interpretation": 1 GB messages), used as shapes only:
no weights, no datasets.

Every call t of workload w draws from its own generator seeded with
``w.seed * 1_000_003 + t`` on the requested device, in fp32, then rounds to
bf16 (round to nearest even).  The oracle and the GPU always receive the
same bf16 bytes: tests copy the generated tensor's bytes to the host.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import List, Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    P: int          # virtual ranks
    rows: int       # tokens
    hidden: int     # hidden size; rows*hidden = N elements per rank
    G: int          # group size
    seed: int
    dist: str       # normal | llama_outliers | sparse_outliers | student_t
    sigma: float = 1.0
    calls: int = 1
    compensate: bool = True
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def N(self) -> int:
        return self.rows * self.hidden

    @property
    def input_bytes(self) -> int:
        return 2 * self.P * self.N


# 1: tiny correctness case, 16 calls, compensator on and off
TINY = Workload("tiny_p2_n4096_g32", P=2, rows=1, hidden=4096, G=32, seed=0,
                dist="normal", calls=16)
# 2: Llama-3-8B TP activations: 2048 tokens x 4096 hidden per rank,
#    N(0,1) with 8 fixed outlier hidden channels x50, 64 calls (2 per layer
#    x 32 layers) sharing one state
LLAMA = Workload("llama3_8b_tp8_2048x4096_g128", P=8, rows=2048, hidden=4096, G=128,
                 seed=1, dist="llama_outliers", calls=64)
# 3: 1 GiB per rank (2^29 bf16), N(0, 0.5^2)
LARGE = Workload("large_p8_1gib_g128", P=8, rows=131072, hidden=4096, G=128, seed=2,
                 dist="normal", sigma=0.5, calls=4)
# 4: depth chain, Qwen3-0.6B-like: 32768 tokens x 1024 hidden, Student-t nu=3,
#    56 all-reduce sites (28 layers x 2)
DEPTH = Workload("depth_chain_p8_32768x1024_g128", P=8, rows=32768, hidden=1024, G=128,
                 seed=3, dist="student_t", calls=56)

SWEEP_MIB = (1, 4, 16, 64, 256, 1024)
SWEEP_P = (2, 4, 8)
SWEEP_G = (32, 64, 128)


def sweep_point(mib: int, P: int, G: int, compensate: bool) -> Workload:
    """5: one sweep point: mib MiB of bf16 per rank, N(0,1) with 0.1% of the
    elements (fresh per call) scaled x30."""
    n = mib * (1 << 20) // 2
    return Workload("sweep_%dmib_p%d_g%d_%s" % (mib, P, G, "comp" if compensate else "off"),
                    P=P, rows=n // 4096 if n >= 4096 else 1, hidden=4096 if n >= 4096 else n,
                    G=G, seed=4, dist="sparse_outliers", calls=1, compensate=compensate)


def sweep() -> List[Workload]:
    return [sweep_point(m, P, G, c) for m in SWEEP_MIB for P in SWEEP_P for G in SWEEP_G
            for c in (True, False)]


def with_size(w: Workload, P: Optional[int] = None, rows: Optional[int] = None,
              hidden: Optional[int] = None, G: Optional[int] = None) -> Workload:
    return replace(w, P=P or w.P, rows=rows or w.rows, hidden=hidden or w.hidden, G=G or w.G)


def call_seed(seed: int, call: int) -> int:
    return seed * 1_000_003 + call


def outlier_channels(hidden: int, count: int = 8) -> torch.Tensor:
    """The fixed outlier hidden channels of the Llama-shaped workload:
    chosen once from seed 0, the same for every rank and call."""
    g = torch.Generator(device="cpu")
    g.manual_seed(0)
    return torch.randperm(hidden, generator=g)[:count]


def _student_t(shape, nu: int, g: torch.Generator, device) -> torch.Tensor:
    z = torch.randn(shape, generator=g, device=device)
    v = torch.zeros(shape, device=device)
    for _ in range(nu):
        v += torch.randn(shape, generator=g, device=device) ** 2
    return z / torch.sqrt(v / nu)


def generate(w: Workload, call: int = 0, device="cpu", out: Optional[torch.Tensor] = None
             ) -> torch.Tensor:
    """[P, N] bf16 inputs of call ``call`` of workload ``w``, drawn rank by
    rank (fp32 then rounded to bf16) on ``device``."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(call_seed(w.seed, call))
    if out is None:
        out = torch.empty((w.P, w.N), dtype=torch.bfloat16, device=device)
    chans = outlier_channels(w.hidden).to(device) if w.dist == "llama_outliers" else None
    for r in range(w.P):
        if w.dist == "normal":
            x = torch.randn(w.N, generator=g, device=device) * w.sigma
        elif w.dist == "llama_outliers":
            x = torch.randn((w.rows, w.hidden), generator=g, device=device)
            x[:, chans] *= 50.0
        elif w.dist == "sparse_outliers":
            x = torch.randn(w.N, generator=g, device=device)
            mask = torch.rand(w.N, generator=g, device=device) < 0.001
            x = torch.where(mask, x * 30.0, x)
        elif w.dist == "student_t":
            x = _student_t((w.N,), 3, g, device) * w.sigma
        else:
            raise ValueError(w.dist)
        out[r].copy_(x.reshape(-1).to(torch.bfloat16))
        del x
    return out


def bf16_bits(t: torch.Tensor):
    """Host numpy uint16 view of a bf16 tensor's bytes."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def column_sample(w: Workload, count: int, seed: int = 12345):
    """Sorted group-column ids: the first, the last and ``count`` distinct
    random ones (for sampled checks of large calls)."""
    import numpy as np
    ncols = w.N // w.G
    rng = np.random.default_rng(seed)
    pick = rng.choice(ncols, size=min(count, ncols), replace=False)
    return np.unique(np.concatenate([pick, [0, ncols - 1]])).astype(np.int64)


def column_elements(cols, G: int):
    """Element indices of the listed group columns, in order."""
    import numpy as np
    cols = np.asarray(cols, np.int64)
    return (cols[:, None] * G + np.arange(G)[None, :]).reshape(-1)
