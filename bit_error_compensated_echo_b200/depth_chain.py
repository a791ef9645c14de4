"""Synthetic depth chain: how the all-reduce's error accumulates over sites.

The pages claim that, with every rounding error carried into the calls that
follow, the total error has a bound that does not grow with the number of
layers, provided the network has no direction along which it keeps
magnifying a perturbation (arXiv abstract on the fugumt mirror; ai4snews
news summary, "Interpretation" and "Perspective").  This harness measures that on a
synthetic pre-norm residual chain of tensor-parallel sites, each followed
by the all-reduce of the P ranks' partial products:

    forward  h_{l+1} = h_l + AR( partial_r = RMSNorm(h_l)[:, B_r] @ W_l[B_r, :] )
    backward g <- g + J_RMSNorm(h_l)^T AR( partial_r = g[:, B_r] @ W_l^T[B_r, :] )

with W_l Haar-orthogonal (QR of a Gaussian, signs fixed, seeded 1000 + l),
B_r the r-th block of hidden/P features, RMSNorm with unit weight and
eps = 1e-6, everything else in fp32.  Orthogonal maps and RMSNorm do not
amplify perturbations, which is the bound's assumption.  Five chains run
side by side: the exact chain (fp32 partials summed in fp32), the
compensated 4-bit all-reduce, the uncompensated one, a bf16 all-reduce
(bf16 partials summed in fp32, rounded to bf16), and "promoted": the
compensated all-reduce under the pages' serving policy, the earlier half of
the layers (two sites each) at 8-bit codes and the rest at 4 bits, on one
state (ai4snews news summary, "Perspective").  Per site it reports the
absolute RMS deviation from the exact chain and the relative Frobenius
deviation.

The matrix products, RMSNorm and the residual adds are torch (they stand
in for the model around the all-reduce); the all-reduce is the library's.
The compensated and uncompensated chains each use their own plan (their own
state), separate for the forward and the backward pass.
"""
from __future__ import annotations

from typing import Callable, Dict, List, Optional

import torch

from . import workloads as W
from .api import EchoPlan
from .policy import LayerPolicy

EPS = 1e-6


def haar_orthogonal(n: int, seed: int, device) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    a = torch.randn((n, n), generator=g, dtype=torch.float64)
    q, r = torch.linalg.qr(a)
    q = q * torch.sign(torch.diagonal(r)).unsqueeze(0)
    return q.to(torch.float32).to(device)


def rmsnorm(h: torch.Tensor) -> torch.Tensor:
    return h * torch.rsqrt((h * h).mean(dim=-1, keepdim=True) + EPS)


def rmsnorm_jt(h: torch.Tensor, u: torch.Tensor) -> torch.Tensor:
    """J_RMSNorm(h)^T u, row by row (the Jacobian is symmetric):
    (u - n * <n, u> / d) / rms with n = RMSNorm(h)."""
    d = h.shape[-1]
    inv = torch.rsqrt((h * h).mean(dim=-1, keepdim=True) + EPS)
    n = h * inv
    return (u - n * (n * u).sum(dim=-1, keepdim=True) / d) * inv


def partials(a: torch.Tensor, w: torch.Tensor, P: int, out: torch.Tensor) -> torch.Tensor:
    """out[r] = a[:, B_r] @ w[B_r, :] for the P feature blocks B_r (fp32)."""
    d = a.shape[-1]
    blk = d // P
    for r in range(P):
        torch.matmul(a[:, r * blk:(r + 1) * blk], w[r * blk:(r + 1) * blk, :], out=out[r])
    return out


class _Chain:
    def __init__(self, name, h0, plan=None):
        self.name, self.h, self.plan = name, h0.clone(), plan


def _ar(kind: str, parts32: torch.Tensor, plan, buf_bf16, out_bf16, bits=None,
        seen=None) -> torch.Tensor:
    """The site's all-reduce of the P partials ([P, T, D] fp32) -> [T, D] fp32.
    seen(plan, x, y) is called after a library call with its [P, N] bf16
    inputs and outputs."""
    if kind == "exact":
        return parts32.sum(dim=0)
    buf_bf16.copy_(parts32)
    if kind == "bf16":
        return buf_bf16.float().sum(dim=0).to(torch.bfloat16).float()
    P = parts32.shape[0]
    x, y = buf_bf16.view(P, -1), out_bf16.view(P, -1)
    plan.allreduce(x, out=y, bits=bits)
    if seen is not None:
        seen(plan, x, y)
    return out_bf16[0].float()


def _dev(h, ref):
    diff = (h - ref).double()
    return (float(diff.pow(2).mean().sqrt()),
            float(diff.norm() / ref.double().norm().clamp_min(1e-30)))


def run(P: int = 8, tokens: int = 32768, hidden: int = 1024, sites: int = 56, G: int = 128,
        seed: int = 3, device: str = "cuda", backward: bool = True,
        observer: Optional[Callable] = None) -> Dict[str, Dict[str, List[float]]]:
    """Run the five chains; returns {pass: {chain: [rms per site]}, ...}.

    observer, if given, is called as observer(direction, site, chain, plan,
    x, y) right after every call of the library's all-reduce (chains comp,
    off and promoted), with the call's plan and its [P, N] bf16 inputs and
    outputs, before anything else touches them; the plan of a chain is the
    same object from its first site to its last within one direction.  It
    lets a caller inspect each call (e.g. check it against a reference)."""
    dev = torch.device(device)
    wl = W.Workload("depth", P=1, rows=tokens, hidden=hidden, G=G, seed=seed, dist="student_t")
    h0 = W.generate(wl, 0, dev)[0].view(tokens, hidden).float()
    N = tokens * hidden
    parts = torch.empty((P, tokens, hidden), dtype=torch.float32, device=dev)
    buf = torch.empty((P, tokens, hidden), dtype=torch.bfloat16, device=dev)
    out = torch.empty_like(buf)
    res: Dict[str, Dict[str, List[float]]] = {}
    policy = LayerPolicy(max(1, sites // 2), 2, 0.5)

    def one_pass(direction: str, start: torch.Tensor, ws, h_exact_fwd=None):
        d = dev.index or 0
        plans = {"comp": EchoPlan(P, N, G, compensate=True, device=d, fixup="deferred"),
                 "off": EchoPlan(P, N, G, compensate=False, device=d),
                 "promoted": EchoPlan(P, N, G, compensate=True, device=d, fixup="deferred",
                                      bits=8)}
        chains = [_Chain("exact", start), _Chain("comp", start, plans["comp"]),
                  _Chain("off", start, plans["off"]), _Chain("bf16", start),
                  _Chain("promoted", start, plans["promoted"])]
        rms = {c.name: [] for c in chains if c.name != "exact"}
        rel = {c.name: [] for c in chains if c.name != "exact"}
        try:
            for step, wmat in enumerate(ws):
                # the site's position in the forward order sets its layer's width
                site = step if direction == "forward" else len(ws) - 1 - step
                for c in chains:
                    bits = policy.bits_for_site(site) if c.name == "promoted" else None
                    seen = None
                    if observer is not None:
                        def seen(plan, x, y, _name=c.name, _site=site):
                            observer(direction, _site, _name, plan, x, y)
                    if direction == "forward":
                        partials(rmsnorm(c.h), wmat, P, parts)
                        c.h = c.h + _ar(c.name, parts, c.plan, buf, out, bits, seen)
                    else:
                        partials(c.h, wmat.t().contiguous(), P, parts)
                        u = _ar(c.name, parts, c.plan, buf, out, bits, seen)
                        c.h = c.h + rmsnorm_jt(h_exact_fwd[len(ws) - 1 - step], u)
                ref = chains[0].h
                for c in chains[1:]:
                    a, b = _dev(c.h, ref)
                    rms[c.name].append(a)
                    rel[c.name].append(b)
        finally:
            for p in plans.values():
                p.close()
        return chains[0].h, rms, rel

    ws = [haar_orthogonal(hidden, 1000 + l, dev) for l in range(1, sites + 1)]
    # exact forward activations per site, for the backward Jacobians
    h_ex = [h0.clone()]
    for wmat in ws[:-1]:
        partials(rmsnorm(h_ex[-1]), wmat, P, parts)
        h_ex.append(h_ex[-1] + parts.sum(dim=0))
    _, rms_f, rel_f = one_pass("forward", h0, ws)
    res["forward_rms"], res["forward_rel"] = rms_f, rel_f
    if backward:
        wg = W.Workload("depth_grad", P=1, rows=tokens, hidden=hidden, G=G, seed=seed + 100,
                        dist="student_t")
        g0 = W.generate(wg, 0, dev)[0].view(tokens, hidden).float()
        _, rms_b, rel_b = one_pass("backward", g0, list(reversed(ws)), h_exact_fwd=h_ex)
        res["backward_rms"], res["backward_rel"] = rms_b, rel_b
    return res
