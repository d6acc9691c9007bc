"""Seeded synthetic inputs for the decode workloads.

This module only draws random inputs with the shapes and distributions of the
workloads (batch-256 serving shapes of Mamba-2 and Gated DeltaNet layers); it
contains none of the method's arithmetic.  The same tensors feed the CUDA
library and, converted to float64 on the host, the CPU oracle.

Distributions (the pages name the layer kinds and batch 256 but no inputs):
  Mamba-2: x ~ N(0,1); B, C ~ N(0,1)/sqrt(N); dt = softplus(0.5 N(0,1) + dt_bias)
           with dt_bias = softplus^{-1}(u), u log-uniform on [1e-3, 1e-1] per head;
           A = -exp(U(0, ln 16)) per head; D ~ N(0,1) per head.
  GDN:     q, k ~ N(0,1) then L2-normalised per head (in fp32, before the cast);
           v ~ N(0,1); beta = sigmoid(N(0,1));
           alpha = exp(-exp(A_log) softplus(N(0,1) + dt_bias)), A_log ~ U(0, ln 16).
x, B, C, q, k, v are cast to the input dtype (bf16 rounds to nearest even);
dt, alpha, beta stay fp32.
"""
import math

import torch
import torch.nn.functional as F

LN16 = math.log(16.0)


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def dt_bias(H, g, device):
    u = torch.exp(torch.empty(H, device=device).uniform_(math.log(1e-3), math.log(1e-1), generator=g))
    return torch.log(torch.expm1(u))


def mamba2_params(H, seed, device="cpu"):
    """Per-head A, D, dt_bias (fp32)."""
    g = _gen(seed, device)
    A = -torch.exp(torch.empty(H, device=device).uniform_(0.0, LN16, generator=g))
    D = torch.randn(H, device=device, generator=g)
    return A, D, dt_bias(H, g, device)


def gdn_params(H, seed, device="cpu"):
    """Per-head A_log, dt_bias (fp32)."""
    g = _gen(seed, device)
    A_log = torch.empty(H, device=device).uniform_(0.0, LN16, generator=g)
    return A_log, dt_bias(H, g, device)


class Mamba2Stream:
    """Draws T steps at a time: x [T,B,H,P], dt [T,B,H], B, C [T,B,G,N]."""

    def __init__(self, batch, nheads, headdim, dstate, ngroups, dtype, dt_bias_h, seed,
                 device="cpu"):
        self.shape = (batch, nheads, headdim, dstate, ngroups)
        self.dtype = dtype
        self.device = torch.device(device)
        self.dt_bias = dt_bias_h.to(self.device)
        self.g = _gen(seed, self.device)

    def next(self, T):
        Bn, H, P, N, G = self.shape
        g, dev = self.g, self.device
        x = torch.randn(T, Bn, H, P, device=dev, generator=g).to(self.dtype)
        Bm = (torch.randn(T, Bn, G, N, device=dev, generator=g) / math.sqrt(N)).to(self.dtype)
        C = (torch.randn(T, Bn, G, N, device=dev, generator=g) / math.sqrt(N)).to(self.dtype)
        dt = F.softplus(0.5 * torch.randn(T, Bn, H, device=dev, generator=g) + self.dt_bias)
        return {"x": x.contiguous(), "dt": dt.contiguous(), "B": Bm.contiguous(), "C": C.contiguous()}


class GdnStream:
    """Draws T steps at a time: q, k [T,B,H,dk], v [T,B,H,dv], alpha, beta [T,B,H]."""

    def __init__(self, batch, nheads, dk, dv, dtype, A_log_h, dt_bias_h, seed, device="cpu"):
        self.shape = (batch, nheads, dk, dv)
        self.dtype = dtype
        self.device = torch.device(device)
        self.A_log = A_log_h.to(self.device)
        self.dt_bias = dt_bias_h.to(self.device)
        self.g = _gen(seed, self.device)

    def next(self, T):
        Bn, H, dk, dv = self.shape
        g, dev = self.g, self.device
        q = torch.randn(T, Bn, H, dk, device=dev, generator=g)
        q = (q / q.norm(dim=-1, keepdim=True)).to(self.dtype)
        k = torch.randn(T, Bn, H, dk, device=dev, generator=g)
        k = (k / k.norm(dim=-1, keepdim=True)).to(self.dtype)
        v = torch.randn(T, Bn, H, dv, device=dev, generator=g).to(self.dtype)
        beta = torch.sigmoid(torch.randn(T, Bn, H, device=dev, generator=g))
        alpha = torch.exp(-torch.exp(self.A_log) *
                          F.softplus(torch.randn(T, Bn, H, device=dev, generator=g) + self.dt_bias))
        return {"q": q.contiguous(), "k": k.contiguous(), "v": v.contiguous(),
                "alpha": alpha.contiguous(), "beta": beta.contiguous()}


def acceptance(rounds, batch, draft, p_accept, seed, device="cpu"):
    """Leading-success counts a in [0, draft] of Bernoulli(p_accept) draft tokens,
    int32 [rounds, batch]: draft j is accepted only if drafts 0..j all succeed."""
    g = _gen(seed, device)
    ok = torch.rand(rounds, batch, draft, device=device, generator=g) < p_accept
    return torch.cumprod(ok.to(torch.int32), dim=-1).sum(dim=-1).to(torch.int32)


def concat(steps):
    """Concatenate a list of step dicts along T."""
    return {k: torch.cat([s[k] for s in steps], dim=0) for k in steps[0]}


def select_t(d, t0, t1):
    """Steps [t0, t1) of a step dict, contiguous."""
    return {k: v[t0:t1].contiguous() for k, v in d.items()}
