"""Seeded synthetic inputs for the GDN chunked prefill, shared by the oracle side
and the CUDA side of every test and of the bench.

This module holds none of the layer's arithmetic: it only draws random tensors
with the shapes and value distributions of the workloads below and returns
them.  Both the oracle and the CUDA path consume exactly these tensors (the
oracle after an exact upcast to float64), so a parity check measures kernel
error, not input rounding.

Distributions (the FlashQLA pages print no workload; these are the standard
GDN-prefill shapes used throughout this repository):
  q, k ~ N(0, 1), then L2-normalised per head vector in fp32: x / max(|x|, 1e-6)
  v    ~ N(0, 1)
  beta = sigmoid(N(0, 1))                       (fp32)
  g    = -softplus(N(mu_g, 1))  (log decay <= 0; mu_g = 0, or -2 for slow decay)
  S0   ~ s0_std * N(0, 1) in fp32, or absent (zero state)
  do   ~ N(0, 1), dST ~ 0.1 * N(0, 1)           (backward workloads)
Draw order from one torch CPU Generator seeded with ``seed``:
  [varlen lengths] -> q -> k -> v -> beta logits -> g logits -> S0 -> do -> dST.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch

DTYPES = {"fp32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str
    B: int
    T: int  # per-sequence length (fixed-length), or 0 for varlen
    Hk: int
    Hv: int
    dk: int
    dv: int
    s0_std: Optional[float] = None
    g_mu: float = 0.0
    varlen: Optional[tuple] = None  # (num_seqs, lo, hi) lengths ~ U[lo, hi]
    backward: bool = False
    chained_calls: int = 1
    notes: str = ""


WORKLOADS = [
    Workload("fwd_fp32_T256_H2_d64", "fp32", 1, 256, 2, 2, 64, 64,
             notes="small fp32 forward, zero initial state"),
    Workload("fwd_bf16_T4096_H16_d128", "bf16", 1, 4096, 16, 16, 128, 128, s0_std=0.1,
             notes="bf16 forward with a random fp32 initial state"),
    Workload("fwd_bf16_varlen8_Hk16_Hv32_d128", "bf16", 1, 0, 16, 32, 128, 128,
             varlen=(8, 512, 16384),
             notes="packed batch of 8 sequences, grouped value heads (2 v heads per q/k head)"),
    Workload("fwd_bf16_T65536_H16_d128_slowdecay", "bf16", 1, 65536, 16, 16, 128, 128, g_mu=-2.0,
             chained_calls=4, notes="long context; also run as 4 chained 16384-token calls"),
    Workload("bwd_bf16_B4_T8192_H16_d128", "bf16", 4, 8192, 16, 16, 128, 128, backward=True,
             notes="backward with do ~ N(0,1) and dST ~ 0.1 N(0,1)"),
]


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    n = x.float().norm(dim=-1, keepdim=True).clamp_min(1e-6)
    return x.float() / n


def make_inputs(B, T, Hk, Hv, dk, dv, dtype="bf16", seed=0, s0_std=None, g_mu=0.0,
                lengths=None, varlen=None, backward=False, device="cpu"):
    """Draw one batch.  Returns a dict of tensors on ``device``.

    Fixed-length: q/k [B,T,Hk,dk], v [B,T,Hv,dv], beta/g [B,T,Hv].
    Varlen (``lengths`` given, or ``varlen=(n, lo, hi)`` drawn first): B = 1,
    T = sum(lengths), plus ``cu_seqlens`` int32 [n+1].
    """
    gen = torch.Generator().manual_seed(seed)
    cu = None
    if varlen is not None and lengths is None:
        n, lo, hi = varlen
        lengths = torch.randint(lo, hi + 1, (n,), generator=gen).tolist()
    if lengths is not None:
        B, T = 1, int(sum(lengths))
        cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    dt = DTYPES[dtype]
    q = _l2norm(torch.randn(B, T, Hk, dk, generator=gen)).to(dt)
    k = _l2norm(torch.randn(B, T, Hk, dk, generator=gen)).to(dt)
    v = torch.randn(B, T, Hv, dv, generator=gen).to(dt)
    beta = torch.sigmoid(torch.randn(B, T, Hv, generator=gen))
    g = -torch.nn.functional.softplus(torch.randn(B, T, Hv, generator=gen) + g_mu)
    N = B if cu is None else cu.numel() - 1
    S0 = None
    if s0_std is not None:
        S0 = s0_std * torch.randn(N, Hv, dk, dv, generator=gen)
    out = dict(q=q, k=k, v=v, beta=beta, g=g, cu_seqlens=cu, initial_state=S0)
    if backward:
        out["do"] = torch.randn(B, T, Hv, dv, generator=gen).to(dt)
        out["dST"] = 0.1 * torch.randn(N, Hv, dk, dv, generator=gen)
    if device != "cpu":
        out = {k_: (t.to(device) if isinstance(t, torch.Tensor) else t) for k_, t in out.items()}
        if cu is not None:
            out["cu_seqlens_host"] = cu.clone()
    elif cu is not None:
        out["cu_seqlens_host"] = cu
    return out


def make_workload(index_or_name, seed=0, device="cpu", **overrides):
    """Inputs for one of ``WORKLOADS`` (by index or name); keyword overrides
    (e.g. ``T=1024``) shrink a shape for a sampled check."""
    w = WORKLOADS[index_or_name] if isinstance(index_or_name, int) else \
        next(x for x in WORKLOADS if x.name == index_or_name)
    kw = dict(B=w.B, T=w.T, Hk=w.Hk, Hv=w.Hv, dk=w.dk, dv=w.dv, dtype=w.dtype, seed=seed,
              s0_std=w.s0_std, g_mu=w.g_mu, varlen=w.varlen, backward=w.backward)
    kw.update(overrides)
    return make_inputs(device=device, **kw)
