"""Helpers of the context-parallel tests: ranks as host threads (collectives through a barrier)
and the float64 oracle as the compute steps of the rank protocol on CPU."""
import threading

import numpy as np
import torch

import oracle
from gated_deltanet_chunked_fwd_b200 import GDN_FLAG_GATE_LOGITS, GDN_FLAG_QK_L2NORM
from gated_deltanet_chunked_fwd_b200.cp import CpOps


class ThreadComm:
    """Collectives between ranks that are threads of one process: every rank deposits its value,
    all wait at a barrier, all read, all wait again.  On one GPU all ranks enqueue on the same
    stream, so a tensor deposited by one rank is complete before another rank's later work
    reads it; no kernel ever waits for another."""

    def __init__(self, rank, world, shared):
        self.rank, self.world, self.s = rank, world, shared

    def _exchange(self, x):
        self.s["slots"][self.rank] = x
        self.s["barrier"].wait()
        vals = list(self.s["slots"])
        self.s["barrier"].wait()
        return vals

    def all_gather(self, t):
        return [x.clone() for x in self._exchange(t.clone())]

    def all_reduce(self, x, op, device):
        vals = self._exchange(int(x))
        return min(vals) if op == "min" else max(vals)

    def broadcast(self, t, src):
        vals = self._exchange(t.clone() if self.rank == src else None)
        if self.rank != src:
            t.copy_(vals[src])
        return t


def run_ranks(world, fn, timeout=300):
    """fn(rank, comm) on `world` threads; returns the results by rank (re-raises a rank's error)."""
    shared = {"slots": [None] * world, "barrier": threading.Barrier(world, timeout=timeout)}
    out, errs = [None] * world, [None] * world

    def body(r):
        try:
            out[r] = fn(r, ThreadComm(r, world, shared))
        except BaseException as e:  # noqa: BLE001 - handed to the caller
            errs[r] = e
            shared["barrier"].abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout)
    for e in errs:
        if e is not None and not isinstance(e, threading.BrokenBarrierError):
            raise e
    for e in errs:
        if e is not None:
            raise e
    return out


def f64(x):
    return x.detach().cpu().double().numpy() if hasattr(x, "detach") else np.asarray(x, np.float64)


def halo_ok_f64(k, beta, g, log_eps, flags=0):
    """Per value head: summed log decay <= log_eps and 0 <= beta |k|^2 <= 2 on every token
    (k [T, Hk, dk], beta / g [T, Hv]), in float64, with the forward's preprocessing."""
    k, beta, g = f64(k), f64(beta), f64(g)
    if flags & GDN_FLAG_GATE_LOGITS:
        beta = 1.0 / (1.0 + np.exp(-beta))
        g = -np.logaddexp(0.0, g)
    Hk, Hv = k.shape[1], beta.shape[1]
    nk = (k * k).sum(-1)  # [T, Hk]
    if flags & GDN_FLAG_QK_L2NORM:
        nk = nk / np.maximum(np.sqrt(nk), oracle.L2_EPS) ** 2
    nk = np.repeat(nk, Hv // Hk, axis=1)
    norm_ok = np.all((beta >= 0) & (beta * nk <= 2.0), axis=0)
    return (g.sum(0) <= log_eps) & norm_ok if k.shape[0] > 0 else np.zeros(Hv, bool)


def oracle_ops():
    """The three compute steps in float64 on CPU (test stand-ins for the CUDA kernels)."""

    def fwd(q, k, v, beta, g, S0, flags):
        o, ST = oracle.fwd(q, k, v, beta, g, initial_state=S0, qk_l2norm=bool(flags & GDN_FLAG_QK_L2NORM),
                           gate_logits=bool(flags & GDN_FLAG_GATE_LOGITS))
        return torch.from_numpy(o), torch.from_numpy(ST)

    def combine(M, X, B):
        return torch.from_numpy(np.einsum("nhij,nhjk->nhik", f64(M), f64(X)) + f64(B))

    def halo_ok(k, beta, g, log_eps, flags):
        return bool(halo_ok_f64(k[0], beta[0], g[0], log_eps, flags).all())

    return CpOps(fwd, combine, halo_ok)


def shards(x, cuts):
    """Split every [1, T, ...] tensor of x at the token offsets `cuts` (0 < c < T)."""
    edges = [0] + list(cuts) + [x["q"].shape[1]]
    return [{n: x[n][:, a:b].contiguous() for n in ("q", "k", "v", "beta", "g")} for a, b in zip(edges, edges[1:])]
