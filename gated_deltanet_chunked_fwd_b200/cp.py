"""Context parallelism across GPUs: one long sequence whose tokens are sharded over the ranks of
a process group (dothoosh.com FlashQLA article, first innovation: gate-driven context
parallelism, which splits long sequences automatically among processing units; its
million-token paragraph).

Rank r holds the r-th contiguous shard of the sequence's tokens, every head.  A shard needs the
state the sequence carries into it; there are two ways to get it (per value head, the state
stored as H = S^T, [dk, dv]):

* gate-driven (``mode="halo"``): rank r > 0 starts a halo of the previous shard's last
  ``halo_chunks`` chunks early, from a zero state.  While the halo's summed log decay is at most
  log(2^-30) and every halo token keeps 0 <= beta |k|^2 <= 2, each token's state map has norm
  <= exp(g_t), so the truncated past changes the shard's entry state by at most 2^-30 |H|.  The
  only exchange is the halo tokens; one forward call per rank.
* exact (``mode="exact"``): the tokens of shard j map its entry state affinely,
  H_exit = M_j H_entry + B_j (M_j = the product of the tokens' maps, dk x dk; B_j = the exit
  state from a zero entry).  Every rank forms (M_j, B_j) with two forward calls (B: S0 = 0;
  M: v = 0 and S0 = [I | 0], which needs dv >= dk), the folds are all-gathered, and rank r
  folds shards 0..r-1 onto S0 in order, X <- M_j X + B_j (``gdn_affine_combine``), then runs its
  shard from X.  Exact up to the arithmetic of the forward itself.
* ``mode="auto"`` takes the halo where every rank's halo passes ``gdn_halo_check`` (a decision
  all ranks reach together through one all-reduce), else the exact way.

The collectives (all-gather of the halos or the folds, an all-reduce of the decision, a
broadcast of the final state) run on ``torch.distributed`` (NCCL between GPUs) through
``TorchComm``; every rank takes the same collective steps in the same order.  The compute steps
are the library's CUDA kernels (``ops=None``).  ``comm`` and ``ops`` are parameters so that the
same rank protocol can run with other collectives (ranks as host threads sharing one GPU) or
other compute (CPU processes).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Callable, Optional

import torch

LOG_EPS = -30.0 * math.log(2.0)  # the forward's warm-up bound: summed log decay <= log(2^-30)


@dataclass
class CpOps:
    """The three compute steps of the protocol.

    fwd(q, k, v, beta, g, S0, flags) -> (o, S_T): a forward call of one shard ([1, T, ...]).
    combine(M, X, B) -> X: X <- M X + B for every value head (M [1, Hv, dk, dk]).
    halo_ok(k, beta, g, log_eps, flags) -> bool: every value head of the halo passes.
    """

    fwd: Callable
    combine: Callable
    halo_ok: Callable


def cuda_ops() -> CpOps:
    """The library's kernels (the default)."""
    from . import gdn_affine_combine, gdn_chunk_fwd, gdn_halo_check

    def fwd(q, k, v, beta, g, S0, flags):
        return gdn_chunk_fwd(q, k, v, beta, g, initial_state=S0, flags=flags)

    def combine(M, X, B):
        return gdn_affine_combine(M, X, B)

    def halo_ok(k, beta, g, log_eps, flags):
        ok = gdn_halo_check(k[0], beta[0], g[0], log_eps, flags=flags)
        return bool(int(ok.min().item()) == 1)  # one small device-to-host read

    return CpOps(fwd, combine, halo_ok)


class TorchComm:
    """The collectives of the protocol on a ``torch.distributed`` process group."""

    def __init__(self, group=None):
        import torch.distributed as dist

        self.dist, self.group = dist, group
        self.rank, self.world = dist.get_rank(group), dist.get_world_size(group)

    def _global(self, r):
        return r if self.group is None else self.dist.get_global_rank(self.group, r)

    def all_gather(self, t: torch.Tensor) -> list:
        out = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(out, t.contiguous(), group=self.group)
        return out

    def all_reduce(self, x: int, op: str, device) -> int:
        t = torch.tensor([int(x)], dtype=torch.int64, device=device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MIN if op == "min" else self.dist.ReduceOp.MAX,
                             group=self.group)
        return int(t.item())

    def broadcast(self, t: torch.Tensor, src: int) -> torch.Tensor:
        self.dist.broadcast(t, src=self._global(src), group=self.group)
        return t


def cp_chunk_fwd(q, k, v, beta, g, *, group=None, initial_state: Optional[torch.Tensor] = None,
                 mode: str = "auto", halo_chunks: int = 4, flags: int = 0, ops: Optional[CpOps] = None,
                 comm=None):
    """Forward of one long sequence sharded over the ranks of ``group`` (rank order = token
    order).  Every rank passes its shard: q, k [1, T_r, Hk, dk]; v [1, T_r, Hv, dv]; beta, g
    [1, T_r, Hv] fp32 (T_r >= 1, shards of any lengths).  ``initial_state`` (fp32
    [1, Hv, dk, dv], H = S^T layout) is read on rank 0 only.

    Returns (o_r [1, T_r, Hv, dv], S_T [1, Hv, dk, dv] of the whole sequence (on every rank),
    the mode taken: "halo" or "exact").  mode "halo" raises if some halo fails the check
    (or some shard is shorter than the halo); "auto" then takes the exact way.
    """
    if mode not in ("auto", "halo", "exact"):
        raise ValueError("mode must be 'auto', 'halo' or 'exact'")
    if q.dim() != 4 or q.shape[0] != 1 or q.shape[1] < 1:
        raise ValueError("each rank passes one non-empty shard: q [1, T_r, Hk, dk]")
    ops = ops if ops is not None else cuda_ops()
    comm = comm if comm is not None else TorchComm(group)
    world, rank = comm.world, comm.rank
    dev = q.device
    T_r = q.shape[1]
    Hv, dk, dv = v.shape[2], q.shape[3], v.shape[3]
    h = halo_chunks * 64

    if world == 1:
        o, ST = ops.fwd(q, k, v, beta, g, initial_state, flags)
        return o, ST, "exact"

    # ---- the gate-driven way, where it holds on every rank
    use_halo = False
    if mode in ("auto", "halo") and halo_chunks > 0:
        lens = comm.all_gather(torch.tensor([T_r], dtype=torch.int64, device=dev))
        if min(int(x.item()) for x in lens[:-1]) >= h:  # every shard that feeds a halo is long enough
            if T_r >= h:
                tail = [x[:, T_r - h:] for x in (q, k, v, beta, g)]
            else:  # the last shard feeds no halo; it still takes part in the gather
                tail = [torch.zeros((1, h) + tuple(x.shape[2:]), dtype=x.dtype, device=dev)
                        for x in (q, k, v, beta, g)]
            halos = [comm.all_gather(x) for x in tail]
            prev = [x[rank - 1] for x in halos] if rank > 0 else None
            ok = 1 if rank == 0 else int(ops.halo_ok(prev[1], prev[3], prev[4], LOG_EPS, flags))
            use_halo = comm.all_reduce(ok, "min", dev) == 1
        if mode == "halo" and not use_halo:
            raise RuntimeError("cp_chunk_fwd: a halo fails the decay / norm check, or a shard is "
                               "shorter than the halo; use mode='auto' or 'exact'")
    if use_halo:
        if rank == 0:
            o, ST = ops.fwd(q, k, v, beta, g, initial_state, flags)
        else:
            cat = [torch.cat([p, x], dim=1).contiguous() for p, x in zip(prev, (q, k, v, beta, g))]
            o_ext, ST = ops.fwd(*cat, None, flags)
            o = o_ext[:, h:].contiguous()
        taken = "halo"
    else:
        # ---- the exact way: folds, all-gathered, combined in order
        if dv < dk:
            raise ValueError("the exact way forms M from S0 = [I | 0] and needs dv >= dk")
        _, B_r = ops.fwd(q, k, v, beta, g, None, flags)
        eye = torch.zeros(1, Hv, dk, dv, dtype=torch.float32, device=dev)
        eye[..., torch.arange(dk), torch.arange(dk)] = 1.0
        _, MI = ops.fwd(q, k, torch.zeros_like(v), beta, g, eye, flags)
        M_r = MI[..., :dk].contiguous()
        Ms = comm.all_gather(M_r)
        Bs = comm.all_gather(B_r.contiguous())
        has0 = comm.all_reduce(1 if (rank == 0 and initial_state is not None) else 0, "max", dev)
        X = torch.zeros(1, Hv, dk, dv, dtype=B_r.dtype, device=dev)
        if has0:
            if rank == 0:
                X.copy_(initial_state)
            X = comm.broadcast(X, 0)
        for j in range(rank):
            X = ops.combine(Ms[j], X, Bs[j])
        o, ST = ops.fwd(q, k, v, beta, g, X if rank > 0 or has0 else None, flags)
        taken = "exact"

    # ---- the sequence's final state: the last rank's
    ST = comm.broadcast(ST.contiguous(), world - 1)
    return o, ST, taken
