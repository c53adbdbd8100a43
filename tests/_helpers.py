"""Helpers shared by the GPU parity tests: rel-L2 and oracle runs on sampled units."""
import numpy as np
import torch

import oracle

# rel-L2 bars: 1e-2 for bf16 tensors (bf16 operands into fp32 accumulation),
# 1e-4 for fp32 tensors (fp32 throughout; no tensor-core shortcut)
TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-4}


def rel_l2(x, ref) -> float:
    x = np.asarray(x.detach().cpu().double().numpy() if hasattr(x, "detach") else x, dtype=np.float64)
    ref = np.asarray(ref.detach().cpu().double().numpy() if hasattr(ref, "detach") else ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 0 else float(num)


def cpu(d):
    return {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def oracle_fwd_units(inp, units):
    """Oracle forward on selected (sequence, value head) units.

    Returns {(n, h): (o [len, dv], S_T [dk, dv])}, each unit run alone (its own
    sequence slice and its own q/k head), from the same rounded inputs."""
    x = cpu(inp)
    q, k, v, beta, g = x["q"], x["k"], x["v"], x["beta"], x["g"]
    Hk, Hv = q.shape[2], v.shape[2]
    grp = Hv // Hk
    cu = x.get("cu_seqlens")
    S0 = x.get("initial_state")
    out = {}
    for n, h in units:
        if cu is not None:
            b, lo, hi = 0, int(cu[n]), int(cu[n + 1])
        else:
            b, lo, hi = n, 0, q.shape[1]
        sl = lambda t, hh: t[b:b + 1, lo:hi, hh:hh + 1]
        s0 = None if S0 is None else S0[n:n + 1, h:h + 1]
        o, ST = oracle.fwd(sl(q, h // grp), sl(k, h // grp), sl(v, h), sl(beta, h), sl(g, h),
                           initial_state=s0)
        out[(n, h)] = (o[0, :, 0], ST[0, 0])
    return out


def gpu_unit(inp, o, ST, n, h):
    """The GPU output and final state of one (sequence, value head) unit."""
    cu = inp.get("cu_seqlens")
    if cu is not None:
        lo, hi = int(cu[n]), int(cu[n + 1])
        return o[0, lo:hi, h], ST[n, h]
    return o[n, :, h], ST[n, h]


def units(inp, heads=None):
    """Every (sequence, head) unit: (n, h, batch row, token slice); heads defaults to the
    value heads."""
    cu = inp.get("cu_seqlens")
    heads = inp["v"].shape[2] if heads is None else heads
    if cu is not None:
        cu = [int(x) for x in cu.cpu()]
        seqs = [(n, 0, slice(cu[n], cu[n + 1])) for n in range(len(cu) - 1)]
    else:
        seqs = [(n, n, slice(0, inp["q"].shape[1])) for n in range(inp["q"].shape[0])]
    return [(n, h, b, sl) for n, b, sl in seqs for h in range(heads)]


def per_unit_rel_l2(x, ref, inp, kind):
    """rel-L2 of every (sequence, head) unit of a [B,T,H,...] token tensor (kind="tok"; H is
    whichever head count the tensor has, q/k or value heads), a [B,T,H] per-token vector
    (kind="vec") or a [N,Hv,dk,dv] state (kind="state").  Units whose reference is all zero
    compare the absolute norm."""
    x = np.asarray(x.detach().cpu().double().numpy() if hasattr(x, "detach") else x, dtype=np.float64)
    ref = np.asarray(ref.detach().cpu().double().numpy() if hasattr(ref, "detach") else ref,
                     dtype=np.float64)
    out = {}
    for n, h, b, sl in units(inp, heads=x.shape[1] if kind == "state" else x.shape[2]):
        if kind == "state":
            a, r = x[n, h], ref[n, h]
        else:
            a, r = x[b, sl, h], ref[b, sl, h]
        den = np.linalg.norm(r.ravel())
        num = np.linalg.norm((a - r).ravel())
        out[(n, h)] = float(num / den) if den > 0 else float(num)
    return out


def assert_every_unit(x, ref, inp, kind, tol, name):
    """Whole-tensor rel-L2 and every unit's rel-L2 below ``tol``; the message names the worst units."""
    whole = rel_l2(x, ref)
    per = per_unit_rel_l2(x, ref, inp, kind)
    worst = sorted(per.items(), key=lambda kv: -kv[1])[:3]
    assert whole < tol, f"{name}: whole-tensor rel-L2 {whole:.3e}"
    assert worst[0][1] < tol, f"{name}: worst units {worst} (of {len(per)}), whole {whole:.3e}"
    return whole, worst[0][1]
