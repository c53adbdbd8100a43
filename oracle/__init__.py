"""Float64 CPU oracle for the GDN layer (gated delta rule), token by token.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA path (``gated_deltanet_chunked_fwd_b200``) and imports nothing
from it.

The arithmetic lives in ``gdn_oracle.c`` (plain C, float64, OpenMP over
independent (sequence, head) units); this module only marshals arrays.  The
layer is the one the FlashQLA pages accelerate (news.hamidun.com FlashQLA page,
"What is FlashQLA": GDN forward and backward in chunked-prefill mode); the rule
itself is the standard gated delta rule

    S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t

with states stored transposed, H = S^T of shape [dk, dv].

Pins (``tests/test_oracle_pins.py``): invariants of the rule, closed forms,
a hand-worked example (``tests/golden/``), torch autograd and finite
differences for the backward; closed forms and central differences for the
optional input preprocessing and its backward.  No function here is "parity
unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgdn_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c with gcc (-O2 -fopenmp) into oracle/libgdn_oracle.so."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        d = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        ci = ctypes.c_int
        lib.gdn_oracle_fwd.argtypes = [ctypes.c_int64, i64p, ci, ci, ci, ci] + [d] * 8
        lib.gdn_oracle_fwd.restype = ci
        lib.gdn_oracle_bwd.argtypes = [ctypes.c_int64, i64p, ci, ci, ci, ci] + [d] * 14
        lib.gdn_oracle_bwd.restype = ci
        lib.gdn_oracle_num_threads.restype = ci
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else all cores)."""
    return int(_load().gdn_oracle_num_threads())


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _pack(q, k, v, beta, g, cu_seqlens):
    """Accept [B,T,H,d] (+ optional cu_seqlens with B == 1) and return packed
    [T_total,H,d] arrays with int64 offsets."""
    q, k, v, beta, g = (_f64(x) for x in (q, k, v, beta, g))
    if q.ndim != 4:
        raise ValueError("q must be [B, T, Hk, dk]")
    B, T = q.shape[:2]
    if cu_seqlens is None:
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        if B != 1:
            raise ValueError("cu_seqlens needs B == 1")
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
    flat = lambda x: np.ascontiguousarray(x.reshape((B * T,) + x.shape[2:]))
    return (B, T, cu) + tuple(flat(x) for x in (q, k, v, beta, g))


# ---- optional input preprocessing ------------------------------------------------------
# Models usually feed the layer from raw projections: q and k are L2-normalised over the head
# dimension, beta is a sigmoid of a logit and the log decay g is minus a softplus.  The pages
# do not describe this step (it is a reading: the plainest form of each map, as the input
# generator applies it); with qk_l2norm / gate_logits the layer takes the raw values and
# applies the maps itself, and the backward returns gradients with respect to the raw values.

L2_EPS = 1e-6  # x / max(||x||, L2_EPS)


def _l2norm(x):
    n = np.sqrt((x * x).sum(-1, keepdims=True))
    return x / np.maximum(n, L2_EPS), n


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _neg_softplus(x):
    """-log(1 + exp(x)), in the form that neither overflows nor loses small values."""
    return -(np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x))))


def preprocess(q, k, beta, g, qk_l2norm=False, gate_logits=False):
    """(q, k, beta, g) as the rule consumes them, from raw inputs (float64):
    q, k -> x / max(||x||_2, 1e-6) over the head dimension when qk_l2norm;
    beta -> sigmoid(beta) and g -> -softplus(g) = -log(1 + exp(g)) when gate_logits."""
    q, k, beta, g = (_f64(x) for x in (q, k, beta, g))
    if qk_l2norm:
        q, k = _l2norm(q)[0], _l2norm(k)[0]
    if gate_logits:
        beta, g = _sigmoid(beta), _neg_softplus(g)
    return q, k, beta, g


def preprocess_bwd(q, k, beta, g, dq, dk, dbeta, dg, qk_l2norm=False, gate_logits=False):
    """Gradients with respect to the raw (q, k, beta, g) from those with respect to the
    preprocessed values (chain rule of the maps above):
      y = x / ||x||:             dx = (dy - y (y . dy)) / ||x||    (dx = dy / 1e-6 below the clamp)
      beta = sigmoid(b):         db = dbeta beta (1 - beta)
      g = -softplus(a):          da = -dg sigmoid(a)"""
    q, k, beta, g, dq, dk, dbeta, dg = (_f64(x) for x in (q, k, beta, g, dq, dk, dbeta, dg))
    if qk_l2norm:
        out = []
        for x, dy in ((q, dq), (k, dk)):
            y, n = _l2norm(x)
            c = np.maximum(n, L2_EPS)
            proj = dy - y * (y * dy).sum(-1, keepdims=True)
            out.append(np.where(n > L2_EPS, proj, dy) / c)
        dq, dk = out
    if gate_logits:
        s = _sigmoid(beta)
        dbeta = dbeta * s * (1.0 - s)
        dg = -dg * _sigmoid(g)
    return dq, dk, dbeta, dg


def fwd(q, k, v, beta, g, cu_seqlens=None, initial_state=None, output_final_state=True,
        qk_l2norm=False, gate_logits=False):
    """o, S_T = rule applied token by token (float64).

    q, k: [B, T, Hk, dk]; v: [B, T, Hv, dv]; beta, g: [B, T, Hv];
    cu_seqlens: optional [N+1] offsets (B must be 1); initial_state: [N, Hv, dk, dv]
    (the transposed state H = S^T).  Returns numpy float64 (o [B,T,Hv,dv], S_T or None).
    qk_l2norm / gate_logits: the inputs are raw and go through `preprocess` first.
    """
    if qk_l2norm or gate_logits:
        q, k, beta, g = preprocess(q, k, beta, g, qk_l2norm, gate_logits)
    B, T, cu, qf, kf, vf, bf, gf = _pack(q, k, v, beta, g, cu_seqlens)
    N = cu.shape[0] - 1
    Hk, dk = qf.shape[1], qf.shape[2]
    Hv, dv = vf.shape[1], vf.shape[2]
    S0 = _f64(initial_state)
    if S0 is not None and S0.shape != (N, Hv, dk, dv):
        raise ValueError(f"initial_state must be {(N, Hv, dk, dv)}")
    o = np.zeros((B * T, Hv, dv))
    ST = np.zeros((N, Hv, dk, dv)) if output_final_state else None
    rc = _load().gdn_oracle_fwd(
        N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), Hk, Hv, dk, dv,
        _ptr(qf), _ptr(kf), _ptr(vf), _ptr(bf), _ptr(gf), _ptr(S0), _ptr(o), _ptr(ST))
    if rc != 0:
        raise RuntimeError(f"gdn_oracle_fwd failed with code {rc}")
    return o.reshape(B, T, Hv, dv), ST


def bwd(q, k, v, beta, g, do, cu_seqlens=None, initial_state=None, dST=None, qk_l2norm=False,
        gate_logits=False):
    """Gradients of <do, o> + <dST, S_T> w.r.t. (q, k, v, beta, g, S0), float64.

    Returns numpy arrays (dq, dk, dv, dbeta, dg, dS0) with the input shapes;
    dq/dk are summed over the value heads that share a q/k head.  With qk_l2norm /
    gate_logits the inputs are raw and the gradients are with respect to them.
    """
    if qk_l2norm or gate_logits:
        raw = (q, k, beta, g)
        q, k, beta, g = preprocess(q, k, beta, g, qk_l2norm, gate_logits)
        res = bwd(q, k, v, beta, g, do, cu_seqlens, initial_state, dST)
        dq, dk_, db, dg_ = preprocess_bwd(*raw, res[0], res[1], res[3], res[4], qk_l2norm, gate_logits)
        return dq, dk_, res[2], db, dg_, res[5]
    B, T, cu, qf, kf, vf, bf, gf = _pack(q, k, v, beta, g, cu_seqlens)
    N = cu.shape[0] - 1
    Hk, dk = qf.shape[1], qf.shape[2]
    Hv, dv = vf.shape[1], vf.shape[2]
    S0 = _f64(initial_state)
    dof = np.ascontiguousarray(_f64(do).reshape(B * T, Hv, dv))
    dSTf = _f64(dST)
    dq = np.zeros_like(qf)
    dk_ = np.zeros_like(kf)
    dv_ = np.zeros_like(vf)
    db = np.zeros_like(bf)
    dg = np.zeros_like(gf)
    dS0 = np.zeros((N, Hv, dk, dv))
    rc = _load().gdn_oracle_bwd(
        N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), Hk, Hv, dk, dv,
        _ptr(qf), _ptr(kf), _ptr(vf), _ptr(bf), _ptr(gf), _ptr(S0), _ptr(dof), _ptr(dSTf),
        _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(db), _ptr(dg), _ptr(dS0))
    if rc != 0:
        raise RuntimeError(f"gdn_oracle_bwd failed with code {rc}")
    shp = lambda x, like: x.reshape((B, T) + like.shape[1:])
    return (shp(dq, qf), shp(dk_, kf), shp(dv_, vf), shp(db, bf), shp(dg, gf), dS0)
