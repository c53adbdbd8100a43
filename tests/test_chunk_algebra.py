"""The chunked (WY / UT-transform) form of the gated delta rule, restated in
float64 torch and checked against the token-by-token oracle.

This pins the algebra the CUDA kernels implement -- forward and backward --
independently of any kernel.  Per chunk of C tokens with entry state H (dk x dv,
H = S^T), gamma = in-chunk cumsum of g, Gam = exp(gamma), E_rs = exp(gamma_r - gamma_s):

  A  = strictly-lower( diag(beta) (K K^T o E) )      T = (I + A)^-1
  W  = T diag(beta Gam) K                             Ut = T diag(beta) V
  U  = Ut - W H                                       P  = lower-incl( Q K^T o E )
  O  = diag(Gam) Q H + P U
  H' = Gam_n H + Kd^T U,   Kd = diag(exp(gamma_n - gamma)) K
The backward is the reverse-mode adjoint of those lines, chunk by chunk in reverse.
"""
import numpy as np
import pytest
import torch

import oracle


def chunk_fwd(q, k, v, beta, g, H0, C):
    """q,k [T,dk], v [T,dv], beta,g [T], H0 [dk,dv]; returns o [T,dv], H_T, per-chunk entry states."""
    T = q.shape[0]
    H = H0.clone()
    o = torch.zeros(T, v.shape[1], dtype=torch.float64)
    entries = []
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        Q, K, V, b, gg = q[sl], k[sl], v[sl], beta[sl], g[sl]
        n = Q.shape[0]
        gam = torch.cumsum(gg, 0)
        Gam = torch.exp(gam)
        E = torch.exp(gam[:, None] - gam[None, :])
        A = torch.tril(b[:, None] * (K @ K.T) * E, -1)
        Tm = torch.linalg.inv(torch.eye(n, dtype=torch.float64) + A)
        W = Tm @ ((b * Gam)[:, None] * K)
        Ut = Tm @ (b[:, None] * V)
        entries.append(H.clone())
        U = Ut - W @ H
        P = torch.tril((Q @ K.T) * E)
        o[sl] = Gam[:, None] * (Q @ H) + P @ U
        Kd = torch.exp(gam[-1] - gam)[:, None] * K
        H = Gam[-1] * H + Kd.T @ U
    return o, H, entries


def chunk_bwd(q, k, v, beta, g, H0, do, dHT, C):
    """Chunkwise adjoint; returns dq, dk, dv, dbeta, dg, dH0."""
    T, dk = q.shape
    _, _, entries = chunk_fwd(q, k, v, beta, g, H0, C)
    dq = torch.zeros_like(q)
    dkk = torch.zeros_like(k)
    dvv = torch.zeros_like(v)
    db = torch.zeros_like(beta)
    dgg = torch.zeros_like(g)
    dH = dHT.clone()  # adjoint of the chunk's exit state
    starts = list(range(0, T, C))
    for ci in reversed(range(len(starts))):
        c0 = starts[ci]
        sl = slice(c0, min(T, c0 + C))
        Q, K, V, b, gg, dO = q[sl], k[sl], v[sl], beta[sl], g[sl], do[sl]
        H = entries[ci]
        n = Q.shape[0]
        gam = torch.cumsum(gg, 0)
        Gam = torch.exp(gam)
        E = torch.exp(gam[:, None] - gam[None, :])
        KK = K @ K.T
        A = torch.tril(b[:, None] * KK * E, -1)
        Tm = torch.linalg.inv(torch.eye(n, dtype=torch.float64) + A)
        Kb = (b * Gam)[:, None] * K
        Vb = b[:, None] * V
        W = Tm @ Kb
        U = Tm @ Vb - W @ H
        P = torch.tril((Q @ K.T) * E)
        dec = torch.exp(gam[-1] - gam)
        Kd = dec[:, None] * K
        # H' = Gam_n H + Kd^T U
        dU = P.T @ dO + Kd @ dH
        dKd = U @ dH.T
        dgam = torch.zeros(n, dtype=torch.float64)
        dgam[-1] += Gam[-1] * (dH * H).sum() + (Kd * dKd).sum()
        dgam -= (Kd * dKd).sum(1)
        dK = dec[:, None] * dKd
        # O = diag(Gam) Q H + P U
        dQs = Gam[:, None] * (dO @ H.T)
        dgam += (Q * dQs).sum(1)
        dP = torch.tril(dO @ U.T)
        dgam += (dP * P).sum(1) - (dP * P).sum(0)
        dQ = dQs + (dP * E) @ K
        dK += (dP * E).T @ Q
        # U = T Vb - W H
        dW = -dU @ H.T
        dT = dW @ Kb.T + dU @ Vb.T
        TdU = Tm.T @ dU
        TdW = Tm.T @ dW
        dvv[sl] = b[:, None] * TdU
        db_ = (TdU * V).sum(1) + Gam * (TdW * K).sum(1)
        dK += (b * Gam)[:, None] * TdW
        dgam += (TdW * Kb).sum(1)
        # T = (I + A)^-1
        dA = torch.tril(-Tm.T @ dT @ Tm.T, -1)
        db_ += (dA * KK * E).sum(1)
        G = dA * E * b[:, None]
        dK += (G + G.T) @ K
        dgam += (dA * A).sum(1) - (dA * A).sum(0)
        dH_prev = Gam[-1] * dH + (Gam[:, None] * Q).T @ dO - W.T @ dU
        dq[sl] = dQ
        dkk[sl] = dK
        db[sl] = db_
        dgg[sl] = torch.flip(torch.cumsum(torch.flip(dgam, [0]), 0), [0])
        dH = dH_prev
    return dq, dkk, dvv, db, dgg, dH


def case(T, dk, dv, seed, g_scale=1.0):
    rs = np.random.default_rng(seed)
    t = lambda *s: torch.tensor(rs.standard_normal(s))
    q = torch.nn.functional.normalize(t(T, dk), dim=-1)
    k = torch.nn.functional.normalize(t(T, dk), dim=-1)
    v = t(T, dv)
    beta = torch.sigmoid(t(T))
    g = -torch.nn.functional.softplus(g_scale * t(T))
    H0 = 0.3 * t(dk, dv)
    return q, k, v, beta, g, H0


def as_oracle(x):
    return x.numpy()[None, :, None]


@pytest.mark.parametrize("T,C,dk,dv", [(37, 8, 5, 3), (200, 64, 16, 8), (64, 64, 8, 8), (1, 64, 4, 4), (129, 64, 6, 5)])
def test_chunk_forward_equals_token_loop(T, C, dk, dv):
    q, k, v, beta, g, H0 = case(T, dk, dv, seed=T)
    o, HT, _ = chunk_fwd(q, k, v, beta, g, H0, C)
    o_ref, ST = oracle.fwd(as_oracle(q), as_oracle(k), as_oracle(v), beta.numpy()[None, :, None],
                           g.numpy()[None, :, None], initial_state=H0.numpy()[None, None])
    np.testing.assert_allclose(o.numpy(), o_ref[0, :, 0], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(HT.numpy(), ST[0, 0], rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("T,C,dk,dv", [(37, 8, 5, 3), (150, 64, 8, 6), (1, 64, 3, 2)])
def test_chunk_backward_equals_token_adjoint(T, C, dk, dv):
    q, k, v, beta, g, H0 = case(T, dk, dv, seed=100 + T)
    rs = np.random.default_rng(7)
    do = torch.tensor(rs.standard_normal((T, dv)))
    dHT = torch.tensor(rs.standard_normal((dk, dv)))
    mine = chunk_bwd(q, k, v, beta, g, H0, do, dHT, C)
    ref = oracle.bwd(as_oracle(q), as_oracle(k), as_oracle(v), beta.numpy()[None, :, None],
                     g.numpy()[None, :, None], do.numpy()[None, :, None],
                     initial_state=H0.numpy()[None, None], dST=dHT.numpy()[None, None])
    ref = [r[0, :, 0] for r in ref[:5]] + [ref[5][0, 0]]
    for name, a, b in zip(["dq", "dk", "dv", "dbeta", "dg", "dS0"], mine, ref):
        np.testing.assert_allclose(a.numpy(), b, rtol=1e-9, atol=1e-10, err_msg=name)


def test_state_transition_contracts_by_the_gate():
    """The fact the multi-SM split relies on: with 0 <= beta |k|^2 <= 2 the linear
    part of a chunk's state map, H -> Gam_n H - Kd^T W H, has spectral norm
    <= exp(sum of the chunk's g)."""
    for seed in range(5):
        q, k, v, beta, g, H0 = case(64, 16, 8, seed=seed, g_scale=0.2)
        gam = torch.cumsum(g, 0)
        E = torch.exp(gam[:, None] - gam[None, :])
        A = torch.tril(beta[:, None] * (k @ k.T) * E, -1)
        Tm = torch.linalg.inv(torch.eye(64, dtype=torch.float64) + A)
        W = Tm @ ((beta * torch.exp(gam))[:, None] * k)
        Kd = torch.exp(gam[-1] - gam)[:, None] * k
        M = torch.exp(gam[-1]) * torch.eye(16, dtype=torch.float64) - Kd.T @ W
        assert torch.linalg.matrix_norm(M, 2) <= torch.exp(gam[-1]) * (1 + 1e-12)
