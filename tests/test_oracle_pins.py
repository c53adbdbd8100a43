"""Pins for the float64 oracle: facts fixed by the gated delta rule itself, not by
re-running the oracle's own formula.

Each test is chosen so that a plausible slip in the oracle (gate applied after
the erase instead of before, output read before the update, a transposed
state, a dropped beta, a wrong sign in the delta write, a wrong group mapping,
a missing term in the adjoint) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, rs, scale=1.0):
    return scale * rs.standard_normal(shape)


def unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def small_case(rs, B=1, T=7, Hk=1, Hv=1, dk=3, dv=4, s0=True):
    q = unit(rnd((B, T, Hk, dk), rs))
    k = unit(rnd((B, T, Hk, dk), rs))
    v = rnd((B, T, Hv, dv), rs)
    beta = 1 / (1 + np.exp(-rnd((B, T, Hv), rs)))
    g = -np.log1p(np.exp(rnd((B, T, Hv), rs)))
    S0 = rnd((B, Hv, dk, dv), rs, 0.5) if s0 else None
    return q, k, v, beta, g, S0


# ----------------------------------------------------------- worked example
def test_hand_worked_example():
    """Three tokens worked by hand in exact binary fractions (tests/golden)."""
    with open(os.path.join(GOLDEN, "tiny_T3_dk2_dv2.json")) as f:
        gold = json.load(f)
    sh = lambda x, *s: np.asarray(x, dtype=np.float64).reshape(*s)
    q = sh(gold["q"], 1, 3, 1, 2)
    k = sh(gold["k"], 1, 3, 1, 2)
    v = sh(gold["v"], 1, 3, 1, 2)
    beta = sh(gold["beta"], 1, 3, 1)
    g = sh(gold["g"], 1, 3, 1)
    H0 = sh(gold["H0"], 1, 1, 2, 2)
    o, ST = oracle.fwd(q, k, v, beta, g, initial_state=H0)
    np.testing.assert_allclose(o.reshape(3, 2), np.asarray(gold["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(ST.reshape(2, 2), np.asarray(gold["HT"]), rtol=0, atol=1e-12)


# --------------------------------------------------------------- invariants
def test_zero_gate_zero_beta_keeps_state():
    """g = 0 and beta = 0 give S_t = S_{t-1}: S_T = S_0 and o_t = S_0 q_t."""
    rs = np.random.default_rng(1)
    q, k, v, beta, g, S0 = small_case(rs, T=9, dk=5, dv=3)
    o, ST = oracle.fwd(q, k, v, 0 * beta, 0 * g, initial_state=S0)
    np.testing.assert_allclose(ST, S0, rtol=0, atol=1e-14)
    expect = np.einsum("bti,bij->btj", q[:, :, 0], S0[:, 0])
    np.testing.assert_allclose(o[:, :, 0], expect, rtol=0, atol=1e-13)


def test_minus_infinity_gate_resets_state():
    """exp(g_t) = 0 at step t gives S_t = beta_t v_t k_t^T regardless of the past."""
    rs = np.random.default_rng(2)
    q, k, v, beta, g, S0 = small_case(rs, T=6, dk=4, dv=5)
    t = 3
    g[0, t, 0] = -np.inf
    qs, ks, vs, bs, gs = (x[:, : t + 1] for x in (q, k, v, beta, g))
    o, ST = oracle.fwd(qs, ks, vs, bs, gs, initial_state=S0)
    expect_H = beta[0, t, 0] * np.outer(k[0, t, 0], v[0, t, 0])  # H = S^T = beta k v^T
    np.testing.assert_allclose(ST[0, 0], expect_H, rtol=0, atol=1e-14)
    np.testing.assert_allclose(o[0, t, 0], expect_H.T @ q[0, t, 0], rtol=0, atol=1e-14)


def test_unit_key_beta_one_recalls_value():
    """With |k_t| = 1 and beta_t = 1 the write is exact: S_t k_t = v_t."""
    rs = np.random.default_rng(3)
    q, k, v, beta, g, S0 = small_case(rs, T=8, dk=6, dv=4)
    beta[:] = 1.0
    for t in range(8):
        _, ST = oracle.fwd(*(x[:, : t + 1] for x in (q, k, v, beta, g)), initial_state=S0)
        np.testing.assert_allclose(ST[0, 0].T @ k[0, t, 0], v[0, t, 0], rtol=0, atol=1e-13)


def test_split_call_equals_single_call():
    """Chunked prefill: two calls chained through S_T -> S_0 equal one call."""
    rs = np.random.default_rng(4)
    q, k, v, beta, g, S0 = small_case(rs, B=2, T=37, Hk=2, Hv=4, dk=5, dv=3)
    o, ST = oracle.fwd(q, k, v, beta, g, initial_state=S0)
    s = 16
    o1, S1 = oracle.fwd(*(x[:, :s] for x in (q, k, v, beta, g)), initial_state=S0)
    o2, S2 = oracle.fwd(*(x[:, s:] for x in (q, k, v, beta, g)), initial_state=S1)
    np.testing.assert_allclose(np.concatenate([o1, o2], 1), o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(S2, ST, rtol=0, atol=1e-13)


def test_varlen_packing_equals_separate_sequences():
    """A packed batch (cu_seqlens) equals running each sequence alone."""
    rs = np.random.default_rng(5)
    lens = [1, 9, 4, 17]
    T = sum(lens)
    q, k, v, beta, g, _ = small_case(rs, T=T, Hk=2, Hv=4, dk=3, dv=2)
    S0 = rnd((len(lens), 4, 3, 2), rs)
    cu = np.concatenate([[0], np.cumsum(lens)])
    o, ST = oracle.fwd(q, k, v, beta, g, cu_seqlens=cu, initial_state=S0)
    for n in range(len(lens)):
        sl = slice(cu[n], cu[n + 1])
        on, Sn = oracle.fwd(*(x[:, sl] for x in (q, k, v, beta, g)), initial_state=S0[n:n + 1])
        np.testing.assert_allclose(o[:, sl], on, rtol=0, atol=1e-14)
        np.testing.assert_allclose(ST[n:n + 1], Sn, rtol=0, atol=1e-14)


def test_grouped_heads_use_contiguous_groups():
    """Value head h reads q/k head h // (Hv/Hk)."""
    rs = np.random.default_rng(6)
    q, k, v, beta, g, S0 = small_case(rs, T=11, Hk=2, Hv=6, dk=3, dv=2)
    o, ST = oracle.fwd(q, k, v, beta, g, initial_state=S0)
    for h in range(6):
        hk = h // 3
        oh, Sh = oracle.fwd(q[:, :, hk:hk + 1], k[:, :, hk:hk + 1], v[:, :, h:h + 1],
                            beta[:, :, h:h + 1], g[:, :, h:h + 1], initial_state=S0[:, h:h + 1])
        np.testing.assert_allclose(o[:, :, h:h + 1], oh, rtol=0, atol=1e-14)
        np.testing.assert_allclose(ST[:, h:h + 1], Sh, rtol=0, atol=1e-14)


# ------------------------------------------------------------- closed forms
def test_beta_zero_is_pure_decay():
    """beta = 0: S_T = exp(sum g) S_0 and o_t = exp(sum_{<=t} g) S_0 q_t."""
    rs = np.random.default_rng(7)
    q, k, v, beta, g, S0 = small_case(rs, T=13, dk=4, dv=4)
    o, ST = oracle.fwd(q, k, v, 0 * beta, g, initial_state=S0)
    cum = np.cumsum(g[0, :, 0])
    np.testing.assert_allclose(ST[0, 0], math.exp(cum[-1]) * S0[0, 0], rtol=1e-13, atol=0)
    for t in range(13):
        np.testing.assert_allclose(o[0, t, 0], math.exp(cum[t]) * S0[0, 0].T @ q[0, t, 0],
                                   rtol=1e-12, atol=1e-15)


def test_single_token_formula():
    """T = 1: S_1 = e^g S_0 (I - b k k^T) + b v k^T, o_1 = S_1 q_1, written in S (dv x dk)."""
    rs = np.random.default_rng(8)
    dk, dv = 5, 3
    q, k, v = rnd((1, 1, 1, dk), rs), rnd((1, 1, 1, dk), rs), rnd((1, 1, 1, dv), rs)
    b, gg = 0.7, -0.4
    S0_math = rnd((dv, dk), rs)  # S in the rule's own orientation
    o, ST = oracle.fwd(q, k, v, np.full((1, 1, 1), b), np.full((1, 1, 1), gg),
                       initial_state=S0_math.T[None, None])
    kk = k[0, 0, 0]
    S1 = math.exp(gg) * S0_math @ (np.eye(dk) - b * np.outer(kk, kk)) + b * np.outer(v[0, 0, 0], kk)
    np.testing.assert_allclose(ST[0, 0], S1.T, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(o[0, 0, 0], S1 @ q[0, 0, 0], rtol=1e-13, atol=1e-14)


def test_orthonormal_keys_associative_recall():
    """g = 0, beta = 1, orthonormal keys: S_T = S_0 (I - sum k k^T) + sum v k^T."""
    rs = np.random.default_rng(9)
    dk, dv, m = 8, 5, 6
    Qm, _ = np.linalg.qr(rs.standard_normal((dk, dk)))
    keys = Qm[:, :m].T
    k = keys.reshape(1, m, 1, dk)
    v = rnd((1, m, 1, dv), rs)
    q = unit(rnd((1, m, 1, dk), rs))
    S0 = rnd((1, 1, dk, dv), rs)
    _, ST = oracle.fwd(q, k, v, np.ones((1, m, 1)), np.zeros((1, m, 1)), initial_state=S0)
    P = keys.T @ keys
    S_math = S0[0, 0].T @ (np.eye(dk) - P) + v[0, :, 0].T @ keys
    np.testing.assert_allclose(ST[0, 0], S_math.T, rtol=0, atol=1e-13)
    _, ST0 = oracle.fwd(q, k, v, np.ones((1, m, 1)), np.zeros((1, m, 1)))
    for i in range(m):
        np.testing.assert_allclose(ST0[0, 0].T @ keys[i], v[0, i, 0], rtol=0, atol=1e-13)


def test_jointly_linear_in_values_and_state():
    """o and S_T are linear in (v, S_0) jointly for fixed (q, k, beta, g)."""
    rs = np.random.default_rng(10)
    q, k, v1, beta, g, S1 = small_case(rs, T=10, Hk=1, Hv=2, dk=4, dv=3)
    v2, S2 = rnd(v1.shape, rs), rnd(S1.shape, rs)
    a, b = 1.7, -0.3
    o1, T1 = oracle.fwd(q, k, v1, beta, g, initial_state=S1)
    o2, T2 = oracle.fwd(q, k, v2, beta, g, initial_state=S2)
    o3, T3 = oracle.fwd(q, k, a * v1 + b * v2, beta, g, initial_state=a * S1 + b * S2)
    np.testing.assert_allclose(o3, a * o1 + b * o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(T3, a * T1 + b * T2, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------ the backward
def torch_token_loop(q, k, v, beta, g, S0, cu, group):
    """Independent float64 restatement of the rule in S (dv x dk) orientation,
    differentiated by torch.autograd."""
    outs, finals = [], []
    Hv = v.shape[2]
    for n in range(len(cu) - 1):
        per_head_o, per_head_S = [], []
        for h in range(Hv):
            S = S0[n, h].T if S0 is not None else torch.zeros(v.shape[-1], q.shape[-1], dtype=q.dtype)
            os_ = []
            for t in range(cu[n], cu[n + 1]):
                kk, qq, vv = k[0, t, h // group], q[0, t, h // group], v[0, t, h]
                I = torch.eye(kk.numel(), dtype=q.dtype)
                S = torch.exp(g[0, t, h]) * S @ (I - beta[0, t, h] * torch.outer(kk, kk)) \
                    + beta[0, t, h] * torch.outer(vv, kk)
                os_.append(S @ qq)
            per_head_o.append(torch.stack(os_) if os_ else torch.zeros(0, v.shape[-1], dtype=q.dtype))
            per_head_S.append(S.T)
        outs.append(torch.stack(per_head_o, 1))
        finals.append(torch.stack(per_head_S))
    return torch.cat(outs, 0)[None], torch.stack(finals)


@pytest.mark.parametrize("lens,Hk,Hv,dk,dv", [([7], 1, 1, 3, 4), ([5, 1, 9], 2, 4, 4, 3), ([70], 1, 2, 3, 2)])
def test_backward_matches_torch_autograd(lens, Hk, Hv, dk, dv):
    """The oracle's hand-written adjoint equals torch.autograd of an independent
    token loop written in S orientation (includes a 70-token case that crosses
    the 64-token checkpoint window)."""
    rs = np.random.default_rng(11)
    T = sum(lens)
    q, k, v, beta, g, _ = small_case(rs, T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv)
    cu = np.concatenate([[0], np.cumsum(lens)])
    S0 = rnd((len(lens), Hv, dk, dv), rs)
    do = rnd((1, T, Hv, dv), rs)
    dST = rnd((len(lens), Hv, dk, dv), rs)
    res = oracle.bwd(q, k, v, beta, g, do, cu_seqlens=cu, initial_state=S0, dST=dST)
    tens = [torch.tensor(x, requires_grad=True) for x in (q, k, v, beta, g, S0)]
    o, ST = torch_token_loop(*tens, list(cu), Hv // Hk)
    loss = (o * torch.tensor(do)).sum() + (ST * torch.tensor(dST)).sum()
    grads = torch.autograd.grad(loss, tens)
    for name, mine, ref in zip(["dq", "dk", "dv", "dbeta", "dg", "dS0"], res, grads):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-11, err_msg=name)


def test_backward_central_differences():
    """Directional central differences of the oracle forward match <grad, dir>."""
    rs = np.random.default_rng(12)
    q, k, v, beta, g, S0 = small_case(rs, T=12, Hk=1, Hv=2, dk=4, dv=3)
    do = rnd((1, 12, 2, 3), rs)
    dST = rnd((1, 2, 4, 3), rs)
    grads = oracle.bwd(q, k, v, beta, g, do, initial_state=S0, dST=dST)

    def L(xs):
        o, ST = oracle.fwd(*xs[:5], initial_state=xs[5])
        return float((o * do).sum() + (ST * dST).sum())

    base = [q, k, v, beta, g, S0]
    h = 1e-6
    for i in range(6):
        for _ in range(2):
            d = rnd(base[i].shape, rs)
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[i] += h * d
            minus[i] -= h * d
            fd = (L(plus) - L(minus)) / (2 * h)
            an = float((grads[i] * d).sum())
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (i, fd, an)


# ---- optional input preprocessing (q / k L2-normalisation, beta and g from logits) ----

def test_preprocess_closed_forms():
    """sigmoid(0) = 1/2, -softplus(0) = -log 2, -softplus tends to -a for large a and to -e^a for
    very negative a; normalised vectors have unit norm, and a vector below the clamp is divided
    by 1e-6."""
    q = np.array([[[[3.0, 4.0]], [[1e-8, 0.0]]]])        # [B=1, T=2, H=1, d=2]
    k = np.array([[[[0.0, -2.0]], [[6.0, 8.0]]]])
    b = np.array([[[0.0], [np.log(3.0)]]])                  # sigmoid: 1/2, 3/4
    a = np.array([[[0.0], [40.0]]])
    qh, kh, bt, g = oracle.preprocess(q, k, b, a, qk_l2norm=True, gate_logits=True)
    np.testing.assert_allclose(qh[0, 0, 0], [0.6, 0.8], rtol=1e-15)
    np.testing.assert_allclose(qh[0, 1, 0], [1e-2, 0.0], rtol=1e-12)
    np.testing.assert_allclose(kh[0, :, 0], [[0.0, -1.0], [0.6, 0.8]], rtol=1e-15)
    np.testing.assert_allclose(bt[0, :, 0], [0.5, 0.75], rtol=1e-15)
    assert g[0, 0, 0] == pytest.approx(-np.log(2.0), rel=1e-15)
    assert g[0, 1, 0] == pytest.approx(-40.0 - np.exp(-40.0), rel=1e-15)
    assert oracle.preprocess(q, k, b, np.array([[[-50.0], [0.0]]]), gate_logits=True)[3][0, 0, 0] == \
        pytest.approx(-np.exp(-50.0), rel=1e-12)
    # flags off: the inputs come back unchanged
    for x, y in zip(oracle.preprocess(q, k, b, a), (q, k, b, a)):
        np.testing.assert_array_equal(x, y)


def test_preprocess_backward_central_differences():
    """The chain rule of the preprocessing maps against central differences of a random linear
    functional of their outputs (a dropped projection term, a sign or a sigmoid' slip fails)."""
    rs = np.random.default_rng(21)
    q = rnd((1, 7, 2, 5), rs)
    k = rnd((1, 7, 2, 5), rs)
    q[0, 3, 1] *= 1e-9  # one vector below the clamp
    b = rnd((1, 7, 3), rs) * 3
    a = rnd((1, 7, 3), rs) * 3
    w = [rnd(x.shape, rs) for x in (q, k, b, a)]

    def L(xs):
        ys = oracle.preprocess(*xs, qk_l2norm=True, gate_logits=True)
        return float(sum((y * wi).sum() for y, wi in zip(ys, w)))

    an = oracle.preprocess_bwd(q, k, b, a, *w, qk_l2norm=True, gate_logits=True)
    base = [q, k, b, a]
    for i in range(4):
        for _ in range(3):
            d = rnd(base[i].shape, rs)
            h = 1e-7 if i < 2 else 1e-6
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[i] += h * d
            minus[i] -= h * d
            if i == 0:  # keep the clamped vector clamped: perturb it within its size
                plus[0][0, 3, 1] = q[0, 3, 1] * (1 + 1e-3 * d[0, 3, 1, 0])
                minus[0][0, 3, 1] = q[0, 3, 1] * (1 - 1e-3 * d[0, 3, 1, 0])
                dd = d.copy()
                dd[0, 3, 1] = q[0, 3, 1] * 1e-3 * d[0, 3, 1, 0] / h
            else:
                dd = d
            fd = (L(plus) - L(minus)) / (2 * h)
            val = float((an[i] * dd).sum())
            assert abs(fd - val) <= 1e-5 * max(1.0, abs(val)), (i, fd, val)


def test_layer_with_preprocessing_central_differences():
    """bwd(..., qk_l2norm, gate_logits) is the gradient of fwd(..., qk_l2norm, gate_logits) with
    respect to the raw q, k, beta and g (directional central differences through the layer)."""
    rs = np.random.default_rng(22)
    q, k, v, beta, g, S0 = small_case(rs, T=9, Hk=1, Hv=2, dk=4, dv=3)
    q, k = q * 3, k * 0.5              # raw, not unit vectors
    beta, g = beta * 4 - 2, g * 3 + 1  # logits of either sign
    do = rnd((1, 9, 2, 3), rs)
    dST = rnd((1, 2, 4, 3), rs)
    kw = dict(qk_l2norm=True, gate_logits=True)
    grads = oracle.bwd(q, k, v, beta, g, do, initial_state=S0, dST=dST, **kw)

    def L(xs):
        o, ST = oracle.fwd(*xs[:5], initial_state=xs[5], **kw)
        return float((o * do).sum() + (ST * dST).sum())

    base = [q, k, v, beta, g, S0]
    h = 1e-6
    for i in range(6):
        d = rnd(base[i].shape, rs)
        plus = [x.copy() for x in base]
        minus = [x.copy() for x in base]
        plus[i] += h * d
        minus[i] -= h * d
        fd = (L(plus) - L(minus)) / (2 * h)
        an = float((grads[i] * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (i, fd, an)
