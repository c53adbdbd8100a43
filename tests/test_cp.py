"""Context parallelism across GPUs for one long sequence (``cp_chunk_fwd``; dothoosh.com FlashQLA
article, first innovation: gate-driven context parallelism).

CPU: the rank protocol with the float64 oracle as its compute steps, the ranks as threads and as
gloo processes: the shards' outputs and the final state must equal the oracle's run of the
whole sequence (the exact way to float64 rounding; the halo within its 2^-30 bound).
GPU (B200): the two kernels of the protocol against float64 arithmetic, and the whole protocol
with the library's kernels, ranks as host threads sharing cuda:0, against the oracle."""
import math
import multiprocessing as mp
import socket

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_chunked_fwd_b200 import GDN_FLAG_GATE_LOGITS, GDN_FLAG_QK_L2NORM
from gated_deltanet_chunked_fwd_b200.cp import LOG_EPS, cp_chunk_fwd
from gated_deltanet_chunked_fwd_b200.inputs import make_inputs
from tests._cp_helpers import halo_ok_f64, oracle_ops, run_ranks, shards
from tests._helpers import TOL, rel_l2


def _cp_threads(x, cuts, mode, halo_chunks, ops=None, flags=0, S0=True):
    parts = shards(x, cuts)

    def rank_fn(r, comm):
        sh = parts[r]
        s0 = x["initial_state"] if (S0 and r == 0) else None
        return cp_chunk_fwd(sh["q"], sh["k"], sh["v"], sh["beta"], sh["g"], initial_state=s0, mode=mode,
                            halo_chunks=halo_chunks, flags=flags, ops=ops, comm=comm)

    res = run_ranks(len(parts), rank_fn)
    o = torch.cat([r[0].cpu() for r in res], dim=1)
    return o, [r[1].cpu() for r in res], [r[2] for r in res]


def _oracle_whole(x, S0=True, flags=0):
    return oracle.fwd(x["q"], x["k"], x["v"], x["beta"], x["g"], initial_state=x["initial_state"] if S0 else None,
                      qk_l2norm=bool(flags & GDN_FLAG_QK_L2NORM), gate_logits=bool(flags & GDN_FLAG_GATE_LOGITS))


@pytest.mark.parametrize("cuts", [(250, 420), (64, 128, 600)])
def test_exact_way_equals_the_whole_sequence(cuts):
    # weak decay (the halo never suffices): auto takes the exact fold on every rank
    x = make_inputs(1, 700, 2, 4, 16, 16, dtype="fp32", seed=3, s0_std=0.5, g_mu=-7.0)
    o, STs, taken = _cp_threads(x, cuts, "auto", 2, ops=oracle_ops())
    o_ref, ST_ref = _oracle_whole(x)
    assert set(taken) == {"exact"}
    assert rel_l2(o, o_ref) < 1e-10
    for ST in STs:  # every rank holds the sequence's final state
        assert rel_l2(ST, ST_ref) < 1e-10


def test_exact_way_without_initial_state():
    x = make_inputs(1, 700, 2, 4, 16, 16, dtype="fp32", seed=4, s0_std=0.5)
    o, STs, taken = _cp_threads(x, (300, 500), "exact", 2, ops=oracle_ops(), S0=False)
    o_ref, ST_ref = _oracle_whole(x, S0=False)
    assert set(taken) == {"exact"}
    assert rel_l2(o, o_ref) < 1e-10 and rel_l2(STs[0], ST_ref) < 1e-10


def test_halo_way_within_its_bound():
    # strong decay (g = -softplus(N(0, 1)), ~ -0.8 per token): a 2-chunk halo sums to ~ -100
    x = make_inputs(1, 700, 2, 4, 16, 16, dtype="fp32", seed=5, s0_std=0.5)
    o, STs, taken = _cp_threads(x, (200, 450), "halo", 2, ops=oracle_ops())
    o_ref, ST_ref = _oracle_whole(x)
    assert set(taken) == {"halo"}
    assert rel_l2(o, o_ref) < 1e-8 and rel_l2(STs[-1], ST_ref) < 1e-8


def test_halo_way_refused_when_a_halo_fails_and_auto_falls_back():
    x = make_inputs(1, 700, 2, 4, 16, 16, dtype="fp32", seed=6, s0_std=0.5)
    # one token of the second shard's halo breaks 0 <= beta |k|^2 <= 2
    x["k"][0, 190] *= 3.0
    with pytest.raises(RuntimeError, match="halo"):
        _cp_threads(x, (200, 450), "halo", 2, ops=oracle_ops())
    o, STs, taken = _cp_threads(x, (200, 450), "auto", 2, ops=oracle_ops())
    o_ref, ST_ref = _oracle_whole(x)
    assert set(taken) == {"exact"} and rel_l2(o, o_ref) < 1e-10


def test_short_shard_takes_the_exact_way():
    x = make_inputs(1, 700, 2, 4, 16, 16, dtype="fp32", seed=7, s0_std=0.5)
    o, STs, taken = _cp_threads(x, (100, 400), "auto", 2, ops=oracle_ops())  # first shard < halo (128)
    assert set(taken) == {"exact"}
    assert rel_l2(o, _oracle_whole(x)[0]) < 1e-10


def test_halo_check_reading():
    # the check in float64 against hand-made halos: decay sum at the bound, beta |k|^2 at 2
    T, Hk, Hv, dk = 4, 1, 2, 2
    k = np.zeros((T, Hk, dk))
    k[:, 0, 0] = 1.0
    beta = np.ones((T, Hv))
    g = np.full((T, Hv), LOG_EPS / T)
    g[:, 1] *= 0.5  # head 1 decays too little
    assert halo_ok_f64(k, beta, g, LOG_EPS).tolist() == [True, False]
    beta[2, 0] = 2.0 + 1e-9  # beta |k|^2 just above 2
    assert halo_ok_f64(k, beta, g, LOG_EPS).tolist() == [False, False]
    assert halo_ok_f64(k[:0], beta[:0], g[:0], LOG_EPS).tolist() == [False, False]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("mode,g_mu,want", [("exact", 0.0, "exact"), ("auto", 0.0, "halo"), ("auto", -7.0, "exact")])
def test_gloo_processes(mode, g_mu, want):
    from tests._cp_worker import worker

    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port, cuts, world = _free_port(), (230, 480), 3
    procs = [ctx.Process(target=worker, args=(r, world, port, queue, mode, g_mu, cuts, 11)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((queue.get(timeout=180) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(r[4] is None for r in res), [r[4] for r in res]
    assert {r[3] for r in res} == {want}
    x = make_inputs(1, 700, 2, 4, 16, 16, dtype="fp32", seed=11, s0_std=0.5, g_mu=g_mu)
    o_ref, ST_ref = _oracle_whole(x)
    o = np.concatenate([r[1] for r in res], axis=1)
    bound = 1e-10 if want == "exact" else 1e-8
    assert rel_l2(o, o_ref) < bound
    for r in res:
        assert rel_l2(r[2], ST_ref) < bound


# ---------------------------------------------------------------- GPU: the library's kernels

@pytest.mark.gpu
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (37, 100)])
def test_affine_combine_kernel(dk, dv):
    from gated_deltanet_chunked_fwd_b200 import gdn_affine_combine

    gen = torch.Generator().manual_seed(dk + dv)
    N, Hv = 2, 3
    M = torch.randn(N, Hv, dk, dk, generator=gen) / math.sqrt(dk)
    X = torch.randn(N, Hv, dk, dv, generator=gen)
    B = torch.randn(N, Hv, dk, dv, generator=gen)
    ref = np.einsum("nhij,nhjk->nhik", M.double().numpy(), X.double().numpy()) + B.double().numpy()
    Xd = X.cuda()
    gdn_affine_combine(M.cuda(), Xd, B.cuda())
    assert rel_l2(Xd, ref) < 1e-6
    Xd = X.cuda()
    gdn_affine_combine(M.cuda(), Xd)  # B = 0
    assert rel_l2(Xd, np.einsum("nhij,nhjk->nhik", M.double().numpy(), X.double().numpy())) < 1e-6


@pytest.mark.gpu
def test_affine_combine_rejects_aliasing():
    from gated_deltanet_chunked_fwd_b200 import GdnError, gdn_affine_combine

    M = torch.zeros(1, 1, 128, 128, device="cuda")
    with pytest.raises(GdnError):
        gdn_affine_combine(M, M[..., :128])


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,flags", [("bf16", 0), ("fp32", 0), ("bf16", GDN_FLAG_GATE_LOGITS | GDN_FLAG_QK_L2NORM)])
def test_halo_check_kernel(dtype, flags):
    from gated_deltanet_chunked_fwd_b200 import gdn_halo_check

    x = make_inputs(1, 256, 2, 8, 128, 128, dtype=dtype, seed=21, g_mu=0.0)
    k, beta, g = x["k"][0].clone(), x["beta"][0].clone(), x["g"][0].clone()
    g[:, 1] = -0.01  # head 1: too little decay
    k[100, 1] *= 2.0  # q/k head 1 (value heads 4-7): beta |k|^2 may exceed 2 at token 100
    beta[100, 5] = 0.9
    if flags & GDN_FLAG_GATE_LOGITS:  # the same gates as raw logits / pre-activations
        beta = torch.log(beta / (1 - beta))
        g = torch.log(torch.expm1(-g))
    ref = halo_ok_f64(k, beta, g, LOG_EPS, flags)
    ok, ld = gdn_halo_check(k.cuda(), beta.cuda(), g.cuda(), LOG_EPS, flags=flags, log_decay=True)
    assert ok.cpu().numpy().astype(bool).tolist() == ref.tolist()
    assert not ref[1] and ref[0]
    if flags & GDN_FLAG_QK_L2NORM:
        assert ref[5]  # normalised k: beta |k|^2 = beta
    else:
        assert not ref[5]
    g_mapped = -np.logaddexp(0.0, g.double().numpy()) if flags & GDN_FLAG_GATE_LOGITS else g.double().numpy()
    assert np.allclose(ld.cpu().numpy(), g_mapped.sum(0), rtol=1e-5)


@pytest.mark.gpu
@pytest.mark.parametrize("mode,g_mu,want", [("exact", 0.0, "exact"), ("auto", 0.0, "halo"), ("auto", -7.0, "exact")])
def test_cp_on_one_gpu_ranks_as_threads(mode, g_mu, want):
    # bf16, d = 128 (the tensor-core path): 4,096 tokens of one sequence in four uneven shards
    x = make_inputs(1, 4096, 2, 4, 128, 128, dtype="bf16", seed=31, s0_std=0.1, g_mu=g_mu)
    xd = {n: t.cuda() for n, t in x.items() if isinstance(t, torch.Tensor)}
    torch.cuda.synchronize()
    o, STs, taken = _cp_threads(xd, (700, 1900, 3000), mode, 4)
    assert set(taken) == {want}
    o_ref, ST_ref = _oracle_whole(x)
    tol = TOL[torch.bfloat16]
    assert rel_l2(o, o_ref) < tol and rel_l2(STs[-1], ST_ref) < tol, (rel_l2(o, o_ref), rel_l2(STs[-1], ST_ref))
    # against one forward call of the whole sequence on the same kernels
    from gated_deltanet_chunked_fwd_b200 import gdn_chunk_fwd

    o1, ST1 = gdn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["beta"], xd["g"], initial_state=xd["initial_state"])
    assert rel_l2(o, o1) < 5e-3 and rel_l2(STs[0], ST1) < 5e-3
