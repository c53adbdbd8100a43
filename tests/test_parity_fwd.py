"""GPU forward parity: libgdn (through the C ABI) against the float64 oracle on
the same seeded inputs, element by element over whole tensors (rel-L2 bars in
_helpers.TOL), at sizes that span several chunks and a ragged tail, and at the
full workload sizes over whole tensors and every (sequence, value head) unit on
its own."""
import math

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_chunked_fwd_b200 import (GDN_FLAG_GATE_LOGITS, GDN_FLAG_PORTABLE, GDN_FLAG_QK_L2NORM,
                                             GDN_FLAG_SPLIT_FORCE,
                                             GDN_FLAG_SPLIT_OFF, gdn_chunk_fwd)
from gated_deltanet_chunked_fwd_b200.inputs import make_inputs, make_workload
from tests._helpers import TOL, assert_every_unit, cpu, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run(inp, flags=0):
    o, ST = gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"],
                          cu_seqlens=inp.get("cu_seqlens"), initial_state=inp.get("initial_state"),
                          cu_seqlens_host=inp.get("cu_seqlens_host"), flags=flags,
                          check_device_status=True)
    torch.cuda.synchronize()
    return o, ST


def full_oracle(inp):
    x = cpu(inp)
    return oracle.fwd(x["q"], x["k"], x["v"], x["beta"], x["g"], cu_seqlens=x.get("cu_seqlens"),
                      initial_state=x.get("initial_state"))


def check_full(inp, flags=0):
    o, ST = run(inp, flags)
    o_ref, ST_ref = full_oracle(inp)
    tol = TOL[inp["q"].dtype]
    assert rel_l2(o, o_ref) < tol, rel_l2(o, o_ref)
    assert rel_l2(ST, ST_ref) < tol, rel_l2(ST, ST_ref)
    return o, ST


def test_workload0_fp32_full():
    check_full(make_workload(0, device=DEV))


CASES = [
    # dtype, B, T, Hk, Hv, dk, dv, s0
    ("fp32", 1, 1, 1, 1, 16, 16, None),
    ("fp32", 2, 65, 1, 2, 64, 64, 0.3),
    ("fp32", 1, 130, 2, 2, 128, 128, 0.3),
    ("fp32", 1, 63, 1, 1, 48, 80, 0.3),
    ("bf16", 1, 64, 2, 2, 128, 128, 0.1),
    ("bf16", 2, 200, 2, 4, 128, 128, 0.1),
    ("bf16", 1, 1, 1, 1, 128, 128, None),
    ("bf16", 1, 65, 1, 1, 64, 64, 0.1),
    ("bf16", 1, 1000, 1, 3, 128, 128, 0.1),
]


@pytest.mark.parametrize("flags", [0, GDN_FLAG_PORTABLE])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_small_shapes(case, flags):
    dt, B, T, Hk, Hv, dk, dv, s0 = case
    check_full(make_inputs(B, T, Hk, Hv, dk, dv, dtype=dt, seed=1, s0_std=s0, device=DEV), flags)


@pytest.mark.parametrize("dt,dk", [("fp32", 64), ("bf16", 128)])
@pytest.mark.parametrize("flags", [0, GDN_FLAG_PORTABLE, GDN_FLAG_SPLIT_FORCE, GDN_FLAG_SPLIT_OFF])
def test_varlen_ragged(dt, dk, flags):
    lengths = [1, 64, 65, 0, 130, 7, 300]
    check_full(make_inputs(1, 0, 2, 4, dk, dk, dtype=dt, seed=2, s0_std=0.2, lengths=lengths,
                           device=DEV), flags)


def test_split_modes_agree_on_long_sequence():
    inp = make_inputs(1, 3000, 1, 2, 128, 128, dtype="bf16", seed=3, s0_std=0.1, device=DEV)
    outs = [run(inp, f) for f in (0, GDN_FLAG_SPLIT_OFF, GDN_FLAG_SPLIT_FORCE, GDN_FLAG_PORTABLE)]
    for o, ST in outs[1:]:
        assert rel_l2(o, outs[0][0]) < 5e-3
        assert rel_l2(ST, outs[0][1]) < 5e-3
    check_full(inp)


def test_empty_input_copies_state():
    inp = make_inputs(1, 0, 1, 2, 64, 64, dtype="fp32", seed=4, s0_std=1.0, device=DEV)
    o, ST = run(inp)
    assert o.numel() == 0
    assert torch.equal(ST, inp["initial_state"])


def test_pure_decay_closed_form():
    """beta = 0: S_T = exp(sum g) S_0 and o_t = exp(cumsum g)_t S_0 q_t."""
    inp = make_inputs(1, 257, 1, 1, 128, 128, dtype="fp32", seed=5, s0_std=1.0, device=DEV)
    inp["beta"].zero_()
    inp["g"].mul_(0.01)
    o, ST = run(inp)
    cum = torch.cumsum(inp["g"][0, :, 0].double(), 0)
    S0 = inp["initial_state"][0, 0].double()
    ref_ST = torch.exp(cum[-1]) * S0
    ref_o = torch.exp(cum)[:, None] * (inp["q"][0, :, 0].double() @ S0)
    assert rel_l2(ST[0, 0], ref_ST) < 1e-5
    assert rel_l2(o[0, :, 0], ref_o) < 1e-5


def test_strong_gate_resets_state():
    """g = -30 (exp(g) ~ 1e-13) wipes the past: the state after that token is beta v k^T."""
    inp = make_inputs(1, 100, 1, 1, 64, 64, dtype="fp32", seed=6, s0_std=1.0, device=DEV)
    inp["g"][0, 99, 0] = -30.0
    o, ST = run(inp)
    b = inp["beta"][0, 99, 0].double()
    ref = b * torch.outer(inp["k"][0, 99, 0].double(), inp["v"][0, 99, 0].double())
    assert rel_l2(ST[0, 0], ref) < 1e-5
    check_full(inp)


def check_every_unit(inp, o, ST, o_ref=None, ST_ref=None, tol=1e-2):
    """o and S_T against the oracle over the whole tensors and unit by unit: every (sequence,
    value head) unit's rel-L2 must pass on its own, so that one bad head or chunk cannot hide
    in a whole-tensor norm."""
    if o_ref is None:
        o_ref, ST_ref = full_oracle(inp)
    assert_every_unit(o, o_ref, inp, "tok", tol, "o")
    assert_every_unit(ST, ST_ref, inp, "state", tol, "S_T")
    return o_ref, ST_ref


@pytest.mark.parametrize("seed", [0, 1])
def test_workload1_full_size_every_unit(seed):
    """B=1, T=4096, H=16, d=128 with a random S0: all 16 heads against the oracle."""
    inp = make_workload(1, seed=seed, device=DEV)
    o, ST = run(inp)
    check_every_unit(inp, o, ST)


def test_workload2_full_size_every_unit():
    """8 packed sequences (512..16384 tokens), 16 q/k heads, 32 value heads: all 256 units."""
    inp = make_workload(2, seed=0, device=DEV)
    o, ST = run(inp)
    check_every_unit(inp, o, ST)


def test_workload3_chained_prefill_equals_single_call():
    """Four 16384-token calls chained through S_T -> S_0 equal one 65536-token call, and both
    match the oracle on every head."""
    inp = make_workload(3, seed=0, device=DEV)
    o, ST = run(inp)
    S = None
    parts = []
    for i in range(4):
        sl = slice(i * 16384, (i + 1) * 16384)
        sub = {k: inp[k][:, sl].contiguous() for k in ("q", "k", "v", "beta", "g")}
        sub["initial_state"] = S
        oi, S = run(sub)
        parts.append(oi)
    oc = torch.cat(parts, 1)
    assert rel_l2(oc, o) < 2e-3
    assert rel_l2(S, ST) < 2e-3
    o_ref, ST_ref = check_every_unit(inp, o, ST)
    check_every_unit(inp, oc, S, o_ref, ST_ref)


# ---- branches of the tensor-core kernels that the workload distributions never reach

def test_tensor_core_exp2_decay_fallback():
    """Inside a chunk the decay factor E_rs = exp(gamma_r - gamma_s) is formed as a_r b_s while
    every |gamma - gamma_31| < 80, else as one exp2 per entry.  Two tokens with g = -60 in the
    same chunk push the in-chunk range past 80 (the tokens before them sit ~60 + the chunk's
    other decay above gamma_31, the last ones ~60 below), so the WY kernel and the fused kernel
    take their exp2 branch for that chunk; the other chunks stay factored."""
    inp = make_inputs(1, 640, 2, 4, 128, 128, dtype="bf16", seed=21, s0_std=0.1, device=DEV)
    for c in (1, 5, 9):  # chunks 1, 5 and 9 of every head
        inp["g"][0, 64 * c + 10, :] = -60.0
        inp["g"][0, 64 * c + 40, :] = -60.0
    g = inp["g"][0, 64:128, 0].double()
    gam = torch.cumsum(g, 0)
    assert (gam - gam[31]).abs().max() >= 80.0  # the branch condition holds
    for flags in (0, GDN_FLAG_SPLIT_FORCE):
        o, ST = run(inp, flags)
        check_every_unit(inp, o, ST)


def test_tensor_core_norm_condition_fallback():
    """A segment that does not start its sequence begins from a zero state a few chunks early
    only while every warm-up token keeps 0 <= beta |k|^2 <= 2 (then each token's state map has
    norm <= exp(g)); a token with beta |k|^2 > 2 in the warm-up makes the segment replay its
    sequence exactly from S0.  Forced short segments (two chunks) and one token per chunk with
    beta = 1.9, |k|^2 = 2.25 (beta |k|^2 = 4.3) reach that branch in every later segment."""
    inp = make_inputs(1, 1024, 1, 2, 128, 128, dtype="bf16", seed=22, s0_std=0.1, device=DEV)
    k = inp["k"].float()
    for c in range(16):
        t = 64 * c + 13
        k[0, t] = k[0, t] * 1.5  # |k|^2 = 2.25 (k is unit-norm)
        inp["beta"][0, t, :] = 1.9
    inp["k"] = k.to(torch.bfloat16)
    assert (inp["beta"][0, 13, 0] * inp["k"][0, 13, 0].float().pow(2).sum()) > 2.0
    for flags in (0, GDN_FLAG_SPLIT_FORCE):
        o, ST = run(inp, flags)
        check_every_unit(inp, o, ST)


def test_tensor_core_weak_decay_forward_fallback():
    """Weak decay, g = -softplus(N(-6, 1)) (about -0.0025 per token): the summed log decay of a
    64-chunk sequence never reaches log(2^-30), so every segment after the first replays its
    sequence from S0 and writes its own outputs (auto split)."""
    inp = make_inputs(1, 4096, 2, 4, 128, 128, dtype="bf16", seed=23, s0_std=0.1, g_mu=-6.0,
                      device=DEV)
    assert float(inp["g"][0, :, 0].double().sum()) > -30 * math.log(2)
    o, ST = run(inp)
    check_every_unit(inp, o, ST)


def test_aliased_initial_and_final_state_is_rejected():
    """S0 and S_T in one buffer (an in-place state update) is rejected on the host: a later
    segment of a split sequence may read S0 after S_T was written."""
    from gated_deltanet_chunked_fwd_b200 import GdnError

    inp = make_inputs(1, 2048, 1, 2, 128, 128, dtype="bf16", seed=24, s0_std=0.1, g_mu=-2.0,
                      device=DEV)
    S = inp["initial_state"]
    for flags in (0, GDN_FLAG_SPLIT_FORCE):
        with pytest.raises(GdnError) as e:
            gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], initial_state=S,
                          final_state=S, flags=flags)
        assert e.value.status == 1  # GDN_ERR_INVALID_ARG


def test_tensor_core_weak_decay_affine_scan():
    """Weak decay (g = -softplus(N(-7, 1))) on 8192 tokens x 16 heads: the split gives nine segments
    of 15 chunks per head and no warm-up reaches log(2^-30), so segments 3-8 take their entry state
    from the affine scan (fold M, B over their own chunks, look back for the nearest published exit
    state, apply the folds in between) and segments 1-2 replay from S0.  Every unit against the
    oracle, and the split run against the unsplit one."""
    inp = make_inputs(1, 8192, 16, 16, 128, 128, dtype="bf16", seed=28, s0_std=0.1, g_mu=-7.0,
                      device=DEV)
    assert float(inp["g"][0, :, :].double().sum(0).max()) > -30 * math.log(2)
    o, ST = run(inp)
    check_every_unit(inp, o, ST)
    o1, ST1 = run(inp, GDN_FLAG_SPLIT_OFF)
    assert rel_l2(o, o1) < 5e-3 and rel_l2(ST, ST1) < 5e-3


def test_tensor_core_weak_decay_varlen_gqa_mixed_scan():
    """Weak decay on a ragged batch with grouped heads (2 q/k heads, 4 value heads): sequences long
    enough to split into several segments take the affine scan for their later segments, short
    ones run unsplit, and the empty and one-token sequences have nothing to scan; every unit
    against the oracle."""
    inp = make_inputs(1, 0, 2, 4, 128, 128, dtype="bf16", seed=32, s0_std=0.1, g_mu=-7.0,
                      lengths=[3000, 200, 0, 9000, 64, 1, 2500], device=DEV)
    o, ST = run(inp)
    check_every_unit(inp, o, ST)


def with_raw_gates(inp, seed):
    """Replace beta and g by raw values for GDN_FLAG_GATE_LOGITS: logits of either sign for beta
    and pre-activations around +1 for g (the layer applies sigmoid and -softplus itself)."""
    gen = torch.Generator().manual_seed(seed)
    shape = inp["beta"].shape
    inp = dict(inp)
    inp["beta"] = (2.0 * torch.randn(shape, generator=gen)).to(inp["beta"].device)
    inp["g"] = (torch.randn(shape, generator=gen) + 1.0).to(inp["g"].device)
    return inp


@pytest.mark.parametrize("dt,flags", [("bf16", 0), ("fp32", 0), ("bf16", GDN_FLAG_PORTABLE)],
                         ids=["tensor-core", "cuda-core-fp32", "cuda-core-bf16"])
def test_gate_logits(dt, flags):
    """GDN_FLAG_GATE_LOGITS: beta and g arrive as logits / pre-activations, ragged sequences,
    grouped heads; o and S_T against the oracle applying sigmoid and -softplus in float64."""
    d = 128 if dt == "bf16" else 64
    inp = with_raw_gates(make_inputs(1, 0, 2, 4, d, d, dtype=dt, seed=33, s0_std=0.1,
                                     lengths=[300, 1, 0, 129], device=DEV), 34)
    o, ST = run(inp, flags | GDN_FLAG_GATE_LOGITS)
    x = cpu(inp)
    o_ref, ST_ref = oracle.fwd(x["q"], x["k"], x["v"], x["beta"], x["g"], cu_seqlens=x["cu_seqlens"],
                               initial_state=x["initial_state"], gate_logits=True)
    tol = TOL[inp["q"].dtype]
    assert rel_l2(o, o_ref) < tol and rel_l2(ST, ST_ref) < tol, (rel_l2(o, o_ref), rel_l2(ST, ST_ref))


def with_raw_qk(inp, seed):
    """Raw q and k rows for GDN_FLAG_QK_L2NORM: the generator's unit rows times random scales in
    [0.3, 3] (and one exactly zero k row), rounded to the tensor dtype again."""
    gen = torch.Generator().manual_seed(seed)
    inp = dict(inp)
    for name in ("q", "k"):
        x = inp[name].float().cpu()
        scale = 0.3 + 2.7 * torch.rand(x.shape[:-1] + (1,), generator=gen)
        x = x * scale
        if name == "k" and x.shape[1] > 5:
            x[0, 5] = 0.0
        inp[name] = x.to(inp[name].dtype).to(inp[name].device)
    return inp


@pytest.mark.parametrize("dt,flags", [("bf16", 0), ("fp32", 0), ("bf16", GDN_FLAG_PORTABLE)],
                         ids=["tensor-core", "cuda-core-fp32", "cuda-core-bf16"])
@pytest.mark.parametrize("gates", [False, True], ids=["qk-norm", "qk-norm+gate-logits"])
def test_qk_l2norm(dt, flags, gates):
    """GDN_FLAG_QK_L2NORM: raw q and k rows (scales 0.3-3, one zero row), ragged sequences,
    grouped heads, alone and with GDN_FLAG_GATE_LOGITS; o and S_T against the oracle
    normalising in float64."""
    d = 128 if dt == "bf16" else 64
    inp = with_raw_qk(make_inputs(1, 0, 2, 4, d, d, dtype=dt, seed=39, s0_std=0.1,
                                  lengths=[300, 1, 0, 129], device=DEV), 40)
    if gates:
        inp = with_raw_gates(inp, 41)
    f = flags | GDN_FLAG_QK_L2NORM | (GDN_FLAG_GATE_LOGITS if gates else 0)
    o, ST = run(inp, f)
    x = cpu(inp)
    o_ref, ST_ref = oracle.fwd(x["q"], x["k"], x["v"], x["beta"], x["g"], cu_seqlens=x["cu_seqlens"],
                               initial_state=x["initial_state"], qk_l2norm=True, gate_logits=gates)
    tol = TOL[inp["q"].dtype]
    assert rel_l2(o, o_ref) < tol and rel_l2(ST, ST_ref) < tol, (rel_l2(o, o_ref), rel_l2(ST, ST_ref))
