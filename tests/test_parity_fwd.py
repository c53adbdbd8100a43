"""GPU forward parity: libgdn (through the C ABI) against the float64 oracle on
the same seeded inputs, element by element over whole tensors (rel-L2 bars in
_helpers.TOL), at sizes that span several chunks and a ragged tail, and at the
full workload sizes on sampled (sequence, head) units the oracle computes alone."""
import math

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_chunked_fwd_b200 import (GDN_FLAG_PORTABLE, GDN_FLAG_SPLIT_FORCE,
                                             GDN_FLAG_SPLIT_OFF, gdn_chunk_fwd)
from gated_deltanet_chunked_fwd_b200.inputs import make_inputs, make_workload
from tests._helpers import TOL, cpu, gpu_unit, oracle_fwd_units, rel_l2

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


@pytest.mark.parametrize("seed", [0, 1])
def test_workload1_full_size_sampled_heads(seed):
    inp = make_workload(1, seed=seed, device=DEV)
    o, ST = run(inp)
    assert torch.isfinite(o.float()).all()
    for (n, h), (o_ref, ST_ref) in oracle_fwd_units(inp, [(0, 0), (0, 9), (0, 15)]).items():
        og, Sg = gpu_unit(inp, o, ST, n, h)
        assert rel_l2(og, o_ref) < 1e-2, (h, rel_l2(og, o_ref))
        assert rel_l2(Sg, ST_ref) < 1e-2


def test_workload2_full_size_sampled_units():
    inp = make_workload(2, seed=0, device=DEV)
    o, ST = run(inp)
    for (n, h), (o_ref, ST_ref) in oracle_fwd_units(inp, [(0, 0), (3, 17), (7, 31)]).items():
        og, Sg = gpu_unit(inp, o, ST, n, h)
        assert rel_l2(og, o_ref) < 1e-2, ((n, h), rel_l2(og, o_ref))
        assert rel_l2(Sg, ST_ref) < 1e-2


def test_workload3_chained_prefill_equals_single_call():
    """Four 16384-token calls chained through S_T -> S_0 equal one 65536-token call."""
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
    for (n, h), (o_ref, ST_ref) in oracle_fwd_units(inp, [(0, 5)]).items():
        assert rel_l2(o[0, :, h], o_ref) < 1e-2
        assert rel_l2(ST[0, h], ST_ref) < 1e-2
        assert rel_l2(oc[0, :, h], o_ref) < 1e-2
        assert rel_l2(S[0, h], ST_ref) < 1e-2
