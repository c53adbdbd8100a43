"""GPU backward parity: libgdn's gdn_chunk_bwd against the oracle's float64
adjoint on the same seeded inputs (dq, dk, dv, dbeta, dg, dS0), whole tensors
at small sizes, and whole tensors plus every (sequence, head) unit on its own at
the full backward workload size."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_chunked_fwd_b200 import (GDN_FLAG_PORTABLE, GDN_FLAG_SPLIT_FORCE,
                                             GDN_FLAG_SPLIT_OFF, gdn_chunk_bwd)
from gated_deltanet_chunked_fwd_b200.inputs import make_inputs, make_workload
from tests._helpers import TOL, assert_every_unit, cpu, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"
NAMES = ["dq", "dk", "dv", "dbeta", "dg", "dS0"]


def run(inp, flags=0):
    res = gdn_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["do"],
                        cu_seqlens=inp.get("cu_seqlens"), initial_state=inp.get("initial_state"),
                        dST=inp.get("dST"), cu_seqlens_host=inp.get("cu_seqlens_host"),
                        flags=flags, check_device_status=True)
    torch.cuda.synchronize()
    return res


def ref(inp):
    x = cpu(inp)
    return oracle.bwd(x["q"], x["k"], x["v"], x["beta"], x["g"], x["do"],
                      cu_seqlens=x.get("cu_seqlens"), initial_state=x.get("initial_state"),
                      dST=x.get("dST"))


def compare(mine, refs, tol, label=""):
    for name, a, b in zip(NAMES, mine, refs):
        err = rel_l2(a, b)
        assert err < tol, f"{label} {name}: rel-L2 {err:.3e} >= {tol}"


CASES = [
    ("fp32", 1, 1, 1, 1, 16, 16, 0.5),
    ("fp32", 1, 150, 1, 1, 64, 64, 0.5),
    ("fp32", 2, 65, 2, 4, 32, 48, 0.5),
    ("fp32", 1, 200, 1, 2, 128, 128, 0.1),
    ("bf16", 1, 130, 1, 1, 128, 128, 0.1),
    ("bf16", 2, 64, 2, 4, 128, 128, None),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_small_shapes(case):
    dt, B, T, Hk, Hv, dk, dv, s0 = case
    inp = make_inputs(B, T, Hk, Hv, dk, dv, dtype=dt, seed=7, s0_std=s0, backward=True, device=DEV)
    compare(run(inp), ref(inp), TOL[inp["q"].dtype], str(case))


@pytest.mark.parametrize("dt", ["fp32", "bf16"])
def test_varlen_ragged(dt):
    inp = make_inputs(1, 0, 2, 4, 64, 64, dtype=dt, seed=8, s0_std=0.2, backward=True,
                      lengths=[3, 64, 0, 129, 1], device=DEV)
    compare(run(inp), ref(inp), TOL[inp["q"].dtype], dt)


def test_zero_upstream_state_gradient_and_no_S0():
    inp = make_inputs(1, 100, 1, 1, 64, 64, dtype="fp32", seed=9, backward=True, device=DEV)
    inp["dST"] = None
    compare(run(inp), ref(inp), 1e-4)


def test_reduced_backward_workload_full_oracle():
    """The backward workload's shape reduced to B=1, T=1024, H=2, d=128, whole tensors."""
    inp = make_workload(4, seed=0, device=DEV, B=1, T=1024, Hk=2, Hv=2)
    compare(run(inp), ref(inp), 1e-2, "reduced")


def test_backward_workload_full_size_every_unit():
    """B=4, T=8192, H=16, d=128: all six gradients against the oracle adjoint over whole
    tensors and for every (sequence, head) unit on its own."""
    inp = make_workload(4, seed=0, device=DEV)
    mine = run(inp)
    refs = ref(inp)
    kinds = ["tok", "tok", "tok", "vec", "vec", "state"]
    for name, a, b, kind in zip(NAMES, mine, refs, kinds):
        assert_every_unit(a, b, inp, kind, 1e-2, name)


@pytest.mark.parametrize("flags", [0, GDN_FLAG_PORTABLE], ids=["tensor-core", "portable"])
def test_varlen_ragged_d128_bf16(flags):
    """bf16 d=128: the shape the tensor-core backward takes (flags=0) and the CUDA-core
    kernels (portable), on ragged sequences with empty and single-token ones, GQA 2:4."""
    inp = make_inputs(1, 0, 2, 4, 128, 128, dtype="bf16", seed=11, s0_std=0.2, backward=True,
                      lengths=[3, 64, 0, 129, 1, 200], device=DEV)
    compare(run(inp, flags), ref(inp), TOL[inp["q"].dtype], f"flags={flags}")


def test_tensor_core_and_portable_backward_agree():
    """The two backward implementations on the same bf16 input agree with each other
    at least as closely as each agrees with the oracle."""
    inp = make_inputs(2, 300, 1, 2, 128, 128, dtype="bf16", seed=12, s0_std=0.1, backward=True,
                      device=DEV)
    a, b, r = run(inp), run(inp, GDN_FLAG_PORTABLE), ref(inp)
    compare(a, r, TOL[inp["q"].dtype], "tensor-core")
    compare(b, r, TOL[inp["q"].dtype], "portable")
    compare(a, [t.double().cpu() for t in b], TOL[inp["q"].dtype], "tc vs portable")


@pytest.mark.parametrize("flags", [GDN_FLAG_SPLIT_OFF, GDN_FLAG_SPLIT_FORCE], ids=["split-off", "split-force"])
def test_tensor_core_split_modes(flags):
    """The tensor-core backward with one segment per sequence (no warm-ups) and with
    two-chunk segments (reverse warm-ups at every segment end), ragged varlen, GQA 2:4."""
    inp = make_inputs(1, 0, 2, 4, 128, 128, dtype="bf16", seed=13, s0_std=0.2, backward=True,
                      lengths=[3, 64, 0, 300, 1, 200], device=DEV)
    compare(run(inp, flags), ref(inp), TOL[inp["q"].dtype], f"flags={flags}")


def test_tensor_core_slow_decay_exact_fallback():
    """Slow decay (g = -softplus(N(-6, 1)), |sum g| over a chunk ~ 0.16): reverse warm-ups never
    reach the 2^-30 bound, so every segment runs from dS_T at the sequence end."""
    inp = make_inputs(2, 700, 1, 2, 128, 128, dtype="bf16", seed=14, s0_std=0.1, g_mu=-6.0,
                      backward=True, device=DEV)
    compare(run(inp), ref(inp), TOL[inp["q"].dtype], "slow decay")


def test_tensor_core_exp2_decay_fallback():
    """Two tokens with g = -60 in one chunk push the chunk's in-chunk log-decay range past 80,
    where the WY, replay and reverse kernels form exp(gamma_r - gamma_s) by exp2 per entry
    instead of the factored a_r b_s."""
    inp = make_inputs(1, 640, 2, 4, 128, 128, dtype="bf16", seed=25, s0_std=0.1, backward=True,
                      device=DEV)
    for c in (1, 5, 9):
        inp["g"][0, 64 * c + 10, :] = -60.0
        inp["g"][0, 64 * c + 40, :] = -60.0
    r = ref(inp)
    for flags in (0, GDN_FLAG_SPLIT_FORCE):
        compare(run(inp, flags), r, TOL[inp["q"].dtype], f"exp2 flags={flags}")


def test_tensor_core_norm_condition_fallback():
    """Tokens with beta |k|^2 > 2 in every chunk: no segment may start from a truncated
    warm-up (forward states or reverse adjoint), so every segment runs exactly."""
    inp = make_inputs(1, 1024, 1, 2, 128, 128, dtype="bf16", seed=26, s0_std=0.1, backward=True,
                      device=DEV)
    k = inp["k"].float()
    for c in range(16):
        t = 64 * c + 13
        k[0, t] = k[0, t] * 1.5
        inp["beta"][0, t, :] = 1.9
    inp["k"] = k.to(torch.bfloat16)
    r = ref(inp)
    for flags in (0, GDN_FLAG_SPLIT_FORCE):
        compare(run(inp, flags), r, TOL[inp["q"].dtype], f"norm flags={flags}")


def test_aliased_state_gradient_is_rejected():
    """dS0 sharing memory with S0 or dS_T is rejected on the host before anything runs."""
    import ctypes

    from gated_deltanet_chunked_fwd_b200 import _abi, _fill_common

    inp = make_inputs(1, 256, 1, 2, 128, 128, dtype="bf16", seed=27, s0_std=0.1, backward=True,
                      device=DEV)
    outs = [torch.empty_like(inp[n]) for n in ("q", "k", "v", "beta", "g")]
    for alias in ("initial_state", "dST"):
        a = _abi.GdnBwdArgs()
        _, host = _fill_common(a, inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], None, None,
                               inp["initial_state"], 0)
        a.dout, a.dST = inp["do"].data_ptr(), inp["dST"].data_ptr()
        a.dq, a.dk_out, a.dv_out, a.dbeta, a.dg = (t.data_ptr() for t in outs)
        a.dS0 = inp[alias].data_ptr()
        n = ctypes.c_size_t(0)
        assert _abi.lib().gdn_chunk_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
        ws = torch.empty(max(n.value, 1), dtype=torch.uint8, device=DEV)
        st = _abi.lib().gdn_chunk_bwd(ctypes.byref(a), ctypes.c_void_p(ws.data_ptr()), n.value, None)
        assert st == 1, alias  # GDN_ERR_INVALID_ARG


def test_tensor_core_weak_decay_affine_scan_replay():
    """Weak decay on 8192 tokens x 16 heads: in the state replay segments 3-8 of each head take
    their entry state from the affine scan (see the forward test), and in the reverse walks (nine
    15-chunk segments per head) segments 0-7 take their exit adjoint from the adjoint scan while the
    last one first walks its chunks without gradients to publish its exit adjoint; all six
    gradients against the oracle adjoint."""
    inp = make_inputs(1, 8192, 16, 16, 128, 128, dtype="bf16", seed=29, s0_std=0.1, g_mu=-7.0,
                      backward=True, device=DEV)
    compare(run(inp), ref(inp), TOL[inp["q"].dtype], "weak decay scan")


def test_tensor_core_weak_decay_adjoint_scan_long_fold_chain():
    """Weak decay on 16384 tokens x 2 heads: the reverse walks split into 64 four-chunk segments per
    head, no reverse warm-up reaches the 2^-30 bound, and the first 63 segments of each head take
    their exit adjoint from the adjoint scan (folds of up to 62 later segments combined); all six
    gradients against the oracle adjoint."""
    inp = make_inputs(1, 16384, 2, 2, 128, 128, dtype="bf16", seed=30, s0_std=0.1, g_mu=-7.0,
                      backward=True, device=DEV)
    compare(run(inp), ref(inp), TOL[inp["q"].dtype], "adjoint scan, long fold chain")


def test_tensor_core_weak_decay_varlen_gqa_mixed_scan():
    """Weak decay on a ragged batch with grouped heads (2 q/k heads, 4 value heads): the long
    sequences split into enough reverse segments for the adjoint scan, the short ones replay or
    run unsplit, and the empty and one-token sequences have no chunk to scan; all six gradients
    against the oracle adjoint."""
    inp = make_inputs(1, 0, 2, 4, 128, 128, dtype="bf16", seed=31, s0_std=0.1, g_mu=-7.0,
                      backward=True, lengths=[3000, 200, 0, 9000, 64, 1, 2500], device=DEV)
    compare(run(inp), ref(inp), TOL[inp["q"].dtype], "weak decay varlen GQA")


@pytest.mark.parametrize("dt,flags", [("bf16", 0), ("fp32", 0)], ids=["tensor-core", "cuda-core-fp32"])
def test_gate_logits(dt, flags):
    """GDN_FLAG_GATE_LOGITS: dbeta and dg are gradients with respect to the raw logits /
    pre-activations; all six gradients against the oracle's chain rule, ragged, grouped heads."""
    from gated_deltanet_chunked_fwd_b200 import GDN_FLAG_GATE_LOGITS
    from tests.test_parity_fwd import with_raw_gates

    d = 128 if dt == "bf16" else 64
    inp = with_raw_gates(make_inputs(1, 0, 2, 4, d, d, dtype=dt, seed=35, s0_std=0.1, backward=True,
                                     lengths=[300, 1, 0, 129], device=DEV), 36)
    x = cpu(inp)
    refs = oracle.bwd(x["q"], x["k"], x["v"], x["beta"], x["g"], x["do"], cu_seqlens=x["cu_seqlens"],
                      initial_state=x["initial_state"], dST=x["dST"], gate_logits=True)
    compare(run(inp, flags | GDN_FLAG_GATE_LOGITS), refs, TOL[inp["q"].dtype], "gate logits")


@pytest.mark.parametrize("dt,flags", [("bf16", 0), ("fp32", 0)], ids=["tensor-core", "cuda-core-fp32"])
@pytest.mark.parametrize("gates", [False, True], ids=["qk-norm", "qk-norm+gate-logits"])
def test_qk_l2norm(dt, flags, gates):
    """GDN_FLAG_QK_L2NORM: dq and dk are gradients with respect to the raw rows (the reduction
    kernel applies the normalisation's chain rule after the group sum), alone and with
    GDN_FLAG_GATE_LOGITS; all six gradients against the oracle, ragged, grouped heads."""
    from gated_deltanet_chunked_fwd_b200 import GDN_FLAG_GATE_LOGITS, GDN_FLAG_QK_L2NORM
    from tests.test_parity_fwd import with_raw_gates, with_raw_qk

    d = 128 if dt == "bf16" else 64
    inp = with_raw_qk(make_inputs(1, 0, 2, 4, d, d, dtype=dt, seed=42, s0_std=0.1, backward=True,
                                  lengths=[300, 1, 0, 129], device=DEV), 43)
    if gates:
        inp = with_raw_gates(inp, 44)
    x = cpu(inp)
    refs = oracle.bwd(x["q"], x["k"], x["v"], x["beta"], x["g"], x["do"], cu_seqlens=x["cu_seqlens"],
                      initial_state=x["initial_state"], dST=x["dST"], qk_l2norm=True, gate_logits=gates)
    f = flags | GDN_FLAG_QK_L2NORM | (GDN_FLAG_GATE_LOGITS if gates else 0)
    compare(run(inp, f), refs, TOL[inp["q"].dtype], f"qk norm gates={gates}")


def test_qk_l2norm_ungrouped_tensor_core():
    """GDN_FLAG_QK_L2NORM without grouped heads: dq / dk go through the fp32 per-head buffers and
    the reduction kernel instead of the direct bf16 stores."""
    from gated_deltanet_chunked_fwd_b200 import GDN_FLAG_QK_L2NORM
    from tests.test_parity_fwd import with_raw_qk

    inp = with_raw_qk(make_inputs(2, 200, 2, 2, 128, 128, dtype="bf16", seed=45, s0_std=0.1,
                                  backward=True, device=DEV), 46)
    x = cpu(inp)
    refs = oracle.bwd(x["q"], x["k"], x["v"], x["beta"], x["g"], x["do"], initial_state=x["initial_state"],
                      dST=x["dST"], qk_l2norm=True)
    compare(run(inp, GDN_FLAG_QK_L2NORM), refs, TOL[inp["q"].dtype], "qk norm ungrouped")
