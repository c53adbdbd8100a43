"""GPU parity of the decode step (gdn_decode_step through the C ABI) against the float64
oracle: one token per sequence is the oracle's token loop with T = 1 and the state passed as
S0; a run of decode steps equals one oracle call over those tokens; prefill then decode equals
prefill over one more token; a state pool addressed by indices updates only its own slots."""
import pytest
import torch

import oracle
from gated_deltanet_chunked_fwd_b200 import gdn_chunk_fwd, gdn_decode_step
from gated_deltanet_chunked_fwd_b200.inputs import make_inputs
from tests._helpers import TOL, assert_every_unit, cpu, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"


def decode_inputs(N, Hk, Hv, dk, dv, dtype, seed, s_std=0.3):
    """One token per sequence ([N, 1, ...] from the shared generator) and a random state."""
    x = make_inputs(N, 1, Hk, Hv, dk, dv, dtype=dtype, seed=seed, s0_std=s_std, device=DEV)
    return x


def oracle_step(x, S):
    c = cpu(x)
    return oracle.fwd(c["q"], c["k"], c["v"], c["beta"], c["g"], initial_state=S.cpu())


def gpu_step(x, S, idx=None):
    c0 = {n: x[n][:, 0].contiguous() for n in ("q", "k", "v", "beta", "g")}
    o = gdn_decode_step(c0["q"], c0["k"], c0["v"], c0["beta"],
                        c0["g"], S, state_indices=idx, check_device_status=True)
    torch.cuda.synchronize()
    return o


@pytest.mark.parametrize("dt,Hk,Hv,dk,dv", [("fp32", 2, 4, 128, 128), ("bf16", 2, 4, 128, 128),
                                            ("fp32", 1, 3, 64, 32), ("bf16", 3, 3, 100, 124)])
def test_one_step_matches_oracle(dt, Hk, Hv, dk, dv):
    x = decode_inputs(5, Hk, Hv, dk, dv, dt, seed=31)
    S = x["initial_state"].clone()
    o_ref, S_ref = oracle_step(x, S)
    o = gpu_step(x, S)
    tol = TOL[x["q"].dtype]
    assert rel_l2(o, o_ref[:, 0]) < tol
    assert rel_l2(S, S_ref) < 1e-5  # the state stays fp32 throughout


@pytest.mark.parametrize("dt", ["fp32", "bf16"])
def test_sixteen_steps_equal_one_oracle_call(dt):
    T = 16
    x = make_inputs(3, T, 2, 4, 128, 128, dtype=dt, seed=32, s0_std=0.2, device=DEV)
    S = x["initial_state"].clone()
    outs = []
    for t in range(T):
        step = {n: x[n][:, t:t + 1] for n in ("q", "k", "v", "beta", "g")}
        outs.append(gpu_step(step, S))
    o = torch.stack(outs, 1)
    c = cpu(x)
    o_ref, S_ref = oracle.fwd(c["q"], c["k"], c["v"], c["beta"], c["g"], initial_state=c["initial_state"])
    tol = TOL[x["q"].dtype]
    assert rel_l2(o, o_ref) < tol
    assert rel_l2(S, S_ref) < (1e-5 if dt == "fp32" else 1e-4)


def test_prefill_then_decode_equals_longer_prefill():
    """The S_T of a 300-token prefill (tensor-core forward) fed to a decode step equals the
    oracle over 301 tokens (last output and final state)."""
    x = make_inputs(1, 301, 2, 4, 128, 128, dtype="bf16", seed=33, s0_std=0.1, device=DEV)
    pre = {n: x[n][:, :300].contiguous() for n in ("q", "k", "v", "beta", "g")}
    _, S = gdn_chunk_fwd(pre["q"], pre["k"], pre["v"], pre["beta"], pre["g"],
                         initial_state=x["initial_state"])
    last = {n: x[n][:, 300:301] for n in ("q", "k", "v", "beta", "g")}
    o = gpu_step(last, S)
    c = cpu(x)
    o_ref, S_ref = oracle.fwd(c["q"], c["k"], c["v"], c["beta"], c["g"], initial_state=c["initial_state"])
    assert rel_l2(o, o_ref[:, 300]) < 1e-2
    assert rel_l2(S, S_ref) < 1e-2


def test_state_pool_with_indices():
    """Sequences address slots of a pool in a shuffled order; a negative index skips its sequence
    (zero output) and slots that no sequence names stay untouched."""
    N, slots = 6, 10
    x = decode_inputs(N, 2, 4, 128, 128, "bf16", seed=34)
    gen = torch.Generator().manual_seed(5)
    pool = 0.3 * torch.randn(slots, 4, 128, 128, generator=gen)
    idx = torch.tensor([7, 2, -1, 0, 9, 4], dtype=torch.int32)
    pool_d = pool.to(DEV)
    o = gpu_step(x, pool_d, idx.to(DEV))
    live = [n for n in range(N) if idx[n] >= 0]
    S_in = torch.stack([pool[int(idx[n])] for n in live])
    sub = {k_: x[k_][live] for k_ in ("q", "k", "v", "beta", "g")}
    o_ref, S_ref = oracle_step(sub, S_in)
    assert rel_l2(o[live], o_ref[:, 0]) < 1e-2
    assert torch.count_nonzero(o[2]) == 0
    for j, n in enumerate(live):
        assert rel_l2(pool_d[int(idx[n])], S_ref[j]) < 1e-5
    untouched = [s for s in range(slots) if s not in idx.tolist()]
    assert torch.equal(pool_d[untouched].cpu(), pool[untouched])


def test_decode_workload_every_unit():
    """The decode workload: 64 sequences, 16 q/k heads, 32 value heads, d = 128, bf16 tokens,
    fp32 states (134 MB, read and written once); every (sequence, head) unit against the oracle."""
    x = decode_inputs(64, 16, 32, 128, 128, "bf16", seed=35, s_std=0.1)
    S = x["initial_state"].clone()
    o_ref, S_ref = oracle_step(x, S)
    o = gpu_step(x, S)
    inp1 = {"q": x["q"], "v": x["v"]}
    assert_every_unit(o[:, None], o_ref, inp1, "tok", 1e-2, "o")
    assert_every_unit(S, S_ref, inp1, "state", 1e-5, "S")


@pytest.mark.parametrize("dt", ["fp32", "bf16"])
def test_gate_logits(dt):
    """GDN_FLAG_GATE_LOGITS in the decode step: beta and g as logits / pre-activations."""
    from gated_deltanet_chunked_fwd_b200 import GDN_FLAG_GATE_LOGITS

    x = decode_inputs(6, 2, 4, 128, 128, dt, seed=37)
    gen = torch.Generator().manual_seed(38)
    x["beta"] = (2.0 * torch.randn(x["beta"].shape, generator=gen)).to(DEV)
    x["g"] = (torch.randn(x["g"].shape, generator=gen) + 1.0).to(DEV)
    S = x["initial_state"].clone()
    c = cpu(x)
    o_ref, S_ref = oracle.fwd(c["q"], c["k"], c["v"], c["beta"], c["g"], initial_state=S.cpu(),
                              gate_logits=True)
    c0 = {n: x[n][:, 0].contiguous() for n in ("q", "k", "v", "beta", "g")}
    o = gdn_decode_step(c0["q"], c0["k"], c0["v"], c0["beta"], c0["g"], S, flags=GDN_FLAG_GATE_LOGITS,
                        check_device_status=True)
    torch.cuda.synchronize()
    assert rel_l2(o, o_ref[:, 0]) < TOL[x["q"].dtype]
    assert rel_l2(S, S_ref) < 1e-5


@pytest.mark.parametrize("dt", ["fp32", "bf16"])
def test_qk_l2norm(dt):
    """GDN_FLAG_QK_L2NORM (with GDN_FLAG_GATE_LOGITS) in the decode step: raw q, k rows."""
    from gated_deltanet_chunked_fwd_b200 import GDN_FLAG_GATE_LOGITS, GDN_FLAG_QK_L2NORM

    x = decode_inputs(6, 2, 4, 128, 128, dt, seed=47)
    gen = torch.Generator().manual_seed(48)
    for name in ("q", "k"):
        y = x[name].float().cpu() * (0.3 + 2.7 * torch.rand(x[name].shape[:-1] + (1,), generator=gen))
        x[name] = y.to(x[name].dtype).to(DEV)
    x["beta"] = (2.0 * torch.randn(x["beta"].shape, generator=gen)).to(DEV)
    x["g"] = (torch.randn(x["g"].shape, generator=gen) + 1.0).to(DEV)
    S = x["initial_state"].clone()
    c = cpu(x)
    o_ref, S_ref = oracle.fwd(c["q"], c["k"], c["v"], c["beta"], c["g"], initial_state=S.cpu(),
                              qk_l2norm=True, gate_logits=True)
    c0 = {n: x[n][:, 0].contiguous() for n in ("q", "k", "v", "beta", "g")}
    o = gdn_decode_step(c0["q"], c0["k"], c0["v"], c0["beta"], c0["g"], S,
                        flags=GDN_FLAG_QK_L2NORM | GDN_FLAG_GATE_LOGITS, check_device_status=True)
    torch.cuda.synchronize()
    assert rel_l2(o, o_ref[:, 0]) < TOL[x["q"].dtype]
    assert rel_l2(S, S_ref) < TOL[x["q"].dtype]
