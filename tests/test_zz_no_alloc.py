"""gdn_chunk_fwd_noalloc: the forward for callers that cannot allocate device memory
(framework plugins or servers whose device memory is pooled and frozen after start-up).

It keeps its scratch in a fixed device array inside libgdn.so instead of a
caller-provided workspace.  Checked here through the C ABI against the regular
gdn_chunk_fwd on the same inputs and against the float64 oracle, on two calls
in a row (the array keeps the previous call's contents, which must not leak
into the next result).  This file
is collected last on purpose, so that a failure here stops a `-x` run only after
every other test has run."""
import ctypes

import oracle
import pytest
import torch

from gated_deltanet_chunked_fwd_b200 import _abi, _fill_common, gdn_chunk_fwd
from gated_deltanet_chunked_fwd_b200.inputs import make_inputs
from tests._helpers import TOL, cpu, rel_l2

pytestmark = pytest.mark.gpu


def call_noalloc(x):
    """o, S_T from gdn_chunk_fwd_noalloc (outputs allocated by the test, not the library)."""
    q, k, v, beta, g = x["q"], x["k"], x["v"], x["beta"], x["g"]
    a = _abi.GdnFwdArgs()
    N, host = _fill_common(a, q, k, v, beta, g, x.get("cu_seqlens"), x.get("cu_seqlens_host"),
                           x.get("initial_state"), 0)
    o = torch.empty(q.shape[0], q.shape[1], v.shape[2], v.shape[3], dtype=q.dtype, device=q.device)
    ST = torch.empty(N, v.shape[2], q.shape[3], v.shape[3], dtype=torch.float32, device=q.device)
    a.o, a.ST = o.data_ptr(), ST.data_ptr()
    st = _abi.lib().gdn_chunk_fwd_noalloc(ctypes.byref(a),
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, _abi.status_string(st)
    torch.cuda.synchronize()
    del host
    return o, ST


@pytest.mark.parametrize("dt,lengths,s0", [("bf16", None, 0.1), ("fp32", [70, 1, 300, 64], 0.2)])
def test_noalloc_matches_gdn_chunk_fwd_twice(dt, lengths, s0):
    for seed in (11, 12):  # two calls in a row, different inputs
        x = make_inputs(1, 640, 2, 4, 128, 128, dtype=dt, seed=seed, s0_std=s0, lengths=lengths,
                        device="cuda")
        o_ref, ST_ref = gdn_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["g"],
                                      cu_seqlens=x.get("cu_seqlens"),
                                      cu_seqlens_host=x.get("cu_seqlens_host"),
                                      initial_state=x.get("initial_state"))
        o, ST = call_noalloc(x)
        tol = TOL[x["q"].dtype]
        assert rel_l2(o, o_ref) < tol, rel_l2(o, o_ref)
        assert rel_l2(ST, ST_ref) < tol, rel_l2(ST, ST_ref)
        c = cpu(x)
        o_or, ST_or = oracle.fwd(c["q"], c["k"], c["v"], c["beta"], c["g"],
                                 cu_seqlens=c.get("cu_seqlens"), initial_state=c.get("initial_state"))
        assert rel_l2(o, o_or) < tol, rel_l2(o, o_or)
        assert rel_l2(ST, ST_or) < tol, rel_l2(ST, ST_or)


def test_noalloc_rejects_problems_beyond_its_scratch():
    x = make_inputs(1, 64 * 600, 1, 1, 128, 128, dtype="bf16", seed=1, device="cuda")
    a = _abi.GdnFwdArgs()
    _, host = _fill_common(a, x["q"], x["k"], x["v"], x["beta"], x["g"], None, None, None, 0)
    o = torch.empty_like(x["v"])
    a.o = o.data_ptr()
    st = _abi.lib().gdn_chunk_fwd_noalloc(ctypes.byref(a), None)
    assert st == 7, _abi.status_string(st)  # GDN_ERR_TOO_LARGE, nothing enqueued
