"""The seeded input generator: shapes, determinism and the stated distributions."""
import torch

from gated_deltanet_chunked_fwd_b200.inputs import WORKLOADS, make_inputs, make_workload


def test_deterministic_and_seeded():
    a = make_inputs(1, 64, 2, 4, 16, 8, dtype="bf16", seed=3, s0_std=0.1, backward=True)
    b = make_inputs(1, 64, 2, 4, 16, 8, dtype="bf16", seed=3, s0_std=0.1, backward=True)
    c = make_inputs(1, 64, 2, 4, 16, 8, dtype="bf16", seed=4, s0_std=0.1, backward=True)
    for key in ("q", "k", "v", "beta", "g", "initial_state", "do", "dST"):
        assert torch.equal(a[key], b[key])
        assert not torch.equal(a[key], c[key])


def test_shapes_dtypes_and_ranges():
    x = make_inputs(2, 100, 2, 4, 16, 8, dtype="fp32", seed=0, s0_std=0.1)
    assert x["q"].shape == (2, 100, 2, 16) and x["v"].shape == (2, 100, 4, 8)
    assert x["beta"].shape == (2, 100, 4) and x["g"].dtype == torch.float32
    assert x["initial_state"].shape == (2, 4, 16, 8)
    assert torch.allclose(x["q"].norm(dim=-1), torch.ones(2, 100, 2), atol=1e-5)
    assert (x["beta"] > 0).all() and (x["beta"] < 1).all() and (x["g"] <= 0).all()


def test_varlen_lengths_and_offsets():
    x = make_inputs(
        1, 0, 2, 4, 16, 8, dtype="bf16", seed=0, varlen=(8, 512, 16384))
    cu = x["cu_seqlens"]
    lens = (cu[1:] - cu[:-1]).tolist()
    assert len(lens) == 8 and all(512 <= n <= 16384 for n in lens)
    assert int(cu[-1]) == x["q"].shape[1] and cu.dtype == torch.int32


def test_workload_table():
    names = [w.name for w in WORKLOADS]
    assert len(names) == 5 and len(set(names)) == 5
    small = make_workload(0)
    assert small["q"].dtype == torch.float32 and small["q"].shape == (1, 256, 2, 64)
    assert small["initial_state"] is None
