"""bench.py's host-side arithmetic: the roofline bound, the algorithmic byte and FLOP counts of
the measured workloads, and the comment-blind source fingerprint that keys the ncu traffic."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_strip_comments_keeps_code_only():
    src = "int a; // note\n/* block\n comment */ int  b;\n"
    assert bench.strip_comments(src) == "int a; int b;"


def test_fingerprint_ignores_comments(tmp_path, monkeypatch):
    d = tmp_path / "gated_deltanet_chunked_fwd_b200" / "csrc"
    d.mkdir(parents=True)
    (d / "x.cu").write_text("int a; // one\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h1 = bench.source_sha16(("x.cu",))
    (d / "x.cu").write_text("/* two */ int a;\n")
    assert bench.source_sha16(("x.cu",)) == h1
    (d / "x.cu").write_text("int b;\n")
    assert bench.source_sha16(("x.cu",)) != h1


def test_forward_bytes_and_flops_per_token_head():
    # 2 (2 dk + 2 dv) bf16 + beta, g fp32 = 1,032 B per token-head at d = 128
    assert bench.fwd_bytes(1, 1, 1, 128, 128, 0) == 1032
    # the headline workload: 65,536 tokens x 16 heads, zero S0, S_T written
    b = bench.fwd_bytes(65536, 16, 16, 128, 128, 1, s0=False, st=True)
    assert b == 65536 * 16 * 1032 + 16 * 128 * 128 * 4
    dense, tri = bench.flops_per_token_head(128, 128)
    assert dense == 180224 and tri == pytest.approx(140629.33, abs=0.01)


def test_roofline_bound_is_the_larger_time():
    hbm, tc = 6546.6, 1648.7
    r = bench.roofline(flops_dense=1e9, byts=1e9, seconds=1e-3, hbm_gbs=hbm, bf16_tflops=tc, src="x")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["frac"] == pytest.approx(1e9 / 1e-3 / 1e9 / hbm)
    assert r["t_roof_us"] == pytest.approx(1e9 / (hbm * 1e9) * 1e6)
    r = bench.roofline(flops_dense=1e13, byts=1e6, seconds=0.02, hbm_gbs=hbm, bf16_tflops=tc, src="x")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["frac"] == pytest.approx(r["frac_tensor"])


def test_decode_bytes():
    # one state read and written (2 x 64 KB) + q, k (shared by 2 heads) + v, o bf16 + beta, g
    b = bench.decode_bytes(1, 1, 2, 128, 128)
    assert b == 2 * (2 * 65536 + 2 * 256 + 8) + 2 * 256
