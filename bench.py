"""Throughput of the GDN chunked-prefill forward on B200, one JSON line.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

A step is one forward pass of the layer over one batch of the long-context bf16
workload: B=1, T=65,536 tokens, H=16 heads, dk=dv=128, C=64, slow decay
(g = -softplus(N(-2,1))), zero initial state, through the C ABI, inputs already
resident in HBM (1.08 GB of algorithmic traffic, well above the 126 MB L2; the
L2 is also flushed by a 2 x L2-size write before every timed step, outside the
timed events).  ``value`` is whole-job tokens/s; with N GPUs every rank runs
its own replica (weak scaling, no collective on the data path) and the time is
the max over ranks.  ``e2e`` times the same call with the inputs in pinned host
memory, including the host->device copies of the inputs and the device->host
copies of o and S_T.

Extra keys, each timed the same way: ``fwd_workloads`` holds the 4,096-token
forward with a random initial state, the packed varlen batch (8 sequences,
16 q/k heads, 32 value heads) and the long context fed as 4 chained
16,384-token calls; ``bwd`` the backward on the B=4, T=8192, H=16 workload.
``fwd_workloads`` also holds the decode step (one token for each of 64
sequences, 16 q/k heads, 32 value heads, fp32 states updated in place) and the
long context with weak decay (g = -softplus(N(-7,1))), where the split takes
its entry states from the affine scan, against GDN_FLAG_SPLIT_OFF.
``cpu_baseline`` times the float64 oracle on a bounded sample of the headline
workload on the host cores.

``--impl reference`` times the oracle (there is no other implementation of this
layer to run here) on a bounded sample per step and prints the same line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN chunked-prefill fwd/bwd tokens/s and TFLOP/s vs BF16 roofline, 1×B200"
CHUNK = 64
HEADLINE = 3  # index of the 65,536-token slow-decay forward in inputs.WORKLOADS
HEADLINE_DESC = "gdn_fwd bf16 B=1 T=65536 H=16 dk=dv=128 C=64 g=-softplus(N(-2,1)) S0=0 (one call)"
ORACLE_SAMPLE_T = 8192  # tokens per head in one bounded oracle sample


def flops_per_token_head(dk, dv, C=CHUNK, backward=False):
    """(dense MMA-tile FLOPs, triangular-aware FLOPs) per token and value head."""
    if backward:
        dense = 16 * dk * dv + 14 * 2 * C * dk + 4 * C * C
        return dense, dense * 385000 / 507904
    dense = 6 * dk * dv + 2 * C * (3 * dk + 2 * dv)
    tri = 6 * dk * dv + C * (3 * dk + 2 * dv) + C * C / 3
    return dense, tri


def fwd_bytes(T_total, Hk, Hv, dk, dv, N, elt=2, s0=True, st=True):
    """Algorithmic HBM bytes of one forward: read q, k, v, beta, g (and S0); write o (and S_T)."""
    states = (int(s0) + int(st)) * N * Hv * dk * dv * 4
    return T_total * (elt * (Hk * 2 * dk + Hv * 2 * dv) + Hv * 8) + states


def bwd_bytes(T_total, Hk, Hv, dk, dv, N, elt=2):
    """Read q, k, v, do, beta, g; write dq, dk, dv, dbeta, dg (+ dS_T read, dS0 write)."""
    return T_total * (elt * (Hk * 4 * dk + Hv * 3 * dv) + Hv * 16) + 2 * N * Hv * dk * dv * 4


def roofline(flops_dense, byts, seconds, hbm_gbs, bf16_tflops, src):
    """t_roof = max(FLOPs / tensor peak, bytes / HBM peak); frac = t_roof / measured time.  The
    bound is whichever term is larger; both fractions are reported."""
    t_hbm = byts / (hbm_gbs * 1e9)
    t_tc = flops_dense / (bf16_tflops * 1e12)
    bound = "tensor" if t_tc >= t_hbm else "hbm"
    achieved_gbs = byts / seconds / 1e9
    achieved_tf = flops_dense / seconds / 1e12
    if bound == "hbm":
        ach, peak, unit = achieved_gbs, hbm_gbs, "GB/s"
    else:
        ach, peak, unit = achieved_tf, bf16_tflops, "TFLOP/s"
    return {"bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
            "t_roof_us": max(t_hbm, t_tc) * 1e6, "frac_hbm": achieved_gbs / hbm_gbs,
            "frac_tensor": achieved_tf / bf16_tflops, "achieved_gbs": achieved_gbs,
            "achieved_tflops_dense": achieved_tf, "peak_gbs": hbm_gbs, "peak_tflops": bf16_tflops,
            "peak_source": src, "algorithmic_bytes": byts, "flops_dense": flops_dense}


FWD_SOURCES = ("gdn_tc_wy.cu", "gdn_tc_fwd.cu", "gdn_tc_common.cuh", "gdn_sm100.cuh",
               "gdn_internal.cuh")


def strip_comments(src: str) -> str:
    """C / C++ source without comments and with runs of whitespace collapsed, so that a
    fingerprint changes with the code, not with its comments (string literals in these files
    hold no comment markers)."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def source_sha16(files=FWD_SOURCES):
    """Fingerprint of the tensor-core forward's code, comments ignored (matches
    profiles/traffic.json)."""
    import hashlib

    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "gated_deltanet_chunked_fwd_b200", "csrc", f)) as fh:
            h.update(strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def traffic_per_call(workload):
    """DRAM bytes (read + write) of one forward call (the WY kernel and the fused kernel) of
    ``workload`` from the committed ncu capture, or None when the code changed since."""
    tp = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(tp):
        return None
    with open(tp) as f:
        rec = json.load(f).get(workload, {})
    return rec.get("bytes_per_call") if rec.get("source_sha16") == source_sha16() else None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


class Clocks:
    """nvidia-smi sampling (every 200 ms) around the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            self.proc.wait(timeout=10)

    def summary(self):
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def dist_setup(n_gpus, backend=None):
    """One process per GPU (torchrun environment); NCCL on GPUs, gloo when there is none."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        timeout = datetime.timedelta(seconds=120)
        if backend == "nccl":
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=timeout,
                                                 device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group(backend, timeout=timeout)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """The largest per-rank value (a step time): the job is as slow as its slowest rank."""
    if world <= 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, ms):
    """Whole-job units per second: every rank runs its own replica on its own batch (weak
    scaling, no collective on the data path), and the step takes ``ms``, the max over ranks."""
    return units_per_rank * world / (ms * 1e-3)


# ----------------------------------------------------------------- oracle arm
def oracle_sample(inp, nheads, units_total):
    """Run the oracle on the first ``nheads`` value heads of a fixed-length workload
    in one call (OpenMP over the heads) and return (seconds, tokens/s scaled to
    the full workload: tokens x nheads / units_total per second, nheads)."""
    import oracle

    x = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    grp = x["v"].shape[2] // x["q"].shape[2]
    hk1 = (nheads + grp - 1) // grp
    nheads = hk1 * grp
    S0 = None if x.get("initial_state") is None else x["initial_state"][:, :nheads]
    t0 = time.perf_counter()
    oracle.fwd(x["q"][:, :, :hk1], x["k"][:, :, :hk1], x["v"][:, :, :nheads],
               x["beta"][:, :, :nheads], x["g"][:, :, :nheads], initial_state=S0)
    dt = time.perf_counter() - t0
    tokens = x["q"].shape[0] * x["q"].shape[1] * nheads / units_total
    return dt, tokens / dt, nheads


def oracle_sample_inputs():
    """The headline workload's shapes and distributions, cut to ORACLE_SAMPLE_T tokens per head."""
    from gated_deltanet_chunked_fwd_b200.inputs import make_workload

    return make_workload(HEADLINE, seed=0, T=ORACLE_SAMPLE_T)


def sample_desc(nh, Hv, reps, seconds):
    return (f"{reps} passes over {nh} of {Hv} value heads x the first {ORACLE_SAMPLE_T} tokens of "
            f"the headline workload's distribution (float64 token loop), {seconds:.1f} s; "
            f"tokens/s scaled by {nh}/{Hv} heads")


def run_reference(args, world, rank):
    if rank != 0:
        return
    import oracle

    inp = oracle_sample_inputs()
    Hv = inp["v"].shape[2]
    nheads = min(Hv, oracle.num_threads())  # bounded sample: one head per host thread
    for _ in range(args.warmup):
        oracle_sample(inp, 1, Hv)
    times = []
    for _ in range(args.steps):
        dt, _, nheads = oracle_sample(inp, nheads, Hv)
        times.append(dt)
    tok_per_step = ORACLE_SAMPLE_T * nheads / Hv
    value = tok_per_step * len(times) / sum(times)
    cores = min(nheads, oracle.num_threads())
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": HEADLINE_DESC, "global_batch": 1, "seq_len": 65536,
                   "parallelism": "none (host oracle)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample_desc(nheads, Hv, len(times), sum(times))},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- our arm
def time_steps(fn, steps, flush, stream):
    """Per-step device time (ms) with CUDA events on ``stream``; L2 flushed before each step."""
    ms = []
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        ms.append(a.elapsed_time(b))
    return ms


class FwdCall:
    """One gdn_chunk_fwd call through the C ABI on fixed device buffers (struct filled once)."""

    def __init__(self, inp, dev, stream, S0=None, ST=None, flags=0):
        import ctypes

        import gated_deltanet_chunked_fwd_b200 as gdn
        from gated_deltanet_chunked_fwd_b200 import _abi

        self.gdn, self.ctypes, self.L = gdn, ctypes, _abi.lib()
        q, k, v = inp["q"], inp["k"], inp["v"]
        self.inp = inp
        B, T, Hk, dk = q.shape
        Hv, dv = v.shape[2], v.shape[3]
        cu = inp.get("cu_seqlens")
        self.N = B if cu is None else cu.numel() - 1
        self.shape = dict(T_total=B * T, Hk=Hk, Hv=Hv, dk=dk, dv=dv, N=self.N)
        self.o = torch.empty(B, T, Hv, dv, dtype=q.dtype, device=dev)
        self.ST = ST if ST is not None else torch.empty(self.N, Hv, dk, dv, dtype=torch.float32,
                                                        device=dev)
        self.S0 = S0 if S0 is not None else inp.get("initial_state")
        a = _abi.GdnFwdArgs()
        self.host = gdn._fill_common(a, q, k, v, inp["beta"], inp["g"], cu, inp.get("cu_seqlens_host"),
                                     self.S0, flags)[1]
        a.o, a.ST = self.o.data_ptr(), self.ST.data_ptr()
        self.a = a
        n = ctypes.c_size_t(0)
        st = self.L.gdn_chunk_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n))
        if st != 0:
            raise gdn.GdnError("gdn_chunk_fwd_workspace_size", st)
        self.ws_n = n.value
        self.ws = torch.empty(max(n.value, 1), dtype=torch.uint8, device=dev)
        self.launches = self.L.gdn_chunk_fwd_launch_count(ctypes.byref(a))
        self.sp = ctypes.c_void_p(stream.cuda_stream)

    def __call__(self):
        st = self.L.gdn_chunk_fwd(self.ctypes.byref(self.a), self.ctypes.c_void_p(self.ws.data_ptr()),
                                  self.ws_n, self.sp)
        if st != 0:
            raise self.gdn.GdnError("gdn_chunk_fwd", st)

    def bytes(self):
        s = self.shape
        return fwd_bytes(s["T_total"], s["Hk"], s["Hv"], s["dk"], s["dv"], s["N"],
                         s0=self.S0 is not None, st=True)


DECODE = dict(N=64, Hk=16, Hv=32, dk=128, dv=128)


def decode_bytes(N, Hk, Hv, dk, dv, elt=2):
    """Algorithmic HBM bytes of one decode step: read and write every fp32 state; read q, k, v,
    beta, g; write o."""
    return N * (Hv * (2 * dk * dv * 4 + 2 * dv * elt + 8) + 2 * Hk * dk * elt)


def decode_bench(dev, stream, rank, measure, world, hbm, bf16, src, steps):
    """One decode token for each of 64 sequences (16 q/k heads, 32 value heads, d = 128, bf16
    tokens, fp32 states updated in place) through the C ABI."""
    import ctypes

    import gated_deltanet_chunked_fwd_b200 as gdn
    from gated_deltanet_chunked_fwd_b200 import _abi
    from gated_deltanet_chunked_fwd_b200.inputs import make_inputs

    d = DECODE
    x = make_inputs(d["N"], 1, d["Hk"], d["Hv"], d["dk"], d["dv"], dtype="bf16", seed=rank,
                    s0_std=0.1, device=dev)
    c0 = {n: x[n][:, 0].contiguous() for n in ("q", "k", "v", "beta", "g")}
    S = x["initial_state"]
    o = torch.empty(c0["v"].shape, dtype=torch.bfloat16, device=dev)
    a = gdn._decode_args(c0["q"], c0["k"], c0["v"], c0["beta"], c0["g"], S, None, o)
    L = _abi.lib()
    sp = ctypes.c_void_p(stream.cuda_stream)

    def step():
        st = L.gdn_decode_step(ctypes.byref(a), sp)
        if st != 0:
            raise gdn.GdnError("gdn_decode_step", st)

    m = measure(step, steps)
    byts = decode_bytes(**d)
    flops = d["N"] * d["Hv"] * 8 * d["dk"] * d["dv"]  # two dots and the rank-1 update per state
    return {"ms": m, "tokens_per_s": job_throughput(d["N"], world, m), "launches": 1,
            "roofline": roofline(flops, byts, m * 1e-3, hbm, bf16, src)}


def e2e_leg(inp, dev, stream, measure, steps, tokens, world):
    """The headline call with pinned host inputs: the H2D copies of q, k, v, beta, g, the call
    through the C ABI, and the D2H copies of o and S_T, all inside the timed region."""
    names = [n for n in ("q", "k", "v", "beta", "g") if inp.get(n) is not None]
    host = {n: inp[n].cpu().pin_memory() for n in names}
    dbuf = {n: torch.empty_like(t, device=dev) for n, t in host.items()}
    ecall = FwdCall(dict(dbuf), dev, stream)
    o_h = torch.empty(ecall.o.shape, dtype=ecall.o.dtype).pin_memory()
    ST_h = torch.empty(ecall.ST.shape, dtype=ecall.ST.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_h.numel() * o_h.element_size() + ST_h.numel() * ST_h.element_size()

    def e2e_step():
        for n_, t in host.items():
            dbuf[n_].copy_(t, non_blocking=True)
        ecall()
        o_h.copy_(ecall.o, non_blocking=True)
        ST_h.copy_(ecall.ST, non_blocking=True)

    ms_e2e = measure(e2e_step, max(2, min(steps, 5)))
    return {"value": job_throughput(tokens, world, ms_e2e), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms": ms_e2e}


def run_ours(args, world, rank, local):
    import gated_deltanet_chunked_fwd_b200 as gdn
    from gated_deltanet_chunked_fwd_b200 import GDN_FLAG_GATE_LOGITS, GDN_FLAG_QK_L2NORM, GDN_FLAG_SPLIT_OFF
    from gated_deltanet_chunked_fwd_b200.inputs import WORKLOADS, make_workload

    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    hbm, bf16, src = measured_peaks()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    scratch = torch.empty(2 * l2 // 4 + 1024, dtype=torch.float32, device=dev)

    def flush():
        scratch.fill_(1.0)

    def measure(fn, steps, warm=3):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        ms = time_steps(fn, steps, flush, stream)
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(sum(ms) / len(ms), world)

    if args.decode_only:
        # the decode workload by itself, so that a profiler sees its launches alone
        r = decode_bench(dev, stream, rank, measure, world, hbm, bf16, src, args.steps)
        if rank == 0:
            print(json.dumps({"workload": "decode_bf16_N64_Hk16_Hv32_d128", **r}), flush=True)
        return

    # ---- headline: one 65,536-token call (fewer with --tokens, to profile a small case)
    inp = make_workload(HEADLINE, seed=rank, device=dev, **({"T": args.tokens} if args.tokens else {}))
    call = FwdCall(inp, dev, stream)
    Hv, dk, dv = call.shape["Hv"], call.shape["dk"], call.shape["dv"]
    tokens = call.shape["T_total"]
    for _ in range(max(args.warmup, 3)):
        call()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with Clocks(local) as clk:
        ms = time_steps(call, args.steps, flush, stream)
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ms_step = max_over_ranks(sum(ms) / len(ms), world)
    value = job_throughput(tokens, world, ms_step)
    dense, tri = flops_per_token_head(dk, dv)
    byts = call.bytes()
    roof = roofline(dense * tokens * Hv, byts, ms_step * 1e-3, hbm, bf16, src)
    roof["traffic"] = traffic_per_call(WORKLOADS[HEADLINE].name) if call.launches == 2 else None
    roof["kernel"] = "whole forward call: gdn_wy_tc_kernel + gdn_fwd_tc_kernel"
    tflops = {"dense": dense * tokens * Hv / (ms_step * 1e-3) / 1e12,
              "triangular": tri * tokens * Hv / (ms_step * 1e-3) / 1e12, "peak_bf16": bf16}

    # ---- e2e: pinned host inputs, H2D + call + D2H of o and S_T, inside the timed region
    e2e = None if args.no_e2e else e2e_leg(inp, dev, stream, measure, args.steps, tokens, world)

    # ---- the other forward workloads (extra keys)
    extra = {}
    if not args.no_extra:
        for idx in (1, 2):
            w = WORKLOADS[idx]
            c = FwdCall(make_workload(idx, seed=rank, device=dev), dev, stream)
            m = measure(c, args.steps)
            t_ = c.shape["T_total"]
            extra[w.name] = {
                "ms": m, "tokens_per_s": job_throughput(t_, world, m), "tokens": t_,
                "launches": c.launches,
                "roofline": dict(roofline(dense * t_ * c.shape["Hv"], c.bytes(), m * 1e-3, hbm, bf16, src),
                                 traffic=traffic_per_call(w.name) if c.launches == 2 else None)}
            del c
        # the headline's tokens fed as 4 chained 16,384-token calls (S_T -> S0)
        parts = []
        prev = None
        for i in range(4):
            sl = slice(i * 16384, (i + 1) * 16384)
            sub = {n: inp[n][:, sl].contiguous() for n in ("q", "k", "v", "beta", "g")}
            c = FwdCall(sub, dev, stream, S0=prev)
            prev = c.ST
            parts.append(c)

        def chained():
            for c in parts:
                c()

        m = measure(chained, args.steps)
        cb = sum(c.bytes() for c in parts)
        extra["fwd_bf16_T65536_H16_d128_slowdecay_4x16384_chained"] = {
            "ms": m, "tokens_per_s": job_throughput(tokens, world, m), "tokens": tokens,
            "launches": sum(c.launches for c in parts),
            "roofline": roofline(dense * tokens * Hv, cb, m * 1e-3, hbm, bf16, src)}
        del parts
        extra["decode_bf16_N64_Hk16_Hv32_d128"] = decode_bench(dev, stream, rank, measure, world,
                                                               hbm, bf16, src, args.steps)
        # the long context with weak decay (g = -softplus(N(-7,1))): no warm-up reaches 2^-30, so
        # later segments take their entry state from the affine scan; against one chain per head
        wk = make_workload(HEADLINE, seed=rank, device=dev, g_mu=-7.0)
        for label, flags in (("split_auto_scan", 0), ("split_off", GDN_FLAG_SPLIT_OFF)):
            c = FwdCall(wk, dev, stream, flags=flags)
            m = measure(c, max(2, min(args.steps, 5)))
            extra[f"fwd_bf16_T65536_H16_d128_weakdecay_{label}"] = {
                "ms": m, "tokens_per_s": job_throughput(tokens, world, m), "tokens": tokens,
                "launches": c.launches,
                "roofline": roofline(dense * tokens * Hv, c.bytes(), m * 1e-3, hbm, bf16, src)}
            del c
        del wk
        # the headline fed raw inputs: q, k rows at random scales and beta, g as logits /
        # pre-activations, normalised and mapped inside (GDN_FLAG_QK_L2NORM | GDN_FLAG_GATE_LOGITS);
        # the logits are drawn so that the mapped beta and g follow the headline's distributions
        # (beta = sigmoid(N(0,1)), g = -softplus(N(g_mu,1)))
        wr = make_workload(HEADLINE, seed=rank, device=dev)
        gen = torch.Generator().manual_seed(rank)
        for name in ("q", "k"):
            x = wr[name].float().cpu()
            wr[name] = (x * (0.3 + 2.7 * torch.rand(x.shape[:-1] + (1,), generator=gen))).to(
                wr[name].dtype).to(dev)
        wr["beta"] = torch.randn(wr["beta"].shape, generator=gen).to(dev)
        wr["g"] = (torch.randn(wr["g"].shape, generator=gen) + WORKLOADS[HEADLINE].g_mu).to(dev)
        c = FwdCall(wr, dev, stream, flags=GDN_FLAG_QK_L2NORM | GDN_FLAG_GATE_LOGITS)
        m = measure(c, max(2, min(args.steps, 5)))
        extra["fwd_bf16_T65536_H16_d128_raw_inputs_fused_preprocessing"] = {
            "ms": m, "tokens_per_s": job_throughput(tokens, world, m), "tokens": tokens,
            "launches": c.launches,
            "roofline": roofline(dense * tokens * Hv, c.bytes(), m * 1e-3, hbm, bf16, src)}
        del c, wr

    # ---- backward on its own workload
    bwd = None
    if not args.no_bwd:
        bi = make_workload(4, seed=rank, device=dev, B=args.bwd_batch)
        qs = [bi[n] for n in ("q", "k", "v", "beta", "g", "do")]
        wsb = torch.empty(max(gdn.gdn_chunk_bwd_workspace_size(*qs[:5]), 1), dtype=torch.uint8,
                          device=dev)

        def bstep():
            gdn.gdn_chunk_bwd(*qs, dST=bi["dST"], workspace=wsb)

        bms = measure(bstep, max(1, min(args.steps, 5)), warm=1)
        bt = bi["q"].shape[0] * bi["q"].shape[1]
        bd, btri = flops_per_token_head(dk, dv, backward=True)
        bb = bwd_bytes(bt, bi["q"].shape[2], Hv, dk, dv, bi["q"].shape[0])
        bwd = {"workload": f"gdn_bwd bf16 B={args.bwd_batch} T=8192 H=16 dk=dv=128 C=64",
               "tokens_per_s": job_throughput(bt, world, bms),
               "ms": bms, "tflops_dense": bd * bt * Hv / (bms * 1e-3) / 1e12,
               "tflops_tri": btri * bt * Hv / (bms * 1e-3) / 1e12,
               "hbm_gbs": bb / (bms * 1e-3) / 1e9,
               "roofline": roofline(bd * bt * Hv, bb, bms * 1e-3, hbm, bf16, src),
               "path": "WY kernel + fused kernel (state replay) + reverse kernel"
                       + (" + dq/dk group reduction" if bi["v"].shape[2] != bi["q"].shape[2] else ""),
               "launches": gdn.launch_count(*qs[:5], backward=True)}
        del bi, qs, wsb
        if not args.no_extra:
            # the long context with weak decay (g = -softplus(N(-7,1))): reverse warm-ups would be
            # ~200 chunks long or fail, so segments take their exit adjoint from the adjoint scan;
            # against one reverse walk per head
            wb = make_workload(4, seed=rank, device=dev, B=1, T=65536, g_mu=-7.0)
            qs = [wb[n] for n in ("q", "k", "v", "beta", "g", "do")]
            wsb = torch.empty(max(gdn.gdn_chunk_bwd_workspace_size(*qs[:5]), 1), dtype=torch.uint8,
                              device=dev)
            wt = wb["q"].shape[1]
            for label, flags in (("split_auto_scan", 0), ("split_off", GDN_FLAG_SPLIT_OFF)):
                def wstep(flags=flags):
                    gdn.gdn_chunk_bwd(*qs, dST=wb["dST"], workspace=wsb, flags=flags)

                wms = measure(wstep, max(1, min(args.steps, 3)), warm=1)
                bwd[f"bwd_bf16_T65536_H16_d128_weakdecay_{label}"] = {
                    "ms": wms, "tokens_per_s": job_throughput(wt, world, wms),
                    "launches": gdn.launch_count(*qs[:5], backward=True, flags=flags),
                    "roofline": roofline(bd * wt * Hv, bwd_bytes(wt, wb["q"].shape[2], Hv, dk, dv, 1),
                                         wms * 1e-3, hbm, bf16, src)}
            del wb, qs, wsb

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu:
        import oracle

        inp_cpu = oracle_sample_inputs()
        nh = min(Hv, oracle.num_threads())
        # repeat the same bounded sample until about 10 s of host time have been measured
        dt_sum, tok_sum, reps = 0.0, 0.0, 0
        while dt_sum < 10.0 and reps < 1000:
            dt, tps, nh = oracle_sample(inp_cpu, nh, Hv)
            dt_sum += dt
            tok_sum += tps * dt
            reps += 1
        cpu_base = {"value": tok_sum / dt_sum, "unit": "tokens/s",
                    "cores": min(nh, oracle.num_threads()), "kind": "oracle",
                    "sample": sample_desc(nh, Hv, reps, dt_sum)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": HEADLINE_DESC if not args.tokens else
                       HEADLINE_DESC.replace("T=65536", f"T={tokens}"),
                       "global_batch": world, "seq_len": tokens, "heads": Hv, "head_dim": dk,
                       "parallelism": f"replicas x{world} (no collective)",
                       "l2": "inputs (1.08 GB) larger than L2; L2 also flushed before every timed "
                             "step (2x L2 write, outside the events)",
                       "path": "tensor-core (WY kernel + fused state chain)" if call.launches <= 2
                       else "cuda-core 4-kernel"},
            "tflops": tflops,
            "roofline": roof,
            "e2e": e2e,
            "gpu_launches": call.launches * args.steps,
            "clocks": clk.summary(),
            "cpu_baseline": cpu_base,
            "fwd_workloads": extra,
            "bwd": bwd,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-bwd", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="headline forward only")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-copy leg (profiling)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="headline shape with this many tokens (profiling a small case; 0 = 65,536)")
    ap.add_argument("--bwd-batch", type=int, default=4,
                    help="sequences in the backward workload (4 = the backward workload; fewer for a small profile)")
    ap.add_argument("--decode-only", action="store_true",
                    help="time the decode workload by itself and print its line (profiling)")
    args = ap.parse_args()
    if args.impl == "reference":
        # the oracle arm runs on rank 0's host cores only; no process group
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        args.gpus = world
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
