"""libgdn.so on the host, without a GPU: the library loads, exports every entry
point that include/gdn.h declares, and rejects bad arguments before it touches
CUDA (every case below returns from host-side checks; no kernel is launched)."""
import ctypes
import os
import re

import pytest

from gated_deltanet_chunked_fwd_b200 import _abi
from gated_deltanet_chunked_fwd_b200._abi import GdnBwdArgs, GdnFwdArgs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
FAKE = 1 << 20  # a 256-byte aligned fake device address; never dereferenced here


def header_functions():
    src = open(os.path.join(ROOT, "include", "gdn.h")).read()
    return re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", src)


def test_library_exports_every_declared_function():
    L = _abi.lib()
    declared = header_functions()
    assert set(_abi.EXPORTS) <= set(declared)
    for fn in declared:
        assert hasattr(L, fn), fn


def test_python_short_names():
    import gated_deltanet_chunked_fwd_b200 as gdn

    assert gdn.chunk_fwd is gdn.gdn_chunk_fwd and gdn.chunk_bwd is gdn.gdn_chunk_bwd
    assert {"chunk_fwd", "chunk_bwd", "gdn_chunk_fwd", "gdn_chunk_bwd"} <= set(gdn.__all__)


def test_status_strings():
    L = _abi.lib()
    for code in range(7):
        assert L.gdn_status_string(code)
    assert L.gdn_status_string(99) == b"unknown status"


def fwd_args(**kw):
    a = GdnFwdArgs()
    a.struct_size = ctypes.sizeof(a)
    a.abi_version = 1
    a.dtype = _abi.GDN_BF16
    a.B, a.T, a.Hk, a.Hv, a.dk, a.dv = 1, 256, 2, 4, 128, 128
    a.q = a.k = a.v = a.o = FAKE
    a.beta = a.g = FAKE
    for k_, v_ in kw.items():
        setattr(a, k_, v_)
    return a


def ws_size(a):
    n = ctypes.c_size_t(0)
    st = _abi.lib().gdn_chunk_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n))
    return st, n.value


def call_fwd(a, ws=FAKE, ws_bytes=1 << 40):
    return _abi.lib().gdn_chunk_fwd(ctypes.byref(a), ctypes.c_void_p(ws), ws_bytes, None)


@pytest.mark.parametrize("field,value,expect", [
    ("abi_version", 2, INVALID), ("struct_size", 8, INVALID), ("dtype", 7, UNSUPPORTED),
    ("Hv", 3, INVALID), ("Hk", 0, INVALID), ("dk", 0, UNSUPPORTED), ("dv", 256, UNSUPPORTED),
    ("B", 0, INVALID), ("T", -1, INVALID),
])
def test_bad_scalars_are_rejected(field, value, expect):
    a = fwd_args(**{field: value})
    assert ws_size(a)[0] == expect
    assert call_fwd(a) == expect


@pytest.mark.parametrize("field", ["q", "k", "v", "o", "beta", "g"])
def test_missing_tensor_is_rejected(field):
    assert call_fwd(fwd_args(**{field: None})) == INVALID


@pytest.mark.parametrize("field,offset", [("q", 2), ("v", 8), ("o", 4), ("beta", 2), ("S0", 4)])
def test_misaligned_tensor_is_rejected(field, offset):
    assert call_fwd(fwd_args(**{field: FAKE + offset})) == INVALID


def test_workspace_checks():
    # the tensor-core path (bf16, 128 x 128) keeps three 8 KB images (T, T diag(beta Gam),
    # T diag(beta)) and one 8-byte gate summary per (image slot, value head),
    # slots = T_total // 64 + N + 1; the portable path keeps fp32 W, U, gamma and states
    st, need_tc = ws_size(fwd_args())
    slots = 256 // 64 + 1 + 1
    assert st == OK and need_tc == -(-(slots * 4 * 3 * 8192 + slots * 4 * 8) // 256) * 256
    assert call_fwd(fwd_args(), ws=0) == WORKSPACE
    a = fwd_args(flags=_abi.GDN_FLAG_PORTABLE)
    st, need = ws_size(a)
    assert st == OK and need > 0 and need % 256 == 0
    assert call_fwd(a, ws=0) == WORKSPACE
    assert call_fwd(a, ws=FAKE, ws_bytes=need - 1) == WORKSPACE
    assert call_fwd(a, ws=FAKE + 16, ws_bytes=need) == WORKSPACE


def test_varlen_host_offsets_are_checked():
    good = (ctypes.c_int32 * 4)(0, 100, 100, 300)
    a = fwd_args(T=300, num_seqs=3, cu_seqlens=FAKE, cu_seqlens_host=ctypes.addressof(good))
    assert ws_size(a)[0] == OK
    bad = (ctypes.c_int32 * 4)(0, 100, 50, 300)  # not monotone
    assert ws_size(fwd_args(T=300, num_seqs=3, cu_seqlens=FAKE,
                            cu_seqlens_host=ctypes.addressof(bad)))[0] == INVALID
    assert ws_size(fwd_args(T=299, num_seqs=3, cu_seqlens=FAKE,
                            cu_seqlens_host=ctypes.addressof(good)))[0] == INVALID  # total != T
    assert ws_size(fwd_args(T=300, num_seqs=3, cu_seqlens=FAKE))[0] == INVALID  # no host copy
    assert ws_size(fwd_args(B=2, T=300, num_seqs=3, cu_seqlens=FAKE,
                            cu_seqlens_host=ctypes.addressof(good)))[0] == INVALID  # B != 1


def test_workspace_grows_with_tokens_and_launch_count():
    L = _abi.lib()
    s1 = ws_size(fwd_args(T=256, flags=_abi.GDN_FLAG_PORTABLE))[1]
    s2 = ws_size(fwd_args(T=1024, flags=_abi.GDN_FLAG_PORTABLE))[1]
    assert s2 > s1
    assert L.gdn_chunk_fwd_launch_count(ctypes.byref(fwd_args())) >= 1
    assert L.gdn_chunk_fwd_launch_count(ctypes.byref(fwd_args(Hv=3))) == -1


def test_backward_argument_checks():
    L = _abi.lib()
    a = GdnBwdArgs()
    a.struct_size = ctypes.sizeof(a)
    a.abi_version = 1
    a.dtype = _abi.GDN_F32
    a.B, a.T, a.Hk, a.Hv, a.dk, a.dv = 2, 100, 1, 2, 64, 64
    for f in ("q", "k", "v", "beta", "g", "dout", "dq", "dk_out", "dv_out", "dbeta", "dg"):
        setattr(a, f, FAKE)
    n = ctypes.c_size_t(0)
    assert L.gdn_chunk_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == OK and n.value > 0
    assert L.gdn_chunk_bwd(ctypes.byref(a), ctypes.c_void_p(0), 0, None) == WORKSPACE
    a.dout = None
    assert L.gdn_chunk_bwd(ctypes.byref(a), ctypes.c_void_p(FAKE), n.value, None) == INVALID


def test_aliased_states_are_rejected():
    """S0 and S_T sharing bytes (the same buffer, or overlapping ranges) are rejected before any
    launch: a later segment of a split sequence may read S0 after S_T was written."""
    state = 4 * 128 * 128 * 4  # N * Hv * dk * dv fp32 of fwd_args()
    for st_addr in (FAKE, FAKE + 256, FAKE + state - 256):
        assert call_fwd(fwd_args(S0=FAKE, ST=st_addr)) == INVALID
    a = GdnBwdArgs()
    a.struct_size = ctypes.sizeof(a)
    a.abi_version = 1
    a.dtype = _abi.GDN_BF16
    a.B, a.T, a.Hk, a.Hv, a.dk, a.dv = 1, 256, 2, 4, 128, 128
    for f in ("q", "k", "v", "beta", "g", "dout", "dq", "dk_out", "dv_out", "dbeta", "dg"):
        setattr(a, f, FAKE)
    L = _abi.lib()
    for s0, dst in ((FAKE, FAKE + state), (FAKE + state, FAKE)):
        a.S0, a.dST, a.dS0 = s0, dst, FAKE + 256
        assert L.gdn_chunk_bwd(ctypes.byref(a), ctypes.c_void_p(FAKE), 1 << 40, None) == INVALID


def test_noalloc_checks_the_struct_before_reading_it():
    """A caller built against a smaller (older) argument struct is rejected from its size field
    alone, before the library copies the struct."""
    L = _abi.lib()
    short = (ctypes.c_uint32 * 2)(8, 1)  # struct_size = 8 bytes, abi_version = 1
    assert L.gdn_chunk_fwd_noalloc(ctypes.cast(short, ctypes.POINTER(GdnFwdArgs)), None) == INVALID
    wrong_abi = fwd_args(abi_version=2)
    assert L.gdn_chunk_fwd_noalloc(ctypes.byref(wrong_abi), None) == INVALID
    assert L.gdn_chunk_fwd_noalloc(None, None) == INVALID


def test_decode_argument_checks():
    """gdn_decode_step rejects bad arguments on the host; N = 0 is a no-op."""
    L = _abi.lib()

    def dargs(**kw):
        a = _abi.GdnDecodeArgs()
        a.struct_size = ctypes.sizeof(a)
        a.abi_version = 1
        a.dtype = _abi.GDN_BF16
        a.N, a.Hk, a.Hv, a.dk, a.dv = 4, 2, 4, 128, 128
        a.q = a.k = a.v = a.o = a.S = FAKE
        a.beta = a.g = FAKE
        for k_, v_ in kw.items():
            setattr(a, k_, v_)
        return a

    call = lambda a: L.gdn_decode_step(ctypes.byref(a), None)
    assert call(dargs(struct_size=8)) == INVALID
    assert call(dargs(abi_version=3)) == INVALID
    assert call(dargs(dtype=5)) == UNSUPPORTED
    assert call(dargs(Hv=3)) == INVALID
    assert call(dargs(dv=130)) == UNSUPPORTED
    assert call(dargs(dv=30)) == UNSUPPORTED  # dv must be a multiple of 4
    assert call(dargs(S=FAKE + 8)) == INVALID  # 16-byte aligned state
    assert call(dargs(q=None)) == INVALID
    assert call(dargs(state_indices=FAKE, num_slots=0)) == INVALID
    assert call(dargs(N=0)) == OK


def test_preprocessing_flags_reach_the_plan():
    """GDN_FLAG_QK_L2NORM routes the tensor-core backward's dq / dk through the fp32 per-head
    buffers and the reduction kernel even without grouped heads: one more launch and a larger
    workspace; GDN_FLAG_GATE_LOGITS changes neither (the maps run inside the existing kernels)."""
    L = _abi.lib()

    def bwd(flags, Hv=2):
        a = GdnBwdArgs()
        a.struct_size = ctypes.sizeof(a)
        a.abi_version = 1
        a.dtype = _abi.GDN_BF16
        a.B, a.T, a.Hk, a.Hv, a.dk, a.dv = 1, 512, 2, Hv, 128, 128
        a.flags = flags
        for f in ("q", "k", "v", "beta", "g", "dout", "dq", "dk_out", "dv_out", "dbeta", "dg"):
            setattr(a, f, FAKE)
        n = ctypes.c_size_t(0)
        assert L.gdn_chunk_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == OK
        return L.gdn_chunk_bwd_launch_count(ctypes.byref(a)), n.value

    plain, gates, norm = bwd(0), bwd(_abi.GDN_FLAG_GATE_LOGITS), bwd(_abi.GDN_FLAG_QK_L2NORM)
    assert gates == plain
    assert norm[0] == plain[0] + 1 and norm[1] > plain[1]
    # with grouped heads the reduction runs anyway
    assert bwd(_abi.GDN_FLAG_QK_L2NORM, Hv=4)[0] == bwd(0, Hv=4)[0]
    # the forward keeps its two launches with either flag
    for f in (_abi.GDN_FLAG_GATE_LOGITS, _abi.GDN_FLAG_QK_L2NORM):
        assert L.gdn_chunk_fwd_launch_count(ctypes.byref(fwd_args(flags=f))) == \
            L.gdn_chunk_fwd_launch_count(ctypes.byref(fwd_args()))
