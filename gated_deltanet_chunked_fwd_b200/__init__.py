"""GDN chunked prefill (forward and backward) on NVIDIA B200 -- Python binding.

``gdn_chunk_fwd`` / ``gdn_chunk_bwd`` / ``gdn_decode_step`` mirror the C entry
points of ``include/gdn.h`` one to one.  This module marshals torch tensors into the C
argument structs, allocates the outputs and the workspace with torch (device
memory) and passes torch's current CUDA stream.  All arithmetic runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback.

The layer is the gated delta rule of the Gated Delta Network (the GDN layer of
the FlashQLA pages, news.hamidun.com "What is FlashQLA"):
    S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t,
states stored transposed (H = S^T, [dk, dv]).
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _abi
from ._abi import (GDN_FLAG_GATE_LOGITS, GDN_FLAG_PORTABLE, GDN_FLAG_QK_L2NORM, GDN_FLAG_SPLIT_FORCE,
                   GDN_FLAG_SPLIT_OFF, GdnBwdArgs, GdnCombineArgs, GdnDecodeArgs, GdnError, GdnFwdArgs,
                   GdnHaloArgs)

__all__ = ["gdn_chunk_fwd", "gdn_chunk_bwd", "gdn_decode_step", "gdn_chunk_fwd_workspace_size",
           "gdn_chunk_bwd_workspace_size", "chunk_fwd", "chunk_bwd", "GdnError",
           "GDN_FLAG_SPLIT_OFF", "GDN_FLAG_SPLIT_FORCE", "GDN_FLAG_PORTABLE", "GDN_FLAG_GATE_LOGITS",
           "GDN_FLAG_QK_L2NORM",
           "decode_step", "gdn_affine_combine", "gdn_halo_check"]

_DT = {torch.float32: _abi.GDN_F32, torch.bfloat16: _abi.GDN_BF16}


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libgdn must be contiguous")
    return t.data_ptr()


def _fill_common(a, q, k, v, beta, g, cu_seqlens, cu_seqlens_host, initial_state, flags):
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4:
        raise ValueError("q, k must be [B, T, Hk, dk] and v [B, T, Hv, dv]")
    if q.dtype not in _DT or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share one dtype: float32 or bfloat16")
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    if beta.dtype != torch.float32 or g.dtype != torch.float32:
        raise ValueError("beta and g must be float32")
    a.struct_size = ctypes.sizeof(a)
    a.abi_version = _abi.GDN_ABI_VERSION
    a.dtype = _DT[q.dtype]
    a.B, a.T, a.Hk, a.Hv, a.dk, a.dv = B, T, Hk, Hv, dk, dv
    a.flags = flags
    a.q, a.k, a.v, a.beta, a.g = _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g)
    host = None
    N = B
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32:
            raise ValueError("cu_seqlens must be int32")
        host = cu_seqlens_host if cu_seqlens_host is not None else cu_seqlens.cpu()
        host = host.to(torch.int32).contiguous()
        N = host.numel() - 1
        a.num_seqs = N
        a.cu_seqlens = _ptr(cu_seqlens)
        a.cu_seqlens_host = host.data_ptr()
    if initial_state is not None:
        if initial_state.dtype != torch.float32 or tuple(initial_state.shape) != (N, Hv, dk, dv):
            raise ValueError(f"initial_state must be float32 [{N}, {Hv}, {dk}, {dv}]")
        a.S0 = _ptr(initial_state)
    return N, host  # keep `host` alive until the call returns


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(fn, status):
    if status != 0:
        raise GdnError(fn, status)


def _dev_status(device, want):
    return torch.zeros(1, dtype=torch.int32, device=device) if want else None


def _raise_dev_status(fn, st):
    if st is not None:
        code = int(st.item())  # synchronises
        if code != 0:
            raise GdnError(fn + " (device)", code)


def gdn_chunk_fwd_workspace_size(q, k, v, beta, g, cu_seqlens=None, cu_seqlens_host=None,
                                 initial_state=None, flags: int = 0) -> int:
    a = GdnFwdArgs()
    _, host = _fill_common(a, q, k, v, beta, g, cu_seqlens, cu_seqlens_host, initial_state, flags)
    n = ctypes.c_size_t(0)
    _check("gdn_chunk_fwd_workspace_size", _abi.lib().gdn_chunk_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    return n.value


def gdn_chunk_fwd(q, k, v, beta, g, cu_seqlens=None, initial_state=None,
                  output_final_state: bool = True, *, cu_seqlens_host=None, flags: int = 0,
                  out=None, final_state=None, workspace=None, check_device_status: bool = False):
    """Chunked-prefill forward.  Returns (o [B,T,Hv,dv] in q's dtype, S_T [N,Hv,dk,dv] fp32 or None).

    q, k: [B,T,Hk,dk]; v: [B,T,Hv,dv]; beta, g: [B,T,Hv] fp32 (g = raw log decay);
    cu_seqlens: int32 [N+1] on the device for packed variable-length batches
    (B == 1), with ``cu_seqlens_host`` its host copy (else one D2H copy is made);
    initial_state: fp32 [N,Hv,dk,dv] (transposed state H = S^T) or None for zeros.
    Enqueued on torch's current stream; nothing is synchronised unless
    ``check_device_status`` is set.
    """
    a = GdnFwdArgs()
    N, host = _fill_common(a, q, k, v, beta, g, cu_seqlens, cu_seqlens_host, initial_state, flags)
    B, T = q.shape[:2]
    Hv, dk, dv = v.shape[2], q.shape[3], v.shape[3]
    o = out if out is not None else torch.empty(B, T, Hv, dv, dtype=q.dtype, device=q.device)
    ST = None
    if output_final_state:
        ST = final_state if final_state is not None else torch.empty(N, Hv, dk, dv, dtype=torch.float32, device=q.device)
    a.o, a.ST = _ptr(o), _ptr(ST)
    st = _dev_status(q.device, check_device_status)
    a.dev_status = _ptr(st)
    L = _abi.lib()
    n = ctypes.c_size_t(0)
    _check("gdn_chunk_fwd_workspace_size", L.gdn_chunk_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    if workspace is None or workspace.numel() < n.value:
        workspace = torch.empty(max(n.value, 1), dtype=torch.uint8, device=q.device)
    _check("gdn_chunk_fwd", L.gdn_chunk_fwd(ctypes.byref(a), ctypes.c_void_p(workspace.data_ptr()),
                                            n.value, _stream(q.device)))
    _raise_dev_status("gdn_chunk_fwd", st)
    del host
    return o, ST


def gdn_chunk_bwd_workspace_size(q, k, v, beta, g, cu_seqlens=None, cu_seqlens_host=None,
                                 initial_state=None, flags: int = 0) -> int:
    a = GdnBwdArgs()
    _, host = _fill_common(a, q, k, v, beta, g, cu_seqlens, cu_seqlens_host, initial_state, flags)
    n = ctypes.c_size_t(0)
    _check("gdn_chunk_bwd_workspace_size", _abi.lib().gdn_chunk_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    return n.value


def gdn_chunk_bwd(q, k, v, beta, g, do, cu_seqlens=None, initial_state=None, dST=None,
                  output_dS0: bool = True, *, cu_seqlens_host=None, flags: int = 0,
                  workspace=None, check_device_status: bool = False):
    """Chunked-prefill backward.  Returns (dq, dk, dv, dbeta, dg, dS0 or None).

    do: [B,T,Hv,dv] in q's dtype; dST: fp32 [N,Hv,dk,dv] or None (zero).
    dq/dk are summed over the value heads sharing a q/k head; dg is w.r.t. raw g.
    """
    a = GdnBwdArgs()
    N, host = _fill_common(a, q, k, v, beta, g, cu_seqlens, cu_seqlens_host, initial_state, flags)
    if do.shape != v.shape or do.dtype != q.dtype:
        raise ValueError("do must match v's shape and q's dtype")
    dev = q.device
    dq, dk = torch.empty_like(q), torch.empty_like(k)
    dv = torch.empty_like(v)
    dbeta, dg = torch.empty_like(beta), torch.empty_like(g)
    dS0 = torch.empty(N, v.shape[2], q.shape[3], v.shape[3], dtype=torch.float32, device=dev) if output_dS0 else None
    a.dout, a.dST = _ptr(do), _ptr(dST)
    a.dq, a.dk_out, a.dv_out = _ptr(dq), _ptr(dk), _ptr(dv)
    a.dbeta, a.dg, a.dS0 = _ptr(dbeta), _ptr(dg), _ptr(dS0)
    st = _dev_status(dev, check_device_status)
    a.dev_status = _ptr(st)
    L = _abi.lib()
    n = ctypes.c_size_t(0)
    _check("gdn_chunk_bwd_workspace_size", L.gdn_chunk_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    if workspace is None or workspace.numel() < n.value:
        workspace = torch.empty(max(n.value, 1), dtype=torch.uint8, device=dev)
    _check("gdn_chunk_bwd", L.gdn_chunk_bwd(ctypes.byref(a), ctypes.c_void_p(workspace.data_ptr()),
                                            n.value, _stream(dev)))
    _raise_dev_status("gdn_chunk_bwd", st)
    del host
    return dq, dk, dv, dbeta, dg, dS0


def _decode_args(q, k, v, beta, g, state, state_indices, o, flags=0):
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[0] != q.shape[0]:
        raise ValueError("q, k must be [N, Hk, dk] and v [N, Hv, dv]")
    if q.dtype not in _DT or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share one dtype: float32 or bfloat16")
    if beta.dtype != torch.float32 or g.dtype != torch.float32 or state.dtype != torch.float32:
        raise ValueError("beta, g and the state must be float32")
    N, Hk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    a = GdnDecodeArgs()
    a.struct_size = ctypes.sizeof(a)
    a.abi_version = _abi.GDN_ABI_VERSION
    a.dtype = _DT[q.dtype]
    a.N, a.Hk, a.Hv, a.dk, a.dv = N, Hk, Hv, dk, dv
    if state_indices is not None:
        if state_indices.dtype != torch.int32 or state_indices.shape != (N,):
            raise ValueError("state_indices must be int32 [N]")
        a.num_slots = state.shape[0]
    elif state.shape[0] != N:
        raise ValueError("without state_indices the state must be [N, Hv, dk, dv]")
    if tuple(state.shape[1:]) != (Hv, dk, dv):
        raise ValueError(f"state must be float32 [slots, {Hv}, {dk}, {dv}]")
    a.q, a.k, a.v, a.beta, a.g = _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g)
    a.S, a.state_indices, a.o = _ptr(state), _ptr(state_indices), _ptr(o)
    a.flags = flags
    return a


def gdn_decode_step(q, k, v, beta, g, state, state_indices=None, *, out=None, flags: int = 0,
                    check_device_status: bool = False):
    """One decode token per sequence; updates ``state`` in place and returns o [N, Hv, dv].

    q, k: [N, Hk, dk]; v: [N, Hv, dv] (one dtype, fp32 or bf16); beta, g: [N, Hv] fp32;
    state: fp32 [N, Hv, dk, dv] (H = S^T, as S_T of gdn_chunk_fwd), or a pool of slots
    [num_slots, Hv, dk, dv] indexed by ``state_indices`` (int32 [N] on the device; negative
    = skip that sequence).  flags: GDN_FLAG_GATE_LOGITS (beta, g as logits), GDN_FLAG_QK_L2NORM
    (raw q, k normalised inside) or 0.
    """
    o = out if out is not None else torch.empty(v.shape, dtype=q.dtype, device=q.device)
    a = _decode_args(q, k, v, beta, g, state, state_indices, o, flags)
    st = _dev_status(q.device, check_device_status)
    a.dev_status = _ptr(st)
    _check("gdn_decode_step", _abi.lib().gdn_decode_step(ctypes.byref(a), _stream(q.device)))
    _raise_dev_status("gdn_decode_step", st)
    return o


def gdn_affine_combine(M, X, B=None):
    """X <- M X + B in place for every (sequence, value head); returns X.

    M: fp32 [N, Hv, dk, dk]; X, B: fp32 [N, Hv, dk, dv] (B None = zero); X must not share
    memory with M or B.  One step of the fold that gives a shard of a long sequence its entry
    state (``cp_chunk_fwd``).
    """
    if M.dtype != torch.float32 or X.dtype != torch.float32 or (B is not None and B.dtype != torch.float32):
        raise ValueError("M, X and B must be float32")
    if M.dim() != 4 or X.dim() != 4 or M.shape[:2] != X.shape[:2] or M.shape[2] != M.shape[3] or \
            M.shape[2] != X.shape[2] or (B is not None and B.shape != X.shape):
        raise ValueError("M must be [N, Hv, dk, dk], X and B [N, Hv, dk, dv]")
    a = GdnCombineArgs()
    a.struct_size = ctypes.sizeof(a)
    a.abi_version = _abi.GDN_ABI_VERSION
    a.N, a.Hv, a.dk, a.dv = X.shape
    a.M, a.B, a.X = _ptr(M), _ptr(B), _ptr(X)
    _check("gdn_affine_combine", _abi.lib().gdn_affine_combine(ctypes.byref(a), _stream(X.device)))
    return X


def gdn_halo_check(k, beta, g, log_eps: float, *, flags: int = 0, log_decay: bool = False):
    """Per value head, whether the tokens of k, beta, g (a halo) can stand in for everything
    before them: int32 [Hv] (1 = yes), and with ``log_decay`` also their summed log decay.

    k: [T, Hk, dk] (fp32 or bf16); beta, g: [T, Hv] fp32; flags: GDN_FLAG_GATE_LOGITS,
    GDN_FLAG_QK_L2NORM as in the forward.
    """
    if k.dim() != 3 or beta.dim() != 2 or g.shape != beta.shape or beta.shape[0] != k.shape[0]:
        raise ValueError("k must be [T, Hk, dk], beta and g [T, Hv]")
    if k.dtype not in _DT or beta.dtype != torch.float32 or g.dtype != torch.float32:
        raise ValueError("k must be float32 or bfloat16, beta and g float32")
    T, Hk, dk = k.shape
    Hv = beta.shape[1]
    ok = torch.empty(Hv, dtype=torch.int32, device=k.device)
    ld = torch.empty(Hv, dtype=torch.float32, device=k.device) if log_decay else None
    a = GdnHaloArgs()
    a.struct_size = ctypes.sizeof(a)
    a.abi_version = _abi.GDN_ABI_VERSION
    a.dtype = _DT[k.dtype]
    a.T, a.Hk, a.Hv, a.dk = T, Hk, Hv, dk
    a.flags = flags
    a.log_eps = float(log_eps)
    a.k, a.beta, a.g = (_ptr(k), _ptr(beta), _ptr(g)) if T > 0 else (None, None, None)
    a.ok, a.log_decay = _ptr(ok), _ptr(ld)
    _check("gdn_halo_check", _abi.lib().gdn_halo_check(ctypes.byref(a), _stream(k.device)))
    return (ok, ld) if log_decay else ok


def launch_count(q, k, v, beta, g, cu_seqlens=None, cu_seqlens_host=None, initial_state=None,
                 flags: int = 0, backward: bool = False) -> int:
    """Kernel launches one gdn_chunk_fwd (or _bwd) call enqueues for these arguments."""
    a = GdnBwdArgs() if backward else GdnFwdArgs()
    _, host = _fill_common(a, q, k, v, beta, g, cu_seqlens, cu_seqlens_host, initial_state, flags)
    fn = _abi.lib().gdn_chunk_bwd_launch_count if backward else _abi.lib().gdn_chunk_fwd_launch_count
    return int(fn(ctypes.byref(a)))


# short names: chunk_fwd(q, k, v, beta, g, cu_seqlens=None, initial_state=None) -> (o, S_T) and
# chunk_bwd(...) -> (dq, dk, dv, dbeta, dg, dS0) are the same calls
chunk_fwd = gdn_chunk_fwd
chunk_bwd = gdn_chunk_bwd
decode_step = gdn_decode_step
