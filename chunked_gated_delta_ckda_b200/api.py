"""Tensor-level helpers over the C ABI: allocate outputs and workspaces with
torch (device memory is torch's job here) and call the library.

    o, ST, cs = chunk_fwd(q, k, v, g, sign, beta, S0=None, save_chunk_states=True)
    grads     = chunk_bwd(q, k, v, g, sign, beta, dO, S0=None, dST=None, chunk_states=cs)
    o, ST, cs, sv = chunk_fwd(..., save_chunk_states=True, save_for_backward=True)
    grads     = chunk_bwd(..., chunk_states=cs, saved=sv)   # no recomputation
    o         = decode_step(q, k, v, g, sign, beta, state)     # state updated in place
    o         = decode_multi(q, k, v, g, sign, beta, pool, slots=None, n_tokens=None,
                             write_state=True)                 # K tokens per sequence
    o, ST     = varlen_fwd(q, k, v, g, sign, beta, cu_seqlens, max_seqlen, S0=None)
    o, ST, sv = varlen_fwd(..., save_for_backward=True)
    grads     = varlen_bwd(q, k, v, g, sign, beta, dO, cu_seqlens, max_seqlen, S0=None, dST=None,
                           saved=sv)                           # packed documents
    x         = prologue_fwd(xq, xk, xv, wq, wk, wv, a, b, g_floor=-5.0)   # q, k, v, g, sign, beta
    grads     = prologue_bwd(xq, xk, xv, wq, wk, wv, a, b, dq, dk, dv, dg, dbeta, g_floor=-5.0)
    x         = prologue_fwd(..., cu_seqlens=cu)       # packed documents (B = 1): no history across them

Shapes and dtypes are those of include/ckda.h: q, k, g, sign [B,T,H,dk]; v
[B,T,H,dv]; beta [B,T,H]; g fp32; sign int8 (None: every sign +1, standard
KDA); q, k, v, beta either fp32 or bf16 (all the same); states fp32
[B,H,dk,dv].
"""
from __future__ import annotations

import functools
from typing import Optional

import torch

from . import _abi
from ._abi import (CKDA_BF16, CKDA_F32, CKDA_OP_CHUNK_BWD, CKDA_OP_CHUNK_FWD, CKDA_OP_VARLEN_BWD,
                   CKDA_OP_VARLEN_FWD)

_ws_cache: dict = {}


def io_code(dtype: torch.dtype) -> int:
    if dtype == torch.float32:
        return CKDA_F32
    if dtype == torch.bfloat16:
        return CKDA_BF16
    raise TypeError("q, k, v, beta must be float32 or bfloat16, got %s" % dtype)


def workspace(op: int, B: int, T: int, H: int, dk: int, dv: int, N: int = 0,
              device=None, cache: bool = True) -> torch.Tensor:
    """A workspace of at least ckda_workspace_size(...) bytes (256-aligned)."""
    n = _abi.ckda_workspace_size(op, B, T, H, dk, dv, N)
    device = torch.device(device or "cuda")
    key = (device, torch.cuda.current_stream(device).cuda_stream)
    if cache:
        ws = _ws_cache.get(key)
        if ws is not None and ws.numel() >= max(n, 1):
            return ws
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
    if cache:
        _ws_cache[key] = ws
    return ws


def _cuda_devices(args, kwargs) -> set:
    """The devices of the CUDA tensors among a call's arguments."""
    return {t.device for t in (*args, *kwargs.values()) if getattr(t, "is_cuda", False)}


def _one_device(fn):
    """Every CUDA tensor of the call on one device, made current for the call:
    the library launches on the current device and torch's current stream, and
    a pointer into another GPU's memory must never reach its kernels."""
    @functools.wraps(fn)
    def call(*args, **kwargs):
        devices = _cuda_devices(args, kwargs)
        if len(devices) > 1:
            raise ValueError("all tensors must be on one CUDA device, got %s" % sorted(map(str, devices)))
        if not devices:
            return fn(*args, **kwargs)  # (the argument checks reject it)
        with torch.cuda.device(devices.pop()):
            return fn(*args, **kwargs)
    return call


def _c(x: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if x is None:
        return None
    if not x.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    return x if x.is_contiguous() else x.contiguous()


def _expect(name, t, shape, dtype=None, optional=False):
    """Shape (and dtype) check of one argument: the library reads exactly the
    bytes the sizes imply, so a mismatch must stop here."""
    if t is None:
        if optional:
            return
        raise ValueError("%s is required" % name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))


def _expect_io(io_dtype, **named):
    for name, t in named.items():
        if t is not None and t.dtype != io_dtype:
            raise TypeError("%s must be %s like q, got %s" % (name, io_dtype, t.dtype))


def _recurrence_inputs(q, k, v, g, sign, beta, lead):
    """q, k, g, sign [*lead, H, dk]; v [*lead, H, dv]; beta [*lead, H]."""
    if q.dim() != len(lead) + 2:
        raise ValueError("q must have shape %s + (H, dk), got %s" % (tuple(lead), tuple(q.shape)))
    H, dk = q.shape[-2], q.shape[-1]
    dv = v.shape[-1]
    io_code(q.dtype)
    _expect("k", k, (*lead, H, dk), q.dtype)
    _expect("v", v, (*lead, H, dv), q.dtype)
    _expect("g", g, (*lead, H, dk), torch.float32)
    _expect("sign", sign, (*lead, H, dk), torch.int8, optional=True)
    _expect("beta", beta, (*lead, H), q.dtype)
    return H, dk, dv


def saved_buffer(B, T, H, dk, dv, dtype, device) -> Optional[torch.Tensor]:
    """The forward-to-backward saved buffer (None: this configuration recomputes)."""
    n = _abi.ckda_saved_size(B, T, H, dk, dv, io_code(dtype))
    return torch.empty(n, dtype=torch.uint8, device=device) if n > 0 else None


@_one_device
def chunk_fwd(q, k, v, g, sign, beta, S0=None, output_final_state=True, save_chunk_states=False,
              ws=None, save_for_backward=False):
    B, T = q.shape[:2]
    H, dk, dv = _recurrence_inputs(q, k, v, g, sign, beta, (B, T))
    _expect("S0", S0, (B, H, dk, dv), torch.float32, optional=True)
    q, k, v, g, sign, beta, S0 = map(_c, (q, k, v, g, sign, beta, S0))
    io = io_code(q.dtype)
    o = torch.empty(B, T, H, dv, dtype=q.dtype, device=q.device)
    ST = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device) if output_final_state else None
    NC = (T + 63) // 64
    cs = (torch.empty(B, H, NC, dk, dv, dtype=torch.float32, device=q.device)
          if save_chunk_states else None)
    if ws is None:
        ws = workspace(CKDA_OP_CHUNK_FWD, B, T, H, dk, dv, device=q.device)
    sv = saved_buffer(B, T, H, dk, dv, q.dtype, q.device) if save_for_backward else None
    _abi.ckda_chunk_fwd(B, T, H, dk, dv, io, q, k, v, g, sign, beta, S0, o, ST, cs, ws, saved=sv)
    if save_for_backward:
        return o, ST, cs, sv
    return o, ST, cs


@_one_device
def chunk_fwd_noalloc(q, k, v, g, sign, beta, S0=None, output_final_state=True, save_chunk_states=False):
    """chunk_fwd for callers that cannot allocate device scratch: the library's
    fixed scratch array stands in for the workspace (the outputs are still
    allocated here).  Runs with the tensors' device current and on its current
    stream, as the C call requires."""
    B, T = q.shape[:2]
    H, dk, dv = _recurrence_inputs(q, k, v, g, sign, beta, (B, T))
    _expect("S0", S0, (B, H, dk, dv), torch.float32, optional=True)
    q, k, v, g, sign, beta, S0 = map(_c, (q, k, v, g, sign, beta, S0))
    o = torch.empty(B, T, H, dv, dtype=q.dtype, device=q.device)
    ST = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device) if output_final_state else None
    cs = (torch.empty(B, H, (T + 63) // 64, dk, dv, dtype=torch.float32, device=q.device)
          if save_chunk_states else None)
    _abi.ckda_chunk_fwd_noalloc(B, T, H, dk, dv, io_code(q.dtype), q, k, v, g, sign, beta, S0, o, ST, cs)
    return o, ST, cs


@_one_device
def chunk_bwd(q, k, v, g, sign, beta, dO, S0=None, dST=None, chunk_states=None, need_dS0=True,
              ws=None, saved=None):
    B, T = q.shape[:2]
    H, dk, dv = _recurrence_inputs(q, k, v, g, sign, beta, (B, T))
    _expect("dO", dO, (B, T, H, dv), q.dtype)
    _expect("S0", S0, (B, H, dk, dv), torch.float32, optional=True)
    _expect("dST", dST, (B, H, dk, dv), torch.float32, optional=True)
    _expect("chunk_states", chunk_states, (B, H, (T + 63) // 64, dk, dv), torch.float32, optional=True)
    if saved is not None and saved.dtype != torch.uint8:
        raise TypeError("saved must be the uint8 buffer chunk_fwd returned")
    q, k, v, g, sign, beta, dO, S0, dST, chunk_states, saved = map(
        _c, (q, k, v, g, sign, beta, dO, S0, dST, chunk_states, saved))
    io = io_code(q.dtype)
    dq = torch.empty_like(q)
    dk_ = torch.empty_like(k)
    dv_ = torch.empty_like(v)
    dg = torch.empty_like(g)
    dbeta = torch.empty_like(beta)
    dS0 = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device) if need_dS0 else None
    if ws is None:
        ws = workspace(CKDA_OP_CHUNK_BWD, B, T, H, dk, dv, device=q.device)
    _abi.ckda_chunk_bwd(B, T, H, dk, dv, io, q, k, v, g, sign, beta, S0, dO, dST, chunk_states,
                        dq, dk_, dv_, dg, dbeta, dS0, ws, saved=saved)
    return dict(dq=dq, dk=dk_, dv=dv_, dg=dg, dbeta=dbeta, dS0=dS0)


@_one_device
def decode_step(q, k, v, g, sign, beta, state, o=None):
    N = q.shape[0]
    H, dk, dv = _recurrence_inputs(q, k, v, g, sign, beta, (N,))
    _expect("state", state, (N, H, dk, dv), torch.float32)
    _expect("o", o, (N, H, dv), q.dtype, optional=True)
    q, k, v, g, sign, beta, o = map(_c, (q, k, v, g, sign, beta, o))
    if not state.is_cuda or not state.is_contiguous():
        raise ValueError("state must be a contiguous CUDA tensor (updated in place)")
    if o is None:
        o = torch.empty(N, H, dv, dtype=q.dtype, device=q.device)
    _abi.ckda_decode_step(N, H, dk, dv, io_code(q.dtype), q, k, v, g, sign, beta, state, o)
    return o


@_one_device
def decode_multi(q, k, v, g, sign, beta, pool, slots=None, n_tokens=None, write_state=True, o=None,
                 want_o=True):
    """K steps per sequence: q, k, g, sign [N,K,H,dk]; v [N,K,H,dv]; beta [N,K,H];
    pool [n_slots,H,dk,dv] fp32 (updated in place when write_state);
    slots / n_tokens: int32 [N] on the device, or None (slot n / all K)."""
    N, K = q.shape[:2]
    H, dk, dv = _recurrence_inputs(q, k, v, g, sign, beta, (N, K))
    if pool.dim() != 4:
        raise ValueError("pool must have shape (n_slots, H, dk, dv), got %s" % (tuple(pool.shape),))
    _expect("pool", pool, (pool.shape[0], H, dk, dv), torch.float32)
    _expect("slots", slots, (N,), torch.int32, optional=True)
    _expect("n_tokens", n_tokens, (N,), torch.int32, optional=True)
    _expect("o", o, (N, K, H, dv), q.dtype, optional=True)
    q, k, v, g, sign, beta, slots, n_tokens, o = map(_c, (q, k, v, g, sign, beta, slots, n_tokens, o))
    if not pool.is_cuda or not pool.is_contiguous():
        raise ValueError("pool must be a contiguous CUDA tensor (updated in place)")
    if o is None and want_o:
        o = torch.empty(N, K, H, dv, dtype=q.dtype, device=q.device)
    _abi.ckda_decode_multi(N, K, H, dk, dv, io_code(q.dtype), q, k, v, g, sign, beta, n_tokens, slots,
                           pool.shape[0], pool, write_state, o)
    return o


def _prologue_shapes(xq, xk, xv, wq, wk, wv, a, b):
    if xq.dim() != 4:
        raise ValueError("xq must have shape (B, T, H, dk), got %s" % (tuple(xq.shape),))
    B, T, H, dk = xq.shape
    dv = xv.shape[-1]
    io_code(xq.dtype)
    _expect("xk", xk, (B, T, H, dk), xq.dtype)
    _expect("xv", xv, (B, T, H, dv), xq.dtype)
    _expect("wq", wq, (H * dk, 4), torch.float32)
    _expect("wk", wk, (H * dk, 4), torch.float32)
    _expect("wv", wv, (H * dv, 4), torch.float32)
    _expect("a", a, (B, T, H, dk), torch.float32)
    _expect("b", b, (B, T, H), xq.dtype)
    return B, T, H, dk, dv


def _prologue_docs(B, cu_seqlens):
    """Packed documents' offsets for the prologue: (tensor, N), or (None, 0)."""
    if cu_seqlens is None:
        return None, 0
    if cu_seqlens.dim() != 1 or cu_seqlens.dtype != torch.int32 or cu_seqlens.numel() < 2:
        raise TypeError("cu_seqlens must be a 1-D int32 tensor of N + 1 >= 2 offsets")
    if B != 1:
        raise ValueError("packed documents (cu_seqlens) take a batch of one row, got B=%d" % B)
    return _c(cu_seqlens), cu_seqlens.numel() - 1


@_one_device
def prologue_fwd(xq, xk, xv, wq, wk, wv, a, b, g_floor=-5.0, cu_seqlens=None):
    """Projections [B,T,H,d] (io dtype), conv taps [H*d, 4] fp32, gate
    pre-activation a [B,T,H,dk] fp32, b [B,T,H] -> dict q, k, v, g, sign, beta
    (the inputs of chunk_fwd).  With cu_seqlens (int32 [N+1], B = 1) the
    convolution's history restarts at each packed document's first token
    (the inputs of varlen_fwd)."""
    B, T, H, dk, dv = _prologue_shapes(xq, xk, xv, wq, wk, wv, a, b)
    cu, N = _prologue_docs(B, cu_seqlens)
    xq, xk, xv, wq, wk, wv, a, b = map(_c, (xq, xk, xv, wq, wk, wv, a, b))
    out = dict(q=torch.empty_like(xq), k=torch.empty_like(xk), v=torch.empty_like(xv),
               g=torch.empty(B, T, H, dk, dtype=torch.float32, device=xq.device),
               sign=torch.empty(B, T, H, dk, dtype=torch.int8, device=xq.device), beta=torch.empty_like(b))
    _abi.ckda_prologue_fwd(B, T, H, dk, dv, io_code(xq.dtype), xq, xk, xv, wq, wk, wv, a, b, g_floor,
                           out["q"], out["k"], out["v"], out["g"], out["sign"], out["beta"],
                           cu_seqlens=cu, N=N)
    return out


@_one_device
def prologue_bwd(xq, xk, xv, wq, wk, wv, a, b, dq, dk, dv, dg, dbeta, g_floor=-5.0, cu_seqlens=None):
    """Gradients of prologue_fwd's inputs (same g_floor and cu_seqlens):
    dict dxq, dxk, dxv, dwq, dwk, dwv, da, db."""
    B, T, H, dk_, dv_ = _prologue_shapes(xq, xk, xv, wq, wk, wv, a, b)
    cu, N = _prologue_docs(B, cu_seqlens)
    _expect("dq", dq, (B, T, H, dk_), xq.dtype)
    _expect("dk", dk, (B, T, H, dk_), xq.dtype)
    _expect("dv", dv, (B, T, H, dv_), xq.dtype)
    _expect("dg", dg, (B, T, H, dk_), torch.float32)
    _expect("dbeta", dbeta, (B, T, H), xq.dtype)
    xq, xk, xv, wq, wk, wv, a, b, dq, dk, dv, dg, dbeta = map(
        _c, (xq, xk, xv, wq, wk, wv, a, b, dq, dk, dv, dg, dbeta))
    out = dict(dxq=torch.empty_like(xq), dxk=torch.empty_like(xk), dxv=torch.empty_like(xv),
               dwq=torch.empty_like(wq), dwk=torch.empty_like(wk), dwv=torch.empty_like(wv),
               da=torch.empty_like(a), db=torch.empty_like(b))
    _abi.ckda_prologue_bwd(B, T, H, dk_, dv_, io_code(xq.dtype), xq, xk, xv, wq, wk, wv, a, b, g_floor,
                           dq, dk, dv, dg, dbeta, out["dxq"], out["dxk"], out["dxv"], out["dwq"], out["dwk"],
                           out["dwv"], out["da"], out["db"], cu_seqlens=cu, N=N)
    return out


@_one_device
def varlen_fwd(q, k, v, g, sign, beta, cu_seqlens, max_seqlen, S0=None, output_final_state=True,
               ws=None, save_for_backward=False):
    """Packed documents: o [1,T,H,dv], ST [N,H,dk,dv] (or None); with
    save_for_backward also the saved buffer for varlen_bwd (None where the
    configuration has no saved form)."""
    if q.dim() != 4 or q.shape[0] != 1:
        raise ValueError("packed q must have shape (1, total_T, H, dk), got %s" % (tuple(q.shape),))
    T = q.shape[1]
    H, dk, dv = _recurrence_inputs(q, k, v, g, sign, beta, (1, T))
    if cu_seqlens.dim() != 1 or cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be a 1-D int32 tensor")
    N = cu_seqlens.numel() - 1
    _expect("S0", S0, (N, H, dk, dv), torch.float32, optional=True)
    q, k, v, g, sign, beta, S0, cu_seqlens = map(_c, (q, k, v, g, sign, beta, S0, cu_seqlens))
    o = torch.empty(1, T, H, dv, dtype=q.dtype, device=q.device)
    ST = torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device) if output_final_state else None
    if ws is None:
        ws = workspace(CKDA_OP_VARLEN_FWD, 1, T, H, dk, dv, N, device=q.device)
    sv = None
    if save_for_backward:
        n = _abi.ckda_varlen_saved_size(T, N, H, dk, dv, io_code(q.dtype))
        sv = torch.empty(n, dtype=torch.uint8, device=q.device) if n > 0 else None
    _abi.ckda_varlen_fwd(T, N, cu_seqlens, int(max_seqlen), H, dk, dv, io_code(q.dtype), q, k, v,
                         g, sign, beta, S0, o, ST, ws, saved=sv)
    if save_for_backward:
        return o, ST, sv
    return o, ST


@_one_device
def varlen_bwd(q, k, v, g, sign, beta, dO, cu_seqlens, max_seqlen, S0=None, dST=None, need_dS0=True, ws=None,
               saved=None):
    """Gradients of varlen_fwd: dict dq, dk, dv, dg, dbeta, dS0 ([N,H,dk,dv] or
    None).  saved: the buffer varlen_fwd(save_for_backward=True) returned for
    the same inputs (else the per-chunk results are recomputed)."""
    if q.dim() != 4 or q.shape[0] != 1:
        raise ValueError("packed q must have shape (1, total_T, H, dk), got %s" % (tuple(q.shape),))
    T = q.shape[1]
    H, dk, dv = _recurrence_inputs(q, k, v, g, sign, beta, (1, T))
    if cu_seqlens.dim() != 1 or cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be a 1-D int32 tensor")
    N = cu_seqlens.numel() - 1
    _expect("dO", dO, (1, T, H, dv), q.dtype)
    _expect("S0", S0, (N, H, dk, dv), torch.float32, optional=True)
    _expect("dST", dST, (N, H, dk, dv), torch.float32, optional=True)
    if saved is not None and saved.dtype != torch.uint8:
        raise TypeError("saved must be the uint8 buffer varlen_fwd returned")
    q, k, v, g, sign, beta, dO, S0, dST, cu_seqlens, saved = map(
        _c, (q, k, v, g, sign, beta, dO, S0, dST, cu_seqlens, saved))
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v), dg=torch.empty_like(g),
               dbeta=torch.empty_like(beta),
               dS0=torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device) if need_dS0 else None)
    if ws is None:
        ws = workspace(CKDA_OP_VARLEN_BWD, 1, T, H, dk, dv, N, device=q.device)
    _abi.ckda_varlen_bwd(T, N, cu_seqlens, int(max_seqlen), H, dk, dv, io_code(q.dtype), q, k, v, g, sign, beta,
                         S0, dO, dST, out["dq"], out["dk"], out["dv"], out["dg"], out["dbeta"], out["dS0"], ws,
                         saved=saved)
    return out
