"""ctypes binding of include/ckda.h: same names, argument marshalling only.

Every function here passes raw device pointers (``tensor.data_ptr()``), sizes
and the CUDA stream handle straight to libckda.so and turns a non-zero status
into :class:`CkdaError`.  All computation happens in the library's kernels;
there is no fallback: if the library is missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "lib", "libckda.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "ckda.h")

CKDA_F32 = 0
CKDA_BF16 = 1
CKDA_OP_CHUNK_FWD = 0
CKDA_OP_CHUNK_BWD = 1
CKDA_OP_VARLEN_FWD = 2
CKDA_OP_VARLEN_BWD = 3
CKDA_CHUNK = 64

STATUS = {0: "CKDA_OK", 1: "CKDA_ERR_INVALID_ARG", 2: "CKDA_ERR_UNSUPPORTED",
          3: "CKDA_ERR_ALIGNMENT", 4: "CKDA_ERR_WORKSPACE", 5: "CKDA_ERR_CUDA",
          6: "CKDA_ERR_TIMEOUT", 7: "CKDA_ERR_DEVICE_ARG", 8: "CKDA_ERR_NOALLOC_CAPACITY"}

_lib = None


class CkdaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = _load().ckda_status_string(status).decode()
        super().__init__("%s: %s (%s)" % (what, STATUS.get(status, status), msg))


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libckda.so is not built (python -m chunked_gated_delta_ckda_b200.build)")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        lib.ckda_workspace_size.argtypes = [I] * 7
        lib.ckda_workspace_size.restype = Z
        lib.ckda_saved_size.argtypes = [I] * 6
        lib.ckda_saved_size.restype = Z
        lib.ckda_chunk_fwd.argtypes = [I] * 6 + [P] * 11 + [Z, P, Z, P]
        lib.ckda_chunk_bwd.argtypes = [I] * 6 + [P] * 11 + [Z] + [P] * 7 + [Z, P]
        lib.ckda_decode_step.argtypes = [I] * 5 + [P] * 9
        lib.ckda_decode_multi.argtypes = [I] * 6 + [P] * 8 + [I, P, I, P, P]
        F = ctypes.c_float
        lib.ckda_prologue_fwd.argtypes = [I] * 6 + [P] * 8 + [F, P, I] + [P] * 7
        lib.ckda_prologue_bwd.argtypes = [I] * 6 + [P] * 8 + [F, P, I] + [P] * 14
        lib.ckda_varlen_fwd.argtypes = [I, I, P, I, I, I, I, I] + [P] * 9 + [P, Z] + [P, Z, P]
        lib.ckda_varlen_bwd.argtypes = [I, I, P, I, I, I, I, I] + [P] * 9 + [P, Z] + [P] * 7 + [Z, P]
        lib.ckda_varlen_saved_size.argtypes = [I] * 6
        lib.ckda_varlen_saved_size.restype = Z
        lib.ckda_chunk_fwd_noalloc.argtypes = [I] * 6 + [P] * 11
        lib.ckda_check_device_status.argtypes = [P, P]
        lib.ckda_selftest_bounded_wait.argtypes = [P, Z, ctypes.c_uint32, P]
        lib.ckda_status_string.argtypes = [I]
        lib.ckda_status_string.restype = ctypes.c_char_p
        lib.ckda_version.argtypes = []
        lib.ckda_profile_enable.argtypes = [I]
        lib.ckda_profile_collect.argtypes = []
        lib.ckda_profile_get.argtypes = [I, ctypes.c_char_p, I, ctypes.POINTER(I),
                                         ctypes.POINTER(ctypes.c_double)]
        lib.ckda_profile_reset.argtypes = []
        lib.ckda_profile_reset.restype = None
        for f in ("ckda_chunk_fwd", "ckda_chunk_bwd", "ckda_decode_step", "ckda_decode_multi", "ckda_varlen_fwd",
                  "ckda_prologue_fwd", "ckda_prologue_bwd", "ckda_varlen_bwd",
                  "ckda_chunk_fwd_noalloc", "ckda_check_device_status", "ckda_selftest_bounded_wait",
                  "ckda_version", "ckda_profile_enable",
                  "ckda_profile_collect", "ckda_profile_get"):
            getattr(lib, f).restype = I
        _lib = lib
    return _lib


def library():
    """The loaded ctypes handle of libckda.so."""
    return _load()


def header_functions() -> list:
    """Names of the functions include/ckda.h declares."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ckda_[a-z_]+)\s*\(", src)))


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(rc: int, what: str):
    if rc != 0:
        raise CkdaError(rc, what)


def _nbytes(ws, ws_bytes):
    if ws_bytes is not None:
        return int(ws_bytes)
    return 0 if ws is None else ws.numel() * ws.element_size()


def ckda_workspace_size(op, B, T, H, dk, dv, N=0) -> int:
    return int(_load().ckda_workspace_size(op, B, T, H, dk, dv, N))


def ckda_saved_size(B, T, H, dk, dv, io_dtype) -> int:
    return int(_load().ckda_saved_size(B, T, H, dk, dv, io_dtype))


def ckda_chunk_fwd(B, T, H, dk, dv, io_dtype, q, k, v, g, sign, beta, S0, o, ST, chunk_states,
                   ws, ws_bytes=None, stream=None, saved=None, saved_bytes=None):
    _check(_load().ckda_chunk_fwd(B, T, H, dk, dv, io_dtype, _p(q), _p(k), _p(v), _p(g),
                                  _p(sign), _p(beta), _p(S0), _p(o), _p(ST), _p(chunk_states),
                                  _p(saved), _nbytes(saved, saved_bytes),
                                  _p(ws), _nbytes(ws, ws_bytes), _s(stream)), "ckda_chunk_fwd")


def ckda_chunk_bwd(B, T, H, dk, dv, io_dtype, q, k, v, g, sign, beta, S0, dO, dST, chunk_states,
                   dq, dk_out, dv_out, dg, dbeta, dS0, ws, ws_bytes=None, stream=None, saved=None,
                   saved_bytes=None):
    _check(_load().ckda_chunk_bwd(B, T, H, dk, dv, io_dtype, _p(q), _p(k), _p(v), _p(g),
                                  _p(sign), _p(beta), _p(S0), _p(dO), _p(dST), _p(chunk_states),
                                  _p(saved), _nbytes(saved, saved_bytes),
                                  _p(dq), _p(dk_out), _p(dv_out), _p(dg), _p(dbeta), _p(dS0),
                                  _p(ws), _nbytes(ws, ws_bytes), _s(stream)), "ckda_chunk_bwd")


def ckda_decode_step(N, H, dk, dv, io_dtype, q, k, v, g, sign, beta, state, o, stream=None):
    _check(_load().ckda_decode_step(N, H, dk, dv, io_dtype, _p(q), _p(k), _p(v), _p(g), _p(sign),
                                    _p(beta), _p(state), _p(o), _s(stream)), "ckda_decode_step")


def ckda_decode_multi(N, K, H, dk, dv, io_dtype, q, k, v, g, sign, beta, n_tokens, slots, n_slots, state,
                      write_state, o, stream=None):
    _check(_load().ckda_decode_multi(N, K, H, dk, dv, io_dtype, _p(q), _p(k), _p(v), _p(g), _p(sign),
                                     _p(beta), _p(n_tokens), _p(slots), n_slots, _p(state),
                                     1 if write_state else 0, _p(o), _s(stream)), "ckda_decode_multi")


def ckda_varlen_bwd(total_T, N, cu_seqlens, max_seqlen, H, dk, dv, io_dtype, q, k, v, g, sign, beta, S0, dO,
                    dST, dq, dk_out, dv_out, dg, dbeta, dS0, ws, ws_bytes=None, stream=None, saved=None,
                    saved_bytes=None):
    _check(_load().ckda_varlen_bwd(total_T, N, _p(cu_seqlens), max_seqlen, H, dk, dv, io_dtype, _p(q), _p(k),
                                   _p(v), _p(g), _p(sign), _p(beta), _p(S0), _p(dO), _p(dST), _p(saved),
                                   _nbytes(saved, saved_bytes), _p(dq), _p(dk_out),
                                   _p(dv_out), _p(dg), _p(dbeta), _p(dS0), _p(ws), _nbytes(ws, ws_bytes),
                                   _s(stream)), "ckda_varlen_bwd")


def ckda_prologue_fwd(B, T, H, dk, dv, io_dtype, xq, xk, xv, wq, wk, wv, a, b, g_floor, q, k, v, g, sign, beta,
                      stream=None, cu_seqlens=None, N=0):
    _check(_load().ckda_prologue_fwd(B, T, H, dk, dv, io_dtype, _p(xq), _p(xk), _p(xv), _p(wq), _p(wk), _p(wv),
                                     _p(a), _p(b), float(g_floor), _p(cu_seqlens), int(N), _p(q), _p(k), _p(v), _p(g), _p(sign), _p(beta),
                                     _s(stream)), "ckda_prologue_fwd")


def ckda_prologue_bwd(B, T, H, dk, dv, io_dtype, xq, xk, xv, wq, wk, wv, a, b, g_floor, dq, dk_in, dv_in, dg, dbeta,
                      dxq, dxk, dxv, dwq, dwk, dwv, da, db, stream=None, cu_seqlens=None, N=0):
    _check(_load().ckda_prologue_bwd(B, T, H, dk, dv, io_dtype, _p(xq), _p(xk), _p(xv), _p(wq), _p(wk), _p(wv),
                                     _p(a), _p(b), float(g_floor), _p(cu_seqlens), int(N), _p(dq), _p(dk_in), _p(dv_in), _p(dg), _p(dbeta),
                                     _p(dxq), _p(dxk), _p(dxv), _p(dwq), _p(dwk), _p(dwv), _p(da), _p(db),
                                     _s(stream)), "ckda_prologue_bwd")


def ckda_varlen_fwd(total_T, N, cu_seqlens, max_seqlen, H, dk, dv, io_dtype, q, k, v, g, sign,
                    beta, S0, o, ST, ws, ws_bytes=None, stream=None, saved=None, saved_bytes=None):
    _check(_load().ckda_varlen_fwd(total_T, N, _p(cu_seqlens), max_seqlen, H, dk, dv, io_dtype,
                                   _p(q), _p(k), _p(v), _p(g), _p(sign), _p(beta), _p(S0), _p(o),
                                   _p(ST), _p(saved), _nbytes(saved, saved_bytes), _p(ws),
                                   _nbytes(ws, ws_bytes), _s(stream)),
           "ckda_varlen_fwd")


def ckda_varlen_saved_size(total_T, N, H, dk, dv, io_dtype):
    return int(_load().ckda_varlen_saved_size(total_T, N, H, dk, dv, io_dtype))


def ckda_chunk_fwd_noalloc(B, T, H, dk, dv, io_dtype, q, k, v, g, sign, beta, S0, o, ST,
                           chunk_states, stream=None):
    """ckda_chunk_fwd without a workspace: the library's fixed scratch array
    is used instead (for callers that cannot allocate device memory).  Every
    pointer must be on the current device and `stream` must belong to it
    (api.chunk_fwd_noalloc makes the tensors' device current)."""
    _check(_load().ckda_chunk_fwd_noalloc(B, T, H, dk, dv, io_dtype, _p(q), _p(k), _p(v), _p(g),
                                          _p(sign), _p(beta), _p(S0), _p(o), _p(ST),
                                          _p(chunk_states), _s(stream)), "ckda_chunk_fwd_noalloc")


def ckda_check_device_status(ws, stream=None) -> int:
    """Device-side status of the last call that used ``ws`` (syncs the stream)."""
    return int(_load().ckda_check_device_status(_p(ws), _s(stream)))


def ckda_selftest_bounded_wait(ws, polls, stream=None):
    """Failure-detection self-test: a bounded wait on a barrier nothing
    arrives at gives up after ``polls`` polls and records the time-out in
    ``ws``'s status word (read it with ckda_check_device_status)."""
    _check(_load().ckda_selftest_bounded_wait(_p(ws), _nbytes(ws, None), int(polls), _s(stream)),
           "ckda_selftest_bounded_wait")


def ckda_status_string(status: int) -> str:
    return _load().ckda_status_string(status).decode()


def ckda_version() -> int:
    return int(_load().ckda_version())


def ckda_profile_enable(on: bool) -> bool:
    return bool(_load().ckda_profile_enable(1 if on else 0))


def ckda_profile_reset() -> None:
    _load().ckda_profile_reset()


def ckda_profile_collect() -> dict:
    """{kernel name: (launches, total ms)} of the launches timed so far."""
    lib = _load()
    n = lib.ckda_profile_collect()
    if n < 0:
        raise CkdaError(-n, "ckda_profile_collect")
    out = {}
    buf = ctypes.create_string_buffer(128)
    cnt = ctypes.c_int()
    tot = ctypes.c_double()
    for i in range(n):
        _check(lib.ckda_profile_get(i, buf, 128, ctypes.byref(cnt), ctypes.byref(tot)),
               "ckda_profile_get")
        out[buf.value.decode()] = (cnt.value, tot.value)
    return out
