"""Plain fp64 CPU oracle for the CKDA recurrence (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares no code with it.

The arithmetic lives in ``ckda_oracle.c`` (token-by-token recurrence with the
signed gate applied directly, and its hand-derived reverse mode).  This module
only compiles it with gcc and marshals numpy arrays.

Every function is pinned by ``tests/test_oracle_pins.py`` to facts the pages
and the mathematics fix (orthogonality at |alpha| = 1, beta = 2; the 2-D
rotation; non-expansiveness; closed forms; dense brute force; finite
differences).  The backward is the exact gradient of the recurrence, pinned by
finite differences; the pages refer to an appendix with a "backward
convention" for the gate's magnitude floor that they do not contain, so no
other convention is implemented or compared.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ckda_oracle.c")
_LIB = os.path.join(_HERE, "libckda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, IEEE double, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # CKDA_ORACLE_LIB points at an alternate build of ckda_oracle.c; only the
        # mutation test (planted mistakes, CPU) sets it.
        alt = os.environ.get("CKDA_ORACLE_LIB")
        if alt:
            lib = ctypes.CDLL(alt)
        else:
            build()
            lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.ckda_oracle_fwd.argtypes = [I, P, I, I, I, P, P, P, P, P, P, P, P, P, I, P, I]
        lib.ckda_oracle_bwd.argtypes = [I, P, I, I, I, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, I]
        lib.ckda_oracle_decode.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P, I]
        for f in (lib.ckda_oracle_fwd, lib.ckda_oracle_bwd, lib.ckda_oracle_decode):
            f.restype = I
        lib.ckda_oracle_default_threads.restype = I
        _lib = lib
    return _lib


def default_threads() -> int:
    return _load().ckda_oracle_default_threads()


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def _sign(x):
    s = np.ascontiguousarray(np.asarray(x, dtype=np.int8))
    if s.size and not np.all(np.abs(s) == 1):
        raise ValueError("sign entries must be +1 or -1")
    return s


def _packed(cu_seqlens, q, k, v, g, sign, beta):
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    sign = _sign(sign)
    T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (T, H, dk) and g.shape == (T, H, dk) and sign.shape == (T, H, dk)
    assert v.shape == (T, H, dv) and beta.shape == (T, H)
    assert cu[0] == 0 and cu[-1] == T and np.all(np.diff(cu) >= 0)
    return cu, q, k, v, g, sign, beta, T, H, dk, dv


def fwd(cu_seqlens, q, k, v, g, sign, beta, S0=None, chunk=0, nthreads=0):
    """Token-by-token forward over packed sequences.

    q, k, g, sign: [T, H, dk]; v: [T, H, dv]; beta: [T, H];
    S0: [N, H, dk, dv] or None (zero).  Returns (o [T,H,dv], ST [N,H,dk,dv],
    chunk_states or None).  With chunk > 0, chunk_states[c] is the state before
    token j*chunk of its sequence, global chunk index c (sequence-major).
    """
    cu, q, k, v, g, sign, beta, T, H, dk, dv = _packed(cu_seqlens, q, k, v, g, sign, beta)
    N = len(cu) - 1
    S0 = None if S0 is None else _f64(S0)
    if S0 is not None:
        assert S0.shape == (N, H, dk, dv)
    o = np.zeros((T, H, dv))
    ST = np.zeros((N, H, dk, dv))
    cs = None
    if chunk > 0:
        nc = int(sum((int(cu[i + 1] - cu[i]) + chunk - 1) // chunk for i in range(N)))
        cs = np.zeros((nc, H, dk, dv))
    rc = _load().ckda_oracle_fwd(N, _ptr(cu), H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                 _ptr(sign), _ptr(beta), _ptr(S0), _ptr(o), _ptr(ST),
                                 int(chunk), _ptr(cs), int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle fwd failed")
    return o, ST, cs


def bwd(cu_seqlens, q, k, v, g, sign, beta, dO, S0=None, dST=None, nthreads=0):
    """Exact reverse mode of ``fwd``.  Returns dict dq, dk, dv, dg, dbeta, dS0."""
    cu, q, k, v, g, sign, beta, T, H, dk, dv = _packed(cu_seqlens, q, k, v, g, sign, beta)
    N = len(cu) - 1
    dO = _f64(dO)
    assert dO.shape == (T, H, dv)
    S0 = None if S0 is None else _f64(S0)
    dST = None if dST is None else _f64(dST)
    out = dict(dq=np.zeros((T, H, dk)), dk=np.zeros((T, H, dk)), dv=np.zeros((T, H, dv)),
               dg=np.zeros((T, H, dk)), dbeta=np.zeros((T, H)), dS0=np.zeros((N, H, dk, dv)))
    rc = _load().ckda_oracle_bwd(N, _ptr(cu), H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                 _ptr(sign), _ptr(beta), _ptr(S0), _ptr(dO), _ptr(dST),
                                 _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                 _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["dS0"]),
                                 int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle bwd failed")
    return out


def decode(q, k, v, g, sign, beta, state, nthreads=0):
    """One recurrent step for independent states.  q,k,g,sign: [N,H,dk];
    v: [N,H,dv]; beta: [N,H]; state: [N,H,dk,dv].  Returns (o, new_state)."""
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    sign = _sign(sign)
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    N, H, dk = q.shape
    dv = v.shape[-1]
    assert st.shape == (N, H, dk, dv)
    o = np.zeros((N, H, dv))
    rc = _load().ckda_oracle_decode(N, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                    _ptr(sign), _ptr(beta), _ptr(st), _ptr(o), int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle decode failed")
    return o, st


def decode_multi(q, k, v, g, sign, beta, pool, n_tokens=None, slots=None, write_state=True,
                 nthreads=0):
    """Up to K recurrent steps per sequence on states held in a slot pool
    ("openeurollm/complex-kda-1.3B-100B" model card: purely recurrent
    inference, one token at a time), written as repeated ``decode`` steps.

    q, k, g, sign: [N,K,H,dk]; v: [N,K,H,dv]; beta: [N,K,H]; pool:
    [n_slots,H,dk,dv].  Sequence n starts from pool[slots[n]] (slot n when
    slots is None) and takes n_tokens[n] steps (clamped to [0, K]; K when
    None); a slot outside [0, n_slots) skips the sequence.  Returns (o
    [N,K,H,dv], with zero rows for the steps not taken; the pool after the
    steps when write_state, else an unchanged copy)."""
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    N, K, H, dk = q.shape
    dv = v.shape[-1]
    sign = np.ones((N, K, H, dk), dtype=np.int8) if sign is None else _sign(sign)
    pool = np.array(pool, dtype=np.float64, copy=True, order="C")
    n_slots = pool.shape[0]
    nt = np.full(N, K, dtype=np.int64) if n_tokens is None else np.clip(np.asarray(n_tokens, np.int64), 0, K)
    sl = np.arange(N, dtype=np.int64) if slots is None else np.asarray(slots, np.int64)
    live = np.array([n for n in range(N) if 0 <= sl[n] < n_slots], dtype=np.int64)
    o = np.zeros((N, K, H, dv))
    st = pool[sl[live]] if len(live) else np.zeros((0, H, dk, dv))
    for t in range(K):
        act = np.nonzero(nt[live] > t)[0]
        if len(act) == 0:
            break
        seqs = live[act]
        ot, new = decode(q[seqs, t], k[seqs, t], v[seqs, t], g[seqs, t], sign[seqs, t], beta[seqs, t],
                         st[act], nthreads=nthreads)
        o[seqs, t] = ot
        st[act] = new
    if write_state and len(live):
        pool[sl[live]] = st
    return o, pool


def batched_cu_seqlens(B: int, T: int) -> np.ndarray:
    """Offsets of B back-to-back sequences of length T ([B,T,...] == [B*T,...])."""
    return np.arange(B + 1, dtype=np.int64) * T


from .prologue import prologue_bwd, prologue_fwd  # noqa: E402,F401  (the token-mixer prologue)
