"""Plain fp64 CPU oracle of the token-mixer prologue (test infrastructure only).

What feeds the recurrence, from the raw per-token projections
("openeurollm/complex-kda-1.3B-100B" model card, architecture: 16 heads of
dimension 128, short convolution of width 4; "Complex KDA: ..." paper text,
section 3 "CKDA": beta in [0, 2] and a signed gate in [-1, 1] carried as
log-magnitude and sign; the gate's exact parameterisation, magnitude floor
and backward convention sit in an appendix the pages do not contain).
Readings taken where the pages are silent:

* short convolution: depthwise and causal over the tokens of each sequence,
  width 4, taps ``w[c, 0..3]`` with ``w[c, 3]`` on the current token, zero
  history before the sequence start, then SiLU; on q, k and v; documents
  packed into one row (``cu_seqlens``) are sequences of their own, as they
  are for the recurrence;
* q and k: L2-normalised per head, ``n / sqrt(sum(n^2) + 1e-6)``;
* signed gate: ``alpha = tanh(a)`` (the [-1, 1] range extension of a
  sigmoid gate, 2 sigmoid(2a) - 1), passed on as ``g = max(log|alpha|,
  g_floor)`` and ``sign = -1 where alpha < 0, else +1``;
* ``beta = 2 sigmoid(b)``;
* gradients: exact for these formulas; none through the sign; the floor's
  clamp passes no gradient where it is active.

Written with plain torch fp64 CPU ops; the backward is torch autograd of that
forward (a library primitive as the step).  Pinned in
``tests/test_oracle_prologue.py`` against numpy's convolution, the unit-norm
and range invariants, closed forms and central finite differences.
"""
from __future__ import annotations

import numpy as np
import torch

EPS = 1e-6
WIDTH = 4


def _t(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float64))


def _docs(T, cu_seqlens):
    """[(start, end)] of the packed documents (None: the whole row)."""
    if cu_seqlens is None:
        return None
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    if len(cu) < 2 or cu[0] != 0 or cu[-1] != T or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must rise from 0 to T")
    return [(s, e) for s, e in zip(cu, cu[1:]) if e > s]


def _conv_silu(x, w, docs=None):
    """x [B,T,H,d], w [H*d, 4] -> SiLU(causal depthwise conv), per sequence
    (per packed document when ``docs`` is given)."""
    if docs is not None:
        return torch.cat([_conv_silu(x[:, s:e], w) for s, e in docs], dim=1)
    B, T, H, d = x.shape
    wt = w.reshape(H, d, WIDTH)
    y = torch.zeros_like(x)
    for j in range(WIDTH):
        shift = WIDTH - 1 - j  # tap j reads token t - shift
        if shift >= T:
            continue
        xs = x if shift == 0 else torch.cat([torch.zeros_like(x[:, :shift]), x[:, :T - shift]], dim=1)
        y = y + xs * wt[:, :, j]
    return y * torch.sigmoid(y)


def _forward(xq, xk, xv, wq, wk, wv, a, b, g_floor, docs=None):
    nq, nk = _conv_silu(xq, wq, docs), _conv_silu(xk, wk, docs)
    q = nq / torch.sqrt((nq * nq).sum(-1, keepdim=True) + EPS)
    k = nk / torch.sqrt((nk * nk).sum(-1, keepdim=True) + EPS)
    v = _conv_silu(xv, wv, docs)
    alpha = torch.tanh(a)
    g = torch.clamp(torch.log(torch.abs(alpha)), min=g_floor)
    beta = 2.0 * torch.sigmoid(b)
    return q, k, v, g, beta, alpha


def _packed(xq, cu_seqlens):
    if cu_seqlens is not None and np.shape(xq)[0] != 1:
        raise ValueError("packed documents take a batch of one row")
    return _docs(np.shape(xq)[1], cu_seqlens)


def prologue_fwd(xq, xk, xv, wq, wk, wv, a, b, g_floor=-np.inf, cu_seqlens=None):
    """xq, xk [B,T,H,dk]; xv [B,T,H,dv]; wq, wk [H*dk, 4]; wv [H*dv, 4];
    a [B,T,H,dk]; b [B,T,H]; cu_seqlens: None, or N + 1 offsets of packed
    documents (B = 1).  Returns numpy fp64 q, k, v, g, beta and the int8 sign."""
    docs = _packed(xq, cu_seqlens)
    with torch.no_grad():
        q, k, v, g, beta, alpha = _forward(*map(_t, (xq, xk, xv, wq, wk, wv, a, b)), float(g_floor), docs)
    sign = np.where(alpha.numpy() < 0, -1, 1).astype(np.int8)
    return dict(q=q.numpy(), k=k.numpy(), v=v.numpy(), g=g.numpy(), beta=beta.numpy(), sign=sign)


def prologue_bwd(xq, xk, xv, wq, wk, wv, a, b, dq, dk, dv, dg, dbeta, g_floor=-np.inf, cu_seqlens=None):
    """Gradients of sum(q dq + k dk + v dv + g dg + beta dbeta) with respect to
    the inputs: dict dxq, dxk, dxv, dwq, dwk, dwv, da, db (numpy fp64)."""
    docs = _packed(xq, cu_seqlens)
    ins = [_t(x).requires_grad_(True) for x in (xq, xk, xv, wq, wk, wv, a, b)]
    q, k, v, g, beta, _ = _forward(*ins, float(g_floor), docs)
    loss = ((q * _t(dq)).sum() + (k * _t(dk)).sum() + (v * _t(dv)).sum() + (g * _t(dg)).sum()
            + (beta * _t(dbeta)).sum())
    grads = torch.autograd.grad(loss, ins)
    names = ("dxq", "dxk", "dxv", "dwq", "dwk", "dwv", "da", "db")
    return {n: gr.numpy() for n, gr in zip(names, grads)}
