"""Seeded synthetic inputs for the CKDA recurrence (shared by tests and bench).

This module draws random numbers and nothing else: it holds none of the
recurrence's arithmetic, does not import the oracle and does not import the
CUDA binding.  Both sides of every parity check read the SAME tensors it
returns (already cast to the I/O dtype), so the oracle sees exactly the values
the kernels see.

Shapes follow the 1.3B model's token mixer ("openeurollm/complex-kda-1.3B-100B"
model card, Architecture: 16 heads of dimension 128, context 4096).  Value
distributions (per the workload definitions this library is measured on):

* q, k ~ N(0, 1), each per-head vector scaled to unit L2 norm;
* v ~ N(0, 1);
* beta = 2 * sigmoid(N(0, 1))               (range [0, 2]);
* log|alpha| = g = -0.05 * softplus(N(0, 1)), optionally clamped below at -5;
* sign(alpha) = -1 with probability 1/4, i.i.d. per token and channel;
* "extreme" tokens (Bernoulli per token-head): g = 0 on every channel and
  beta = 2, i.e. the orthogonal signed-Householder transition;
* initial states ~ N(0, 0.1^2) where a workload carries one; d_o ~ N(0, 1).

Draw order within one workload is fixed: q, k, v, beta-logit, g-logit, sign,
extremes, S0, dO (only those the workload uses), all fp32 from one
``torch.Generator('cpu')`` seeded with the workload's seed.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass
class Workload:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    io_dtype: torch.dtype
    seed: int
    g_floor: Optional[float] = None
    extreme_p: float = 0.0
    with_S0: bool = False
    with_dO: bool = False
    with_dST: bool = False
    doc_lens: Optional[list] = None  # packed variable-length workload
    decode_steps: int = 0  # recurrent decode workload
    note: str = ""
    extra: dict = field(default_factory=dict)


# The five workloads this library is built and measured against.
TINY = Workload("tiny_fwd_fp32", B=1, H=2, T=256, dk=64, dv=64, io_dtype=torch.float32, seed=0,
                note="tiny forward, fp32 I/O, zero initial state")
LAYER_FWD = Workload("layer_fwd_bf16", B=8, H=16, T=4096, dk=128, dv=128, io_dtype=torch.bfloat16,
                     seed=1, g_floor=-5.0, extreme_p=0.05,
                     note="1.3B-layer forward, bf16 I/O, fp32 gate and state")
LAYER_FWDBWD = Workload("layer_fwdbwd_bf16", B=8, H=16, T=4096, dk=128, dv=128,
                        io_dtype=torch.bfloat16, seed=2, g_floor=-5.0, extreme_p=0.05,
                        with_dO=True, note="1.3B-layer forward+backward, bf16 I/O")
VARLEN_TOTAL = 65536
VARLEN = Workload("varlen_fwd_bf16", B=1, H=16, T=VARLEN_TOTAL, dk=128, dv=128,
                  io_dtype=torch.bfloat16, seed=3, g_floor=-5.0, extreme_p=0.05,
                  note="packed documents, state reset at each boundary")
LONG = Workload("long_fwd_bf16", B=1, H=16, T=VARLEN_TOTAL, dk=128, dv=128, io_dtype=torch.bfloat16,
                seed=3, g_floor=-5.0, extreme_p=0.05, with_S0=True,
                note="one 65536-token sequence with a random initial state")
DECODE = Workload("decode_bf16", B=256, H=16, T=1, dk=128, dv=128, io_dtype=torch.bfloat16,
                  seed=4, with_S0=True, decode_steps=512,
                  note="recurrent decode, 512 consecutive one-token steps")

# Multi-token decode on a slot pool: 256 live sequences placed at random in a
# pool of 512 states, 4 tokens each per call (a speculative-decoding verify
# width; every call commits all 4).
DECODE_MULTI = Workload("decode_multi_bf16", B=256, T=4, H=16, dk=128, dv=128, io_dtype=torch.bfloat16,
                        seed=5, with_S0=True, decode_steps=64, extra={"n_slots": 512},
                        note="4 tokens per sequence per call, states in a 512-slot pool")


def _gen(seed: int) -> torch.Generator:
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    return gen


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def draw(shape_t: tuple, H: int, dk: int, dv: int, io_dtype: torch.dtype, gen: torch.Generator,
         g_floor: Optional[float] = None, extreme_p: float = 0.0) -> dict:
    """Per-token inputs of leading shape ``shape_t`` (e.g. (B, T) or (N,)).

    Returns q, k, v, beta in ``io_dtype``; g fp32; sign int8 (+1/-1).
    """
    q = _unit(torch.randn(*shape_t, H, dk, generator=gen))
    k = _unit(torch.randn(*shape_t, H, dk, generator=gen))
    v = torch.randn(*shape_t, H, dv, generator=gen)
    beta = 2.0 * torch.sigmoid(torch.randn(*shape_t, H, generator=gen))
    g = -0.05 * torch.nn.functional.softplus(torch.randn(*shape_t, H, dk, generator=gen))
    if g_floor is not None:
        g = g.clamp_min(g_floor)
    sign = torch.where(torch.rand(*shape_t, H, dk, generator=gen) < 0.25,
                       torch.tensor(-1, dtype=torch.int8), torch.tensor(1, dtype=torch.int8))
    if extreme_p > 0:
        ext = torch.rand(*shape_t, H, generator=gen) < extreme_p
        g = torch.where(ext[..., None], torch.zeros((), dtype=g.dtype), g)
        beta = torch.where(ext, torch.full((), 2.0), beta)
    return dict(q=q.to(io_dtype).contiguous(), k=k.to(io_dtype).contiguous(),
                v=v.to(io_dtype).contiguous(), beta=beta.to(io_dtype).contiguous(),
                g=g.float().contiguous(), sign=sign.contiguous())


def make(w: Workload, B: Optional[int] = None, T: Optional[int] = None, H: Optional[int] = None) -> dict:
    """Inputs of a batched workload [B, T, H, d] (optionally resized)."""
    B = w.B if B is None else B
    T = w.T if T is None else T
    H = w.H if H is None else H
    gen = _gen(w.seed)
    out = draw((B, T), H, w.dk, w.dv, w.io_dtype, gen, w.g_floor, w.extreme_p)
    out["S0"] = (0.1 * torch.randn(B, H, w.dk, w.dv, generator=gen)) if w.with_S0 else None
    out["dO"] = torch.randn(B, T, H, w.dv, generator=gen).to(w.io_dtype) if w.with_dO else None
    out["dST"] = torch.randn(B, H, w.dk, w.dv, generator=gen) if w.with_dST else None
    return out


def doc_lengths(total: int, mean: float, lo: int, hi: int, gen: torch.Generator) -> list:
    """Document lengths ~ Geometric(p = 1/mean) on {1, 2, ...}, clipped to
    [lo, hi], drawn until they cover ``total`` tokens; the last one is cut to
    the remainder; a remainder shorter than ``lo`` joins the previous document
    (split again if that exceeds ``hi``)."""
    p = 1.0 / mean
    lens = []
    acc = 0
    while acc < total:
        u = float(torch.rand((), generator=gen).clamp_min(1e-300))
        L = max(1, math.ceil(math.log(u) / math.log1p(-p)))
        L = min(max(L, lo), hi)
        L = min(L, total - acc)
        lens.append(L)
        acc += L
    if len(lens) > 1 and lens[-1] < lo:
        last = lens.pop()
        merged = lens.pop() + last
        while merged > hi:
            lens.append(hi)
            merged -= hi
        lens.append(merged)
    return lens


def make_varlen(w: Workload = VARLEN, total: Optional[int] = None, H: Optional[int] = None,
                mean: float = 1500.0, lo: int = 16, hi: int = 4096, lens: Optional[list] = None) -> dict:
    """Packed documents: q, k, v, ... of shape [1, total, H, d] plus cu_seqlens (int32)."""
    total = w.T if total is None else total
    H = w.H if H is None else H
    gen = _gen(w.seed)
    if lens is None:
        lens = doc_lengths(total, mean, lo, hi, gen)
    total = int(sum(lens))
    out = draw((1, total), H, w.dk, w.dv, w.io_dtype, gen, w.g_floor, w.extreme_p)
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0).to(torch.int32)
    out["cu_seqlens"] = cu
    out["lens"] = list(lens)
    out["S0"] = (0.1 * torch.randn(len(lens), H, w.dk, w.dv, generator=gen)) if w.with_S0 else None
    return out


def make_decode_state(w: Workload = DECODE, N: Optional[int] = None, H: Optional[int] = None) -> torch.Tensor:
    N = w.B if N is None else N
    H = w.H if H is None else H
    return 0.1 * torch.randn(N, H, w.dk, w.dv, generator=_gen(w.seed))


def make_decode_step(w: Workload = DECODE, step: int = 0, N: Optional[int] = None,
                     H: Optional[int] = None) -> dict:
    """Per-token inputs [N, H, d] of decode step ``step`` (independently seeded
    per step, so any step can be regenerated alone)."""
    N = w.B if N is None else N
    H = w.H if H is None else H
    gen = _gen(w.seed * 1_000_003 + 7919 * (step + 1))
    return draw((N,), H, w.dk, w.dv, w.io_dtype, gen, w.g_floor, w.extreme_p)


def make_decode_multi(w: Workload = DECODE_MULTI, call: int = 0) -> dict:
    """Per-token inputs [N, K, H, d] of multi-token decode call ``call``
    (independently seeded per call) and the slot table: a fixed random
    placement of the N sequences in the pool."""
    N, K = w.B, w.T
    gen = _gen(w.seed * 1_000_003 + 7919 * (call + 1))
    out = draw((N, K), w.H, w.dk, w.dv, w.io_dtype, gen, w.g_floor, w.extreme_p)
    out["slots"] = torch.randperm(w.extra["n_slots"], generator=_gen(w.seed))[:N].to(torch.int32)
    return out


def make_decode_pool(w: Workload = DECODE_MULTI) -> torch.Tensor:
    """The state pool [n_slots, H, dk, dv], N(0, 0.1^2)."""
    return 0.1 * torch.randn(w.extra["n_slots"], w.H, w.dk, w.dv, generator=_gen(w.seed + 1))


def make_prologue(w: Workload = LAYER_FWDBWD, B: Optional[int] = None) -> dict:
    """Inputs of the token-mixer prologue at a layer's shape: projections
    xq, xk, xv ~ N(0, 1) in the I/O dtype, conv taps ~ N(0, 0.5^2) fp32
    [H*d, 4], gate pre-activation a ~ N(0, 1.5^2) fp32, beta pre-activation
    b ~ N(0, 2^2); and the upstream gradients dq, dk, dv, dbeta ~ N(0, 1)
    (I/O dtype), dg ~ N(0, 1) fp32."""
    B = w.B if B is None else B
    T, H, dk, dv, io = w.T, w.H, w.dk, w.dv, w.io_dtype
    gen = _gen(w.seed * 7 + 11)
    r = lambda *shape: torch.randn(*shape, generator=gen)
    return dict(xq=r(B, T, H, dk).to(io), xk=r(B, T, H, dk).to(io), xv=r(B, T, H, dv).to(io),
                wq=0.5 * r(H * dk, 4), wk=0.5 * r(H * dk, 4), wv=0.5 * r(H * dv, 4),
                a=1.5 * r(B, T, H, dk), b=(2.0 * r(B, T, H)).to(io),
                dq=r(B, T, H, dk).to(io), dk=r(B, T, H, dk).to(io), dv=r(B, T, H, dv).to(io),
                dg=r(B, T, H, dk), dbeta=r(B, T, H).to(io))
