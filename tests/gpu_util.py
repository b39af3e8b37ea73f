"""Helpers of the GPU parity tests: run the oracle on the exact (cast) inputs
the kernels see, and compare with the tolerances the workloads state."""
import numpy as np
import torch

import oracle

TOL = {torch.float32: dict(rel_l2=1e-4, max_abs=None),
       torch.bfloat16: dict(rel_l2=1e-2, max_abs=2e-2)}


def f64(t):
    if t is None:
        return None
    return t.detach().to("cpu", torch.float64).numpy()


def rel_l2(got, ref):
    nr = np.linalg.norm(ref)
    nd = np.linalg.norm(got - ref)
    return nd / nr if nr > 0 else nd


def check(name, got, ref, io_dtype):
    """fp32 I/O: relative L2 <= 1e-4.  bf16 I/O: relative L2 <= 1e-2 and
    max-abs <= 2e-2 * max|ref|.  Per whole tensor."""
    got = f64(got) if isinstance(got, torch.Tensor) else np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), name + ": non-finite values"
    tol = TOL[io_dtype]
    r = rel_l2(got, ref)
    assert r <= tol["rel_l2"], "%s: rel-L2 %.3e > %.1e" % (name, r, tol["rel_l2"])
    if tol["max_abs"] is not None:
        m = np.abs(got - ref).max() if got.size else 0.0
        lim = tol["max_abs"] * (np.abs(ref).max() if ref.size else 0.0)
        assert m <= lim + 1e-30, "%s: max-abs %.3e > %.3e" % (name, m, lim)
    return r


def batched_to_packed(x):
    """[B, T, H, D] -> [B*T, H, D] (same memory order)."""
    return x.reshape(-1, *x.shape[2:])


def oracle_fwd_batched(inp, S0=None, chunk=0):
    B, T = inp["q"].shape[:2]
    cu = oracle.batched_cu_seqlens(B, T)
    P = lambda key: f64(batched_to_packed(inp[key]))
    o, ST, cs = oracle.fwd(cu, P("q"), P("k"), P("v"), P("g"), inp["sign"].reshape(B * T, *inp["sign"].shape[2:]).numpy(),
                           P("beta"), S0=f64(S0), chunk=chunk)
    o = o.reshape(B, T, *o.shape[1:])
    return o, ST, cs


def oracle_bwd_batched(inp, dO, S0=None, dST=None):
    B, T = inp["q"].shape[:2]
    cu = oracle.batched_cu_seqlens(B, T)
    P = lambda x: f64(batched_to_packed(x))
    r = oracle.bwd(cu, P(inp["q"]), P(inp["k"]), P(inp["v"]), P(inp["g"]),
                   inp["sign"].reshape(B * T, *inp["sign"].shape[2:]).numpy(), P(inp["beta"]),
                   P(dO), S0=f64(S0), dST=f64(dST))
    for key in ("dq", "dk", "dv", "dg", "dbeta"):
        r[key] = r[key].reshape(B, T, *r[key].shape[1:])
    return r


def to_dev(inp, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def random_inputs(B, T, H, dk, dv, io_dtype, seed, gscale=0.05, sign_p=0.25, extreme_p=0.0):
    """Small seeded inputs with the workloads' value distributions (and a
    configurable decay strength)."""
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(B, T, H, dk, generator=gen)
    k = torch.randn(B, T, H, dk, generator=gen)
    q = q / q.norm(dim=-1, keepdim=True)
    k = k / k.norm(dim=-1, keepdim=True)
    v = torch.randn(B, T, H, dv, generator=gen)
    beta = 2 * torch.sigmoid(torch.randn(B, T, H, generator=gen))
    g = -gscale * torch.nn.functional.softplus(torch.randn(B, T, H, dk, generator=gen))
    sign = torch.where(torch.rand(B, T, H, dk, generator=gen) < sign_p,
                       torch.tensor(-1, dtype=torch.int8), torch.tensor(1, dtype=torch.int8))
    if extreme_p > 0:
        ext = torch.rand(B, T, H, generator=gen) < extreme_p
        g = torch.where(ext[..., None], torch.zeros(()), g)
        beta = torch.where(ext, torch.full((), 2.0), beta)
    S0 = 0.1 * torch.randn(B, H, dk, dv, generator=gen)
    dO = torch.randn(B, T, H, dv, generator=gen)
    dST = torch.randn(B, H, dk, dv, generator=gen)
    return dict(q=q.to(io_dtype), k=k.to(io_dtype), v=v.to(io_dtype), beta=beta.to(io_dtype),
                g=g.float().contiguous(), sign=sign.contiguous(), S0=S0, dO=dO.to(io_dtype), dST=dST)
