"""The chunked WY/UT algebra the kernels implement equals the oracle's token
recurrence (forward and backward) to fp64 rounding, including partial last
chunks, packed sequences, initial states and an upstream state gradient."""
import numpy as np
import pytest

import oracle
from tests import chunked_form as cf

RNG = np.random.default_rng(777)


def _inputs(T, H, dk, dv, gscale=0.05):
    q = RNG.standard_normal((T, H, dk))
    k = RNG.standard_normal((T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = RNG.standard_normal((T, H, dv))
    beta = 2 / (1 + np.exp(-RNG.standard_normal((T, H))))
    g = -gscale * np.log1p(np.exp(RNG.standard_normal((T, H, dk))))
    sign = np.where(RNG.random((T, H, dk)) < 0.25, -1, 1).astype(np.int8)
    return q, k, v, g, sign, beta


@pytest.mark.parametrize("lens,C,gscale", [([130], 64, 0.05), ([64, 1, 37, 200], 16, 0.3),
                                          ([90], 32, 2.0)])
def test_chunked_forward_and_backward_match_oracle(lens, C, gscale):
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, dk, dv = int(cu[-1]), 2, 8, 6
    q, k, v, g, sign, beta = _inputs(T, H, dk, dv, gscale)
    N = len(lens)
    S0 = RNG.standard_normal((N, H, dk, dv))
    dO = RNG.standard_normal((T, H, dv))
    dST = RNG.standard_normal((N, H, dk, dv))
    o_ref, ST_ref, cs_ref = oracle.fwd(cu, q, k, v, g, sign, beta, S0=S0, chunk=C)
    gr = oracle.bwd(cu, q, k, v, g, sign, beta, dO, S0=S0, dST=dST)
    ci = 0
    for i in range(N):
        a, b = cu[i], cu[i + 1]
        for h in range(H):
            args = (q[a:b, h], k[a:b, h], v[a:b, h], g[a:b, h], sign[a:b, h], beta[a:b, h])
            o, ST, starts = cf.fwd(*args, S0[i, h], C=C)
            np.testing.assert_allclose(o, o_ref[a:b, h], atol=1e-11)
            np.testing.assert_allclose(ST, ST_ref[i, h], atol=1e-11)
            np.testing.assert_allclose(np.stack(starts), cs_ref[ci:ci + len(starts), h], atol=1e-11)
            bw = cf.bwd(*args, S0[i, h], dO[a:b, h], dST[i, h], C=C)
            for name in ("dq", "dk", "dv", "dg"):
                np.testing.assert_allclose(bw[name], gr[name][a:b, h], atol=1e-9, err_msg=name)
            np.testing.assert_allclose(bw["dbeta"], gr["dbeta"][a:b, h], atol=1e-9)
            np.testing.assert_allclose(bw["dS0"], gr["dS0"][i, h], atol=1e-9)
        ci += len(starts)


@pytest.mark.parametrize("T,C,gscale", [(200, 64, 0.05), (97, 16, 1.5)])
def test_u_chain_reordering_matches(T, C, gscale):
    """The U-carried forward and the dU-carried reverse pass (reorderings of
    the sequential passes that shorten their per-chunk dependence) equal
    the oracle's outputs, final state and dS_0, and the S-carried chunked
    form's per-chunk dU."""
    H, dk, dv = 1, 8, 6
    q, k, v, g, sign, beta = _inputs(T, H, dk, dv, gscale)
    S0 = RNG.standard_normal((1, H, dk, dv))
    dO = RNG.standard_normal((T, H, dv))
    dST = RNG.standard_normal((1, H, dk, dv))
    cu = np.array([0, T])
    o_ref, ST_ref, _ = oracle.fwd(cu, q, k, v, g, sign, beta, S0=S0)
    gr = oracle.bwd(cu, q, k, v, g, sign, beta, dO, S0=S0, dST=dST)
    args = (q[:, 0], k[:, 0], v[:, 0], g[:, 0], sign[:, 0], beta[:, 0])
    o, ST = cf.fwd_u_chain(*args, S0[0, 0], C=C)
    np.testing.assert_allclose(o, o_ref[:, 0], atol=1e-11)
    np.testing.assert_allclose(ST, ST_ref[0, 0], atol=1e-11)
    dUs, dSend, dS0 = cf.bwd_du_chain(*args, S0[0, 0], dO[:, 0], dST[0, 0], C=C)
    np.testing.assert_allclose(dS0, gr["dS0"][0, 0], atol=1e-9)
    # the S-carried reverse pass, chunk by chunk
    _, _, starts = cf.fwd(*args, S0[0, 0], C=C)
    dS = dST[0, 0].copy()
    for j in range(len(starts) - 1, -1, -1):
        sl = slice(j * C, min(j * C + C, T))
        x = cf.chunk_intra(*(a[sl] for a in args))
        dU = x["Aq"].T @ dO[sl, 0] + x["Khat"] @ dS
        np.testing.assert_allclose(dUs[j], dU, atol=1e-10)
        np.testing.assert_allclose(dSend[j], dS, atol=1e-10)
        dS = x["d"][:, None] * dS + x["QG"].T @ dO[sl, 0] - x["W"].T @ dU
