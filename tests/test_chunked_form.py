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
