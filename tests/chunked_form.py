"""The chunked (WY/UT) form of the CKDA recurrence, in plain numpy fp64.

This is the algebra the CUDA kernels implement, written out densely so that
its exactness can be checked against the token-by-token oracle on the CPU
(tests/test_chunked_form.py).  It is test code: the kernels do not use it.

Per chunk of C tokens with start state S (true, signed frame):
  Gam_r = sum_{s<=r} g_s            (chunk-local log-magnitude cumsum)
  p_r   = prod_{s<=r} sign_s        (chunk-local sign product; the pages'
                                     running product P_t equals
                                     P_{chunk start} * p_t, and the start
                                     factor cancels because S is kept in the
                                     true frame at chunk boundaries)
  k' = p k, q' = p q, K_G = k' e^Gam, Q_G = q' e^Gam
  A   = strict_tril( sum_c k'_rc k'_sc e^{Gam_rc - Gam_sc} )
  A_q =        tril( sum_c q'_rc k'_sc e^{Gam_rc - Gam_sc} )
  T   = (I + Diag(beta) A)^{-1} Diag(beta),  W = T K_G,  U0 = T V
  U   = U0 - W S
  O   = Q_G S + A_q U
  S'  = Diag(p_C e^{Gam_C}) S + Khat^T U,  Khat_s = p_C k'_s e^{Gam_C - Gam_s}
"""
import numpy as np


def _pair_decay(Gam):
    """D[r, s, c] = exp(Gam_rc - Gam_sc) for s <= r, else 0."""
    n = Gam.shape[0]
    diff = Gam[:, None, :] - Gam[None, :, :]
    mask = np.tril(np.ones((n, n), dtype=bool))[:, :, None]
    return np.exp(np.where(mask, diff, -np.inf))


def chunk_intra(q, k, v, g, sign, beta):
    n = q.shape[0]
    Gam = np.cumsum(g, axis=0)
    p = np.cumprod(sign.astype(np.float64), axis=0)
    kp, qp = p * k, p * q
    E = np.exp(Gam)
    D = _pair_decay(Gam)
    A = np.einsum("rc,sc,rsc->rs", kp, kp, D) * np.tril(np.ones((n, n)), -1)
    Aq = np.einsum("rc,sc,rsc->rs", qp, kp, D)
    L = np.eye(n) + beta[:, None] * A
    M = np.linalg.inv(L)
    Tm = M * beta[None, :]
    KG, QG = kp * E, qp * E
    W, U0 = Tm @ KG, Tm @ v
    Khat = p[-1] * kp * np.exp(Gam[-1] - Gam)
    d = p[-1] * np.exp(Gam[-1])
    return dict(Gam=Gam, p=p, kp=kp, qp=qp, E=E, D=D, A=A, Aq=Aq, M=M, Tm=Tm, KG=KG, QG=QG,
                W=W, U0=U0, Khat=Khat, d=d)


def fwd(q, k, v, g, sign, beta, S0, C=64):
    """One head of one sequence: q,k,g,sign [T,dk]; v [T,dv]; beta [T]."""
    T = q.shape[0]
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    starts = []
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        x = chunk_intra(q[sl], k[sl], v[sl], g[sl], sign[sl], beta[sl])
        starts.append(S.copy())
        U = x["U0"] - x["W"] @ S
        o[sl] = x["QG"] @ S + x["Aq"] @ U
        S = x["d"][:, None] * S + x["Khat"].T @ U
    return o, S, starts


def bwd(q, k, v, g, sign, beta, S0, dO, dST, C=64):
    T, dk = q.shape
    dv = v.shape[1]
    _, _, starts = fwd(q, k, v, g, sign, beta, S0, C)
    dq, dkk, dvv = np.zeros((T, dk)), np.zeros((T, dk)), np.zeros((T, dv))
    dg, dbeta = np.zeros((T, dk)), np.zeros(T)
    dS = dST.copy()
    chunks = list(range(0, T, C))
    for ci in reversed(range(len(chunks))):
        c0 = chunks[ci]
        sl = slice(c0, min(c0 + C, T))
        n = sl.stop - sl.start
        x = chunk_intra(q[sl], k[sl], v[sl], g[sl], sign[sl], beta[sl])
        Sc, dS1, dOc = starts[ci], dS, dO[sl]
        U = x["U0"] - x["W"] @ Sc
        # reverse state pass
        dU = x["Aq"].T @ dOc + x["Khat"] @ dS1
        dS = x["d"][:, None] * dS1 + x["QG"].T @ dOc - x["W"].T @ dU
        # per-chunk gradient
        lo_incl = np.tril(np.ones((n, n)))
        lo_strict = np.tril(np.ones((n, n)), -1)
        dQG = dOc @ Sc.T
        dAq = (dOc @ U.T) * lo_incl
        dKhat = U @ dS1.T
        dd = np.sum(Sc * dS1, axis=1)
        dW = -dU @ Sc.T
        dT = (dU @ v[sl].T + dW @ x["KG"].T) * lo_incl
        dvv[sl] = x["Tm"].T @ dU
        dKG = x["Tm"].T @ dW
        dM = dT * beta[sl][None, :]
        db = np.sum(dT * x["M"], axis=0)
        dL = -x["M"].T @ dM @ x["M"].T
        dN = dL * lo_strict
        dA = beta[sl][:, None] * dN
        db += np.sum(dN * x["A"], axis=1)
        kp, qp, D, Gam = x["kp"], x["qp"], x["D"], x["Gam"]
        DKl = np.einsum("rs,sc,rsc->rc", dA, kp, D)
        DKr = np.einsum("rs,rc,rsc->sc", dA, kp, D)
        DQl = np.einsum("rs,sc,rsc->rc", dAq, kp, D)
        DKr2 = np.einsum("rs,rc,rsc->sc", dAq, qp, D)
        dkp = DKl + DKr + DKr2
        dqp = DQl.copy()
        dGam = kp * DKl - kp * DKr + qp * DQl - kp * DKr2
        dkp += dKG * x["E"]
        dGam += dKG * x["KG"]
        dqp += dQG * x["E"]
        dGam += dQG * x["QG"]
        pC = x["p"][-1]
        dkp += pC * dKhat * np.exp(Gam[-1] - Gam)
        dGam -= dKhat * x["Khat"]
        dGamC = np.sum(dKhat * x["Khat"], axis=0) + dd * x["d"]
        dGam[-1] += dGamC
        dg[sl] = np.cumsum(dGam[::-1], axis=0)[::-1]
        dq[sl] = x["p"] * dqp
        dkk[sl] = x["p"] * dkp
        dbeta[sl] = db
    return dict(dq=dq, dk=dkk, dv=dvv, dg=dg, dbeta=dbeta, dS0=dS)


def fwd_u_chain(q, k, v, g, sign, beta, S0, C=64):
    """The forward with the chunk-to-chunk dependence carried by U instead of
    S (a reordering for the sequential pass, not yet what the kernels run):

        U_{j+1} = U0_{j+1} - (W_{j+1} Diag(d_j)) S_j - (W_{j+1} Khat_j^T) U_j

    since S_{j+1} = Diag(d_j) S_j + Khat_j^T U_j.  Step j+1's U needs S_j,
    not S_{j+1}: the S update runs one step behind, off the U chain, whose
    only product per step is the 64 x 64 one R_{j+1} U_j."""
    T = q.shape[0]
    xs = [chunk_intra(q[c0:c0 + C], k[c0:c0 + C], v[c0:c0 + C], g[c0:c0 + C], sign[c0:c0 + C],
                      beta[c0:c0 + C]) for c0 in range(0, T, C)]
    o = np.zeros((T, v.shape[1]))
    S = S0.copy()
    U = xs[0]["U0"] - xs[0]["W"] @ S
    for j, x in enumerate(xs):
        sl = slice(j * C, min(j * C + C, T))
        o[sl] = x["QG"] @ S + x["Aq"] @ U
        if j + 1 < len(xs):
            nx = xs[j + 1]
            P = nx["W"] * x["d"][None, :]          # W_{j+1} Diag(d_j), off the chain
            R = nx["W"] @ x["Khat"].T               # W_{j+1} Khat_j^T, 64 x 64, off the chain
            U_next = nx["U0"] - P @ S - R @ U
        S = x["d"][:, None] * S + x["Khat"].T @ U
        if j + 1 < len(xs):
            U = U_next
    return o, S


def bwd_du_chain(q, k, v, g, sign, beta, S0, dO, dST, C=64):
    """The reverse state pass with the dependence carried by dU (the
    counterpart of fwd_u_chain): with dS_j = Diag(d_j) dS_{j+1} +
    QG_j^T dO_j - W_j^T dU_j,

        dU_{j-1} = [A_q_{j-1}^T dO_{j-1} + Khat_{j-1} QG_j^T dO_j]
                   + (Khat_{j-1} Diag(d_j)) dS_{j+1} - (Khat_{j-1} W_j^T) dU_j.

    Returns the per-chunk dU and the chunk-end state gradients dS_{j+1},
    and dS_0, as the reverse pass does."""
    T = q.shape[0]
    xs = [chunk_intra(q[c0:c0 + C], k[c0:c0 + C], v[c0:c0 + C], g[c0:c0 + C], sign[c0:c0 + C],
                      beta[c0:c0 + C]) for c0 in range(0, T, C)]
    n = len(xs)
    dOs = [dO[j * C:min(j * C + C, T)] for j in range(n)]
    dUs, dSend = [None] * n, [None] * n
    dS = dST.copy()                                   # dS_{n}
    dU = xs[-1]["Aq"].T @ dOs[-1] + xs[-1]["Khat"] @ dS
    for j in range(n - 1, -1, -1):
        x = xs[j]
        dUs[j], dSend[j] = dU, dS
        if j > 0:
            px = xs[j - 1]
            Y = px["Khat"] * x["d"][None, :]          # Khat_{j-1} Diag(d_j), off the chain
            Z = px["Khat"] @ x["W"].T                 # Khat_{j-1} W_j^T, 64 x 64, off the chain
            base = px["Aq"].T @ dOs[j - 1] + px["Khat"] @ (x["QG"].T @ dOs[j])
            dU_prev = base + Y @ dS - Z @ dU
        dS = x["d"][:, None] * dS + x["QG"].T @ dOs[j] - x["W"].T @ dU
        if j > 0:
            dU = dU_prev
    return dUs, dSend, dS
