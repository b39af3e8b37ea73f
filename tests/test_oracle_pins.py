"""Pins of the fp64 oracle to facts fixed by the pages and by the mathematics.

None of these re-type the oracle's loop: each checks it against a different
statement -- a hand-worked example, a closed form, an invariant the pages
prove (orthogonality, the planar rotation, non-expansiveness, the spectrum),
a dense-matrix formulation, or finite differences of the oracle itself.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(12345)


def rand_inputs(rng, T, H, dk, dv, *, sign_p=0.25, unit=True, beta_max=2.0, gscale=0.3):
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    if unit:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    beta = rng.uniform(0.0, beta_max, (T, H))
    g = -gscale * rng.exponential(1.0, (T, H, dk))
    sign = np.where(rng.random((T, H, dk)) < sign_p, -1, 1).astype(np.int8)
    return q, k, v, g, sign, beta


def transition(dk, g, sign, beta, k):
    """The dense transition of one token, read out of the oracle itself: the
    oracle's step applied to S_{t-1} = I with v = 0."""
    cu = np.array([0, 1])
    one = lambda x: np.asarray(x)[None, None]
    _, ST, _ = oracle.fwd(cu, one(np.zeros(dk)), one(k), one(np.zeros(dk)), one(g), one(sign),
                          np.array([[beta]]), S0=np.eye(dk)[None, None])
    return ST[0, 0]


# ---------------------------------------------------------------------------
# hand-worked examples
# ---------------------------------------------------------------------------

def test_worked_example_two_tokens():
    vals = {}
    with open(os.path.join(GOLDEN, "worked_example_2tok.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, val = line.split()
            vals[key] = float(val)
    q = np.array([[[1.0, 0.0]], [[0.0, 1.0]]])
    k = np.array([[[0.6, 0.8]], [[1.0, 0.0]]])
    v = np.array([[[0.5]], [[2.0]]])
    g = np.array([[[0.0, 0.0]], [[math.log(0.5), 0.0]]])
    sign = np.array([[[1, -1]], [[-1, 1]]], dtype=np.int8)
    beta = np.array([[2.0], [1.0]])
    S0 = np.array([1.0, 0.0]).reshape(1, 1, 2, 1)
    o, ST, _ = oracle.fwd([0, 2], q, k, v, g, sign, beta, S0=S0)
    assert o[0, 0, 0] == pytest.approx(vals["o1"], abs=1e-14)
    assert o[1, 0, 0] == pytest.approx(vals["o2"], abs=1e-14)
    assert ST[0, 0, 0, 0] == pytest.approx(vals["S2_0"], abs=1e-14)
    assert ST[0, 0, 1, 0] == pytest.approx(vals["S2_1"], abs=1e-14)


def test_rotation_2d_golden():
    rows = np.loadtxt(os.path.join(GOLDEN, "rotation_2d.txt"), comments="#")
    for phi_over_pi, a00, a01, a10, a11 in rows:
        phi = phi_over_pi * math.pi
        A = transition(2, [0.0, 0.0], [1, -1], 2.0, [math.cos(phi), math.sin(phi)])
        np.testing.assert_allclose(A, [[a00, a01], [a10, a11]], atol=1e-15)


def test_rotation_2d_angle_and_powers():
    """alpha = (1,-1), beta = 2: rotation by pi + 2 phi (det +1, eigenvalues
    exp(+-i theta)); n identical tokens rotate by n theta."""
    for phi in RNG.uniform(-math.pi, math.pi, 20):
        k = [math.cos(phi), math.sin(phi)]
        A = transition(2, [0.0, 0.0], [1, -1], 2.0, k)
        th = math.pi + 2 * phi
        R = np.array([[math.cos(th), -math.sin(th)], [math.sin(th), math.cos(th)]])
        np.testing.assert_allclose(A, R, atol=1e-14)
        assert np.linalg.det(A) == pytest.approx(1.0, abs=1e-14)
        ev = np.sort_complex(np.linalg.eigvals(A))
        np.testing.assert_allclose(ev, np.sort_complex(np.exp([1j * th, -1j * th])), atol=1e-12)
        n = 7
        T = n
        q = np.zeros((T, 1, 2))
        kk = np.tile(np.array(k), (T, 1, 1))
        v = np.zeros((T, 1, 2))
        g = np.zeros((T, 1, 2))
        sg = np.tile(np.array([1, -1], dtype=np.int8), (T, 1, 1))
        beta = np.full((T, 1), 2.0)
        _, ST, _ = oracle.fwd([0, T], q, kk, v, g, sg, beta, S0=np.eye(2)[None, None])
        Rn = np.array([[math.cos(n * th), -math.sin(n * th)], [math.sin(n * th), math.cos(n * th)]])
        np.testing.assert_allclose(ST[0, 0], Rn, atol=1e-12)


def test_rotation_direction_distinguishes_factor_order():
    """Diag(alpha) acts before the reflection: the reverse order would give
    the rotation by pi - 2 phi, which differs for generic phi."""
    phi = 0.3
    A = transition(2, [0.0, 0.0], [1, -1], 2.0, [math.cos(phi), math.sin(phi)])
    th_wrong = math.pi - 2 * phi
    Rw = np.array([[math.cos(th_wrong), -math.sin(th_wrong)], [math.sin(th_wrong), math.cos(th_wrong)]])
    assert np.abs(A - Rw).max() > 0.5


# ---------------------------------------------------------------------------
# invariants the pages state
# ---------------------------------------------------------------------------

def test_orthogonal_case_preserves_frobenius_norm():
    """|alpha| = 1, beta = 2, unit k, v = 0: every transition is orthogonal, so
    the state's Frobenius norm is preserved exactly over many steps."""
    T, H, dk, dv = 300, 3, 8, 5
    q, k, _, _, sign, _ = rand_inputs(RNG, T, H, dk, dv, sign_p=0.5)
    v = np.zeros((T, H, dv))
    g = np.zeros((T, H, dk))
    beta = np.full((T, H), 2.0)
    S0 = RNG.standard_normal((1, H, dk, dv))
    _, ST, cs = oracle.fwd([0, T], q, k, v, g, sign, beta, S0=S0, chunk=1)
    for h in range(H):
        n0 = np.linalg.norm(S0[0, h])
        assert np.linalg.norm(ST[0, h]) == pytest.approx(n0, rel=1e-12)
        norms = np.linalg.norm(cs[:, h].reshape(T, -1), axis=1)
        np.testing.assert_allclose(norms, n0, rtol=1e-12)


def test_transitions_orthogonal_at_extremes():
    for _ in range(50):
        dk = int(RNG.integers(2, 9))
        k = RNG.standard_normal(dk)
        k /= np.linalg.norm(k)
        sign = np.where(RNG.random(dk) < 0.5, -1, 1).astype(np.int8)
        A = transition(dk, np.zeros(dk), sign, 2.0, k)
        np.testing.assert_allclose(A.T @ A, np.eye(dk), atol=1e-14)


def test_non_expansive():
    """||A_t||_2 <= 1 for unit k, beta in [0, 2], |alpha| <= 1."""
    for _ in range(300):
        dk = int(RNG.integers(1, 10))
        k = RNG.standard_normal(dk)
        k /= np.linalg.norm(k)
        g = -RNG.exponential(0.5, dk) * (RNG.random(dk) < 0.7)
        sign = np.where(RNG.random(dk) < 0.4, -1, 1).astype(np.int8)
        beta = float(RNG.choice([0.0, 2.0, RNG.uniform(0, 2)]))
        A = transition(dk, g, sign, beta, k)
        assert np.linalg.svd(A, compute_uv=False)[0] <= 1.0 + 1e-12


def test_spectrum_structure():
    """At most one non-real conjugate pair; none when all gates are positive
    or beta <= 1 (section 3 "Diagonal Gate"; section 4, Theorem 8)."""
    n_complex_seen = 0
    for trial in range(400):
        dk = int(RNG.integers(2, 9))
        k = RNG.standard_normal(dk)
        k /= np.linalg.norm(k)
        g = -RNG.exponential(0.3, dk)
        mode = trial % 3
        if mode == 0:
            sign = np.ones(dk, dtype=np.int8)
            beta = RNG.uniform(0, 2)
        elif mode == 1:
            sign = np.where(RNG.random(dk) < 0.5, -1, 1).astype(np.int8)
            beta = RNG.uniform(0, 1)
        else:
            sign = np.where(RNG.random(dk) < 0.5, -1, 1).astype(np.int8)
            beta = RNG.uniform(1, 2)
        A = transition(dk, g, sign, beta, k)
        ev = np.linalg.eigvals(A)
        n_nonreal = int(np.sum(np.abs(ev.imag) > 1e-9))
        assert n_nonreal <= 2
        if mode in (0, 1):
            assert n_nonreal == 0, (mode, ev)
        n_complex_seen += n_nonreal > 0
    assert n_complex_seen > 10  # the signed, beta > 1 regime does reach complex pairs


def test_scalar_gate_symmetric_and_factors_out():
    """Scalar gate: each transition is symmetric, and over steps the gates
    factor out of the product (section 3 "Scalar Gate")."""
    T, dk = 12, 5
    k = RNG.standard_normal((T, 1, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    beta = RNG.uniform(0, 2, (T, 1))
    a_mag = -RNG.exponential(0.2, T)
    a_sign = np.where(RNG.random(T) < 0.5, -1, 1)
    g = np.repeat(a_mag[:, None, None], dk, axis=2)
    sign = np.repeat(a_sign[:, None, None], dk, axis=2).astype(np.int8)
    for t in range(T):
        A = transition(dk, g[t, 0], sign[t, 0], beta[t, 0], k[t, 0])
        np.testing.assert_allclose(A, A.T, atol=1e-14)
    zeros = np.zeros((T, 1, dk))
    _, ST, _ = oracle.fwd([0, T], zeros, k, zeros, g, sign, beta, S0=np.eye(dk)[None, None])
    _, ST1, _ = oracle.fwd([0, T], zeros, k, zeros, np.zeros_like(g), np.ones_like(sign), beta,
                           S0=np.eye(dk)[None, None])
    scale = np.prod(a_sign * np.exp(a_mag))
    np.testing.assert_allclose(ST[0, 0], scale * ST1[0, 0], atol=1e-14)


# ---------------------------------------------------------------------------
# the sign trick of the model card
# ---------------------------------------------------------------------------

def test_sign_folding_identity_bitwise():
    """Signed recurrence == unsigned recurrence on k' = P k, q' = P q, with
    P_t the running product of signs; S_T = Diag(P_T) S'_T.  Exact in fp64."""
    T, H, dk, dv = 97, 2, 6, 4
    q, k, v, g, sign, beta = rand_inputs(RNG, T, H, dk, dv)
    S0 = RNG.standard_normal((1, H, dk, dv))
    o, ST, _ = oracle.fwd([0, T], q, k, v, g, sign, beta, S0=S0)
    P = np.cumprod(sign.astype(np.float64), axis=0)
    o2, ST2, _ = oracle.fwd([0, T], P * q, P * k, v, g, np.ones_like(sign), beta, S0=S0)
    assert np.array_equal(o, o2)
    assert np.array_equal(ST[0], P[-1][:, :, None] * ST2[0])


# ---------------------------------------------------------------------------
# closed forms and brute force
# ---------------------------------------------------------------------------

def test_dense_brute_force_products():
    """S_T = (A_T..A_1) S_0 + sum_t (A_T..A_{t+1}) beta_t k_t v_t^T with the
    explicit dense A_t = (I - beta k k^T) Diag(alpha), and o_t = S_t^T q_t."""
    for T in (1, 2, 5, 16):
        dk, dv, H = 5, 3, 2
        q, k, v, g, sign, beta = rand_inputs(RNG, T, H, dk, dv, unit=False)
        S0 = RNG.standard_normal((1, H, dk, dv))
        o, ST, _ = oracle.fwd([0, T], q, k, v, g, sign, beta, S0=S0)
        for h in range(H):
            A = [(np.eye(dk) - beta[t, h] * np.outer(k[t, h], k[t, h]))
                 @ np.diag(sign[t, h] * np.exp(g[t, h])) for t in range(T)]
            for tt in range(1, T + 1):
                prod = np.eye(dk)
                for t in range(tt):
                    prod = A[t] @ prod
                S = prod @ S0[0, h]
                for s in range(tt):
                    P = np.eye(dk)
                    for t in range(s + 1, tt):
                        P = A[t] @ P
                    S = S + P @ (beta[s, h] * np.outer(k[s, h], v[s, h]))
                np.testing.assert_allclose(o[tt - 1, h], S.T @ q[tt - 1, h], atol=1e-12)
            np.testing.assert_allclose(ST[0, h], S, atol=1e-12)


def test_first_token_from_zero_state():
    """From S_0 = 0: S_1 = beta k v^T, o_1 = beta (k.q) v (the update is read
    after it is applied)."""
    q, k, v, g, sign, beta = rand_inputs(RNG, 1, 4, 7, 3)
    o, ST, _ = oracle.fwd([0, 1], q, k, v, g, sign, beta)
    for h in range(4):
        np.testing.assert_allclose(ST[0, h], beta[0, h] * np.outer(k[0, h], v[0, h]), atol=1e-15)
        np.testing.assert_allclose(o[0, h], beta[0, h] * (k[0, h] @ q[0, h]) * v[0, h], atol=1e-15)


def test_scalar_key_closed_form():
    """dk = 1: S_t = (1 - beta k^2) alpha S_{t-1} + beta k v_t."""
    T, dv = 40, 3
    q, k, v, g, sign, beta = rand_inputs(RNG, T, 1, 1, dv, unit=False)
    S0 = RNG.standard_normal((1, 1, 1, dv))
    o, ST, _ = oracle.fwd([0, T], q, k, v, g, sign, beta, S0=S0)
    S = S0[0, 0, 0].copy()
    for t in range(T):
        a = sign[t, 0, 0] * math.exp(g[t, 0, 0])
        kk = k[t, 0, 0]
        S = (1 - beta[t, 0] * kk * kk) * a * S + beta[t, 0] * kk * v[t, 0]
        np.testing.assert_allclose(o[t, 0], S * q[t, 0, 0], atol=1e-12)
    np.testing.assert_allclose(ST[0, 0, 0], S, atol=1e-12)


def test_beta_zero_is_pure_signed_decay():
    T, H, dk, dv = 30, 2, 6, 4
    q, k, v, g, sign, _ = rand_inputs(RNG, T, H, dk, dv)
    beta = np.zeros((T, H))
    S0 = RNG.standard_normal((1, H, dk, dv))
    o, ST, _ = oracle.fwd([0, T], q, k, v, g, sign, beta, S0=S0)
    alpha = sign * np.exp(g)
    cum = np.cumprod(alpha, axis=0)
    for t in range(T):
        St = cum[t][:, :, None] * S0[0]
        np.testing.assert_allclose(o[t], np.einsum("hij,hi->hj", St, q[t]), atol=1e-13)
    np.testing.assert_allclose(ST[0], cum[-1][:, :, None] * S0[0], atol=1e-13)


def test_unit_gate_is_deltanet_and_positive_gate_is_kda():
    """g = 0, sign = +1: plain DeltaNet S_t = S - beta k (k^T S - v^T)."""
    T, H, dk, dv = 25, 1, 4, 3
    q, k, v, _, _, beta = rand_inputs(RNG, T, H, dk, dv)
    g = np.zeros((T, H, dk))
    sign = np.ones((T, H, dk), dtype=np.int8)
    o, ST, _ = oracle.fwd([0, T], q, k, v, g, sign, beta)
    S = np.zeros((dk, dv))
    for t in range(T):
        kt, vt = k[t, 0], v[t, 0]
        S = S - beta[t, 0] * np.outer(kt, kt @ S - vt)
        np.testing.assert_allclose(o[t, 0], S.T @ q[t, 0], atol=1e-13)


# ---------------------------------------------------------------------------
# packing, continuation and decode
# ---------------------------------------------------------------------------

def test_packed_sequences_reset_state():
    lens = [5, 1, 17, 64, 65, 3]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, dk, dv = int(cu[-1]), 2, 5, 4
    q, k, v, g, sign, beta = rand_inputs(RNG, T, H, dk, dv)
    S0 = RNG.standard_normal((len(lens), H, dk, dv))
    o, ST, cs = oracle.fwd(cu, q, k, v, g, sign, beta, S0=S0, chunk=16)
    c = 0
    for i, L in enumerate(lens):
        a, b = cu[i], cu[i + 1]
        oi, STi, csi = oracle.fwd([0, L], q[a:b], k[a:b], v[a:b], g[a:b], sign[a:b], beta[a:b],
                                 S0=S0[i:i + 1], chunk=16)
        np.testing.assert_array_equal(o[a:b], oi)
        np.testing.assert_array_equal(ST[i], STi[0])
        np.testing.assert_array_equal(cs[c:c + len(csi)], csi)
        c += len(csi)
    assert c == len(cs)


def test_chunk_states_are_prefix_final_states():
    """chunk_states[c] is the state before token j*chunk of its sequence: the
    final state of the forward over that sequence's first j*chunk tokens (the
    initial state itself for j = 0), at the global chunk index that counts the
    earlier sequences' ceil(len / chunk) chunks first."""
    lens = [37, 16, 1, 50]
    cu = np.concatenate([[0], np.cumsum(lens)])
    H, dk, dv, chunk = 2, 4, 3, 16
    q, k, v, g, sign, beta = rand_inputs(RNG, int(cu[-1]), H, dk, dv)
    S0 = RNG.standard_normal((len(lens), H, dk, dv))
    _, _, cs = oracle.fwd(cu, q, k, v, g, sign, beta, S0=S0, chunk=chunk)
    c = 0
    for i, L in enumerate(lens):
        a = cu[i]
        for j in range((L + chunk - 1) // chunk):
            n = j * chunk
            if n == 0:
                want = S0[i]
            else:
                sl = slice(a, a + n)
                _, want, _ = oracle.fwd([0, n], q[sl], k[sl], v[sl], g[sl], sign[sl], beta[sl],
                                        S0=S0[i:i + 1])
                want = want[0]
            np.testing.assert_array_equal(cs[c], want)
            c += 1
    assert c == len(cs)


def test_state_continuation():
    T1, T2, H, dk, dv = 37, 50, 2, 4, 6
    q, k, v, g, sign, beta = rand_inputs(RNG, T1 + T2, H, dk, dv)
    S0 = RNG.standard_normal((1, H, dk, dv))
    o, ST, _ = oracle.fwd([0, T1 + T2], q, k, v, g, sign, beta, S0=S0)
    o1, S1, _ = oracle.fwd([0, T1], q[:T1], k[:T1], v[:T1], g[:T1], sign[:T1], beta[:T1], S0=S0)
    o2, S2, _ = oracle.fwd([0, T2], q[T1:], k[T1:], v[T1:], g[T1:], sign[T1:], beta[T1:], S0=S1)
    np.testing.assert_array_equal(o, np.concatenate([o1, o2]))
    np.testing.assert_array_equal(ST, S2)


def test_decode_steps_equal_forward():
    T, N, H, dk, dv = 9, 3, 2, 5, 4
    q, k, v, g, sign, beta = rand_inputs(RNG, T * N, H, dk, dv)
    shp = lambda x: x.reshape(N, T, *x.shape[1:])
    q, k, v, g, sign, beta = map(shp, (q, k, v, g, sign, beta))
    S0 = RNG.standard_normal((N, H, dk, dv))
    flat = lambda x: x.reshape(N * T, *x.shape[2:])
    o, ST, _ = oracle.fwd(np.arange(N + 1) * T, flat(q), flat(k), flat(v), flat(g), flat(sign),
                          flat(beta), S0=S0)
    o = o.reshape(N, T, H, dv)
    st = S0.copy()
    for t in range(T):
        ot, st = oracle.decode(q[:, t], k[:, t], v[:, t], g[:, t], sign[:, t], beta[:, t], st)
        np.testing.assert_array_equal(ot, o[:, t])
    np.testing.assert_array_equal(st, ST)


def test_decode_multi_equals_forward_per_sequence():
    """Several steps per sequence from pooled, permuted slots with ragged step
    counts: each sequence's outputs and final state are the token forward's
    over its first n_tokens tokens from its slot's state (state
    continuation), untouched slots stay bitwise, skipped sequences give zeros."""
    N, K, H, dk, dv, n_slots = 5, 4, 2, 5, 3, 8
    q, k, v, g, sign, beta = rand_inputs(RNG, N * K, H, dk, dv)
    shp = lambda x: x.reshape(N, K, *x.shape[1:])
    q, k, v, g, sign, beta = map(shp, (q, k, v, g, sign, beta))
    pool = RNG.standard_normal((n_slots, H, dk, dv))
    slots = np.array([6, 1, -1, 3, 8])      # -1 and 8 (= n_slots) are skipped
    n_tok = np.array([4, 0, 2, 9, 1])       # 9 is clamped to K
    o, new = oracle.decode_multi(q, k, v, g, sign, beta, pool, n_tokens=n_tok, slots=slots)
    for n in range(N):
        s = slots[n]
        if not 0 <= s < n_slots:
            assert np.all(o[n] == 0)
            continue
        L = min(int(n_tok[n]), K)
        if L:
            on, Sn, _ = oracle.fwd([0, L], q[n, :L], k[n, :L], v[n, :L], g[n, :L], sign[n, :L], beta[n, :L],
                                   S0=pool[s:s + 1])
            np.testing.assert_array_equal(o[n, :L], on)
            np.testing.assert_array_equal(new[s], Sn[0])
        else:
            np.testing.assert_array_equal(new[s], pool[s])
        assert np.all(o[n, L:] == 0)
    for s in set(range(n_slots)) - {6, 1, 3}:
        np.testing.assert_array_equal(new[s], pool[s])
    # verify (no write-back): same outputs, pool unchanged
    o2, same = oracle.decode_multi(q, k, v, g, sign, beta, pool, n_tokens=n_tok, slots=slots,
                                   write_state=False)
    np.testing.assert_array_equal(o2, o)
    np.testing.assert_array_equal(same, pool)


def test_decode_multi_commit_after_verify():
    """Speculative decoding: verifying K draft tokens and then committing the
    first a of them leaves the state the forward over those a tokens gives."""
    N, K, H, dk, dv = 3, 5, 1, 4, 4
    q, k, v, g, sign, beta = rand_inputs(RNG, N * K, H, dk, dv)
    shp = lambda x: x.reshape(N, K, *x.shape[1:])
    q, k, v, g, sign, beta = map(shp, (q, k, v, g, sign, beta))
    pool = RNG.standard_normal((N, H, dk, dv))
    o_ver, _ = oracle.decode_multi(q, k, v, g, sign, beta, pool, write_state=False)
    acc = np.array([2, 5, 0])
    o_com, new = oracle.decode_multi(q, k, v, g, sign, beta, pool, n_tokens=acc)
    for n in range(N):
        np.testing.assert_array_equal(o_com[n, :acc[n]], o_ver[n, :acc[n]])
        ref = pool[n:n + 1]
        if acc[n]:
            _, ref, _ = oracle.fwd([0, acc[n]], q[n, :acc[n]], k[n, :acc[n]], v[n, :acc[n]], g[n, :acc[n]],
                                   sign[n, :acc[n]], beta[n, :acc[n]], S0=pool[n:n + 1])
        np.testing.assert_array_equal(new[n], ref[0])


# ---------------------------------------------------------------------------
# gradients against central finite differences of the oracle's forward
# ---------------------------------------------------------------------------

def _loss(cu, inp, dO, dST):
    o, ST, _ = oracle.fwd(cu, inp["q"], inp["k"], inp["v"], inp["g"], inp["sign"], inp["beta"],
                          S0=inp["S0"])
    return float(np.sum(o * dO) + np.sum(ST * dST))


def _fd_check(cu, inp, dO, dST, grads, names, eps=1e-6, exhaustive=True, ndir=6, rtol=1e-6):
    for name in names:
        x = inp[name]
        gname = "d" + name
        if exhaustive:
            fd = np.zeros_like(x)
            it = np.nditer(x, flags=["multi_index"])
            for _ in it:
                idx = it.multi_index
                old = x[idx]
                x[idx] = old + eps
                lp = _loss(cu, inp, dO, dST)
                x[idx] = old - eps
                lm = _loss(cu, inp, dO, dST)
                x[idx] = old
                fd[idx] = (lp - lm) / (2 * eps)
            scale = max(1.0, np.abs(fd).max())
            np.testing.assert_allclose(grads[gname], fd, atol=rtol * scale * 10, rtol=0,
                                       err_msg=name)
        else:
            for _ in range(ndir):
                d = RNG.standard_normal(x.shape)
                x0 = x.copy()
                inp[name] = x0 + eps * d
                lp = _loss(cu, inp, dO, dST)
                inp[name] = x0 - eps * d
                lm = _loss(cu, inp, dO, dST)
                inp[name] = x0
                fd = (lp - lm) / (2 * eps)
                an = float(np.sum(grads[gname] * d))
                assert an == pytest.approx(fd, rel=rtol, abs=rtol * 1e-2), name


def test_gradients_exhaustive_finite_differences():
    lens = [3, 5]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, dk, dv = int(cu[-1]), 1, 3, 2
    q, k, v, g, sign, beta = rand_inputs(RNG, T, H, dk, dv, unit=False)
    inp = dict(q=q, k=k, v=v, g=g, sign=sign, beta=beta,
               S0=RNG.standard_normal((len(lens), H, dk, dv)))
    dO = RNG.standard_normal((T, H, dv))
    dST = RNG.standard_normal((len(lens), H, dk, dv))
    gr = oracle.bwd(cu, q, k, v, g, sign, beta, dO, S0=inp["S0"], dST=dST)
    _fd_check(cu, inp, dO, dST, gr, ["q", "k", "v", "g", "beta", "S0"])


def test_gradients_directional_across_checkpoints():
    """Sequences longer than the oracle's 64-token checkpoint interval."""
    lens = [150, 64, 1]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, dk, dv = int(cu[-1]), 2, 8, 8
    q, k, v, g, sign, beta = rand_inputs(RNG, T, H, dk, dv)
    inp = dict(q=q, k=k, v=v, g=g, sign=sign, beta=beta,
               S0=RNG.standard_normal((len(lens), H, dk, dv)))
    dO = RNG.standard_normal((T, H, dv))
    dST = RNG.standard_normal((len(lens), H, dk, dv))
    gr = oracle.bwd(cu, q, k, v, g, sign, beta, dO, S0=inp["S0"], dST=dST)
    _fd_check(cu, inp, dO, dST, gr, ["q", "k", "v", "g", "beta", "S0"], exhaustive=False,
              ndir=4, rtol=1e-6)


def test_gradient_without_upstream_state_grad():
    T, H, dk, dv = 20, 1, 4, 3
    q, k, v, g, sign, beta = rand_inputs(RNG, T, H, dk, dv)
    inp = dict(q=q, k=k, v=v, g=g, sign=sign, beta=beta, S0=None)
    dO = RNG.standard_normal((T, H, dv))
    gr = oracle.bwd([0, T], q, k, v, g, sign, beta, dO)
    _fd_check([0, T], inp, dO, np.zeros((1, H, dk, dv)), gr, ["k", "g"], exhaustive=False, ndir=4)
