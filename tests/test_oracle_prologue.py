"""Pins of the prologue oracle (oracle/prologue.py) to facts outside itself:
numpy's convolution, unit norms, the gate's closed forms, and central
finite differences for its gradients."""
import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(2024)


def _inputs(B, T, H, dk, dv, rng=RNG, ascale=1.5):
    return dict(
        xq=rng.standard_normal((B, T, H, dk)), xk=rng.standard_normal((B, T, H, dk)),
        xv=rng.standard_normal((B, T, H, dv)),
        wq=0.5 * rng.standard_normal((H * dk, 4)), wk=0.5 * rng.standard_normal((H * dk, 4)),
        wv=0.5 * rng.standard_normal((H * dv, 4)),
        a=ascale * rng.standard_normal((B, T, H, dk)), b=2.0 * rng.standard_normal((B, T, H)))


def _silu(y):
    return y / (1.0 + np.exp(-y))


def _np_conv(x, w):
    """numpy reference: per sequence and channel, np.convolve with the taps
    reversed (tap 3 on the current token), cut to the causal part."""
    B, T, H, d = x.shape
    out = np.zeros_like(x)
    for b in range(B):
        for h in range(H):
            for c in range(d):
                out[b, :, h, c] = np.convolve(x[b, :, h, c], w[h * d + c, ::-1])[:T]
    return out


def test_short_conv_silu_matches_numpy_convolve():
    x = _inputs(2, 11, 2, 5, 3)
    r = oracle.prologue_fwd(**x)
    np.testing.assert_allclose(r["v"], _silu(_np_conv(x["xv"], x["wv"])), rtol=1e-13, atol=1e-14)
    for name in ("q", "k"):
        n = _silu(_np_conv(x["x" + name], x["w" + name]))
        scale = np.sqrt((n * n).sum(-1, keepdims=True) + 1e-6)
        np.testing.assert_allclose(r[name] * scale, n, rtol=1e-12, atol=1e-14)
        norms = np.linalg.norm(r[name], axis=-1)
        big = (n * n).sum(-1) > 1.0
        np.testing.assert_allclose(norms[big], 1.0, atol=1e-6)


def test_conv_restarts_at_each_sequence():
    """Each batch row is its own sequence: its first outputs see no history."""
    x = _inputs(2, 9, 1, 4, 4)
    r = oracle.prologue_fwd(**x)
    solo = oracle.prologue_fwd(**{k: (v[1:2] if v.ndim >= 3 else v) for k, v in x.items()})
    for name in ("q", "k", "v"):  # (reductions may be ordered differently for another batch size)
        np.testing.assert_allclose(r[name][1:2], solo[name], rtol=1e-14, atol=1e-15)


def test_single_tap_reduces_to_pointwise():
    """Only the current-token tap set: no mixing over time, v = silu(w3 x)."""
    x = _inputs(1, 7, 2, 3, 4)
    x["wv"][:, :3] = 0.0
    r = oracle.prologue_fwd(**x)
    np.testing.assert_allclose(r["v"], _silu(x["xv"] * x["wv"][:, 3].reshape(2, 4)), rtol=1e-13)


def test_signed_gate_closed_forms():
    x = _inputs(1, 6, 2, 4, 4)
    a = x["a"]
    a[0, 0, 0, :] = [0.0, 1e-30, -40.0, 40.0]   # zero, underflowing magnitude, saturated
    floor = -5.0
    r = oracle.prologue_fwd(**x, g_floor=floor)
    alpha = np.tanh(a)
    with np.errstate(divide="ignore"):
        keep = np.log(np.abs(alpha)) >= floor
    np.testing.assert_allclose((r["sign"] * np.exp(r["g"]))[keep], alpha[keep], rtol=1e-13)
    assert np.all(r["g"][~keep] == floor)
    assert np.all(r["sign"] == np.where(alpha < 0, -1, 1))
    assert r["sign"][0, 0, 0, 0] == 1 and r["g"][0, 0, 0, 0] == floor          # alpha = 0
    assert r["g"][0, 0, 0, 2] == 0.0 and r["sign"][0, 0, 0, 2] == -1            # tanh(-40) = -1
    assert np.all(r["g"] <= 0.0)
    # beta = 2 sigmoid(b): 1 at b = 0, in (0, 2), symmetric: beta(b) + beta(-b) = 2
    b = x["b"]
    b[0, 0, 0] = 0.0
    r = oracle.prologue_fwd(**x)
    assert r["beta"][0, 0, 0] == 1.0
    neg = oracle.prologue_fwd(**{**x, "b": -b})
    np.testing.assert_allclose(r["beta"] + neg["beta"], 2.0, rtol=1e-14)
    assert np.all((r["beta"] > 0) & (r["beta"] < 2))


@pytest.mark.parametrize("g_floor", [-np.inf, -1.0])
def test_gradients_central_differences(g_floor):
    """Every input's gradient against central differences of the forward's
    weighted sum, exhaustively on a tiny case (T spans the conv window, two
    sequences); at g_floor = -1 about a third of the gate entries are clamped
    and must get zero gradient."""
    rng = np.random.default_rng(7)
    x = _inputs(2, 6, 2, 3, 2, rng=rng, ascale=1.0)
    up = dict(dq=rng.standard_normal((2, 6, 2, 3)), dk=rng.standard_normal((2, 6, 2, 3)),
              dv=rng.standard_normal((2, 6, 2, 2)), dg=rng.standard_normal((2, 6, 2, 3)),
              dbeta=rng.standard_normal((2, 6, 2)))

    def loss(inp):
        r = oracle.prologue_fwd(**inp, g_floor=g_floor)
        return sum(float(np.sum(r[n] * up["d" + n])) for n in ("q", "k", "v", "g", "beta"))

    grads = oracle.prologue_bwd(**x, **up, g_floor=g_floor)
    eps = 1e-6
    for name in ("xq", "xk", "xv", "wq", "wk", "wv", "a", "b"):
        gr = grads["d" + name]
        assert gr.shape == x[name].shape
        fd = np.zeros_like(gr)
        for idx in np.ndindex(x[name].shape):
            xp = {k: v.copy() for k, v in x.items()}
            xm = {k: v.copy() for k, v in x.items()}
            xp[name][idx] += eps
            xm[name][idx] -= eps
            fd[idx] = (loss(xp) - loss(xm)) / (2 * eps)
        np.testing.assert_allclose(gr, fd, rtol=1e-5, atol=1e-7, err_msg=name)
    if np.isfinite(g_floor):
        clamped = np.log(np.abs(np.tanh(x["a"]))) < g_floor
        assert clamped.sum() > 3
        assert np.all(grads["da"][clamped] == 0.0)


def test_packed_documents_equal_batch_rows():
    """Three documents of equal length packed in one row give what three
    batch rows give: outputs, input gradients, and the taps' gradients (sums
    over every token either way)."""
    rng = np.random.default_rng(11)
    x = _inputs(3, 5, 2, 3, 2, rng=rng)
    up = dict(dq=rng.standard_normal((3, 5, 2, 3)), dk=rng.standard_normal((3, 5, 2, 3)),
              dv=rng.standard_normal((3, 5, 2, 2)), dg=rng.standard_normal((3, 5, 2, 3)),
              dbeta=rng.standard_normal((3, 5, 2)))
    row = lambda v: v.reshape((1, -1) + v.shape[2:])
    px = {k: (row(v) if k[0] != "w" else v) for k, v in x.items()}
    pu = {k: row(v) for k, v in up.items()}
    cu = [0, 5, 10, 15]
    r, pr = oracle.prologue_fwd(**x), oracle.prologue_fwd(**px, cu_seqlens=cu)
    for n in ("q", "k", "v", "g", "beta", "sign"):
        np.testing.assert_allclose(pr[n], row(r[n]), rtol=1e-14, atol=1e-15, err_msg=n)
    g, pg = oracle.prologue_bwd(**x, **up), oracle.prologue_bwd(**px, **pu, cu_seqlens=cu)
    for n in ("dxq", "dxk", "dxv", "da", "db"):
        np.testing.assert_allclose(pg[n], row(g[n]), rtol=1e-13, atol=1e-14, err_msg=n)
    for n in ("dwq", "dwk", "dwv"):
        np.testing.assert_allclose(pg[n], g[n], rtol=1e-12, atol=1e-13, err_msg=n)


def test_packed_ragged_documents_match_numpy_convolve():
    """Ragged documents (one shorter than the window, one empty): numpy's
    convolution restarted at each document start."""
    rng = np.random.default_rng(12)
    cu = [0, 2, 2, 9, 13]
    x = _inputs(1, 13, 2, 3, 4, rng=rng)
    r = oracle.prologue_fwd(**x, cu_seqlens=cu)
    want = np.concatenate([_np_conv(x["xv"][:, s:e], x["wv"]) for s, e in zip(cu, cu[1:]) if e > s], axis=1)
    np.testing.assert_allclose(r["v"], _silu(want), rtol=1e-13, atol=1e-14)
    with pytest.raises(ValueError):
        oracle.prologue_fwd(**x, cu_seqlens=[0, 5, 4, 13])
    with pytest.raises(ValueError):
        oracle.prologue_fwd(**x, cu_seqlens=[0, 12])


def test_packed_gradients_central_differences():
    """Input and tap gradients of a packed row (a two-token document, an
    empty one, a five-token one) against central differences."""
    rng = np.random.default_rng(13)
    cu = [0, 2, 2, 7]
    x = _inputs(1, 7, 1, 2, 2, rng=rng, ascale=1.0)
    up = dict(dq=rng.standard_normal((1, 7, 1, 2)), dk=rng.standard_normal((1, 7, 1, 2)),
              dv=rng.standard_normal((1, 7, 1, 2)), dg=rng.standard_normal((1, 7, 1, 2)),
              dbeta=rng.standard_normal((1, 7, 1)))

    def loss(inp):
        r = oracle.prologue_fwd(**inp, cu_seqlens=cu)
        return sum(float(np.sum(r[n] * up["d" + n])) for n in ("q", "k", "v", "g", "beta"))

    grads = oracle.prologue_bwd(**x, **up, cu_seqlens=cu)
    eps = 1e-6
    for name in ("xq", "xk", "xv", "wq", "wk", "wv"):
        gr = grads["d" + name]
        fd = np.zeros_like(gr)
        for idx in np.ndindex(x[name].shape):
            xp = {k: v.copy() for k, v in x.items()}
            xm = {k: v.copy() for k, v in x.items()}
            xp[name][idx] += eps
            xm[name][idx] -= eps
            fd[idx] = (loss(xp) - loss(xm)) / (2 * eps)
        np.testing.assert_allclose(gr, fd, rtol=1e-5, atol=1e-7, err_msg=name)
