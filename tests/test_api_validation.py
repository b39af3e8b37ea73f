"""The tensor-level API checks shapes and dtypes before anything reaches the
library (which reads exactly the bytes the sizes imply), and refuses host
tensors.  Runs on CPU: every call here stops before a launch."""
import pytest
import torch

from chunked_gated_delta_ckda_b200 import api


def _inputs(lead, H=2, dk=64, dv=64, io=torch.bfloat16):
    z = lambda *s, dt=io: torch.zeros(*lead, *s, dtype=dt)
    return dict(q=z(H, dk), k=z(H, dk), v=z(H, dv), g=z(H, dk, dt=torch.float32), sign=z(H, dk, dt=torch.int8),
                beta=z(H))


def _call_fwd(x, **kw):
    return api.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["sign"], x["beta"], **kw)


def test_well_formed_host_tensors_are_refused_as_host_tensors():
    with pytest.raises(ValueError, match="CUDA"):
        _call_fwd(_inputs((1, 8)))


@pytest.mark.parametrize("name,bad", [("k", lambda t: t[..., :32]), ("v", lambda t: t[:, :4]),
                                      ("beta", lambda t: t[..., :1]), ("sign", lambda t: t[..., :7])])
def test_shape_mismatch(name, bad):
    x = _inputs((1, 8))
    x[name] = bad(x[name]).contiguous()
    with pytest.raises(ValueError, match=name):
        _call_fwd(x)


@pytest.mark.parametrize("name,dt", [("g", torch.bfloat16), ("sign", torch.float32), ("k", torch.float32),
                                     ("beta", torch.float32)])
def test_dtype_mismatch(name, dt):
    x = _inputs((1, 8))
    x[name] = x[name].to(dt)
    with pytest.raises(TypeError, match=name):
        _call_fwd(x)


def test_state_shapes_checked():
    x = _inputs((1, 8))
    with pytest.raises(ValueError, match="S0"):
        _call_fwd(x, S0=torch.zeros(1, 2, 64, 32))
    d = _inputs((3,))
    with pytest.raises(ValueError, match="state"):
        api.decode_step(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], torch.zeros(3, 2, 64, 32))
    with pytest.raises(ValueError, match="CUDA"):  # right shapes, host memory
        api.decode_step(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], torch.zeros(3, 2, 64, 64))


def test_decode_multi_arguments_checked():
    m = _inputs((4, 3))
    args = (m["q"], m["k"], m["v"], m["g"], m["sign"], m["beta"])
    with pytest.raises(ValueError, match="pool"):
        api.decode_multi(*args, torch.zeros(5, 2, 64, 128))
    with pytest.raises(TypeError, match="slots"):
        api.decode_multi(*args, torch.zeros(5, 2, 64, 64), slots=torch.zeros(4, dtype=torch.int64))
    with pytest.raises(ValueError, match="n_tokens"):
        api.decode_multi(*args, torch.zeros(5, 2, 64, 64), n_tokens=torch.zeros(3, dtype=torch.int32))


def test_prologue_arguments_checked():
    B, T, H, d = 1, 8, 2, 64
    z = lambda *s, dt=torch.bfloat16: torch.zeros(*s, dtype=dt)
    x = dict(xq=z(B, T, H, d), xk=z(B, T, H, d), xv=z(B, T, H, d), wq=z(H * d, 4, dt=torch.float32),
             wk=z(H * d, 4, dt=torch.float32), wv=z(H * d, 4, dt=torch.float32), a=z(B, T, H, d, dt=torch.float32),
             b=z(B, T, H))
    bad = dict(x, wq=z(H * d, 3, dt=torch.float32))
    with pytest.raises(ValueError, match="wq"):
        api.prologue_fwd(**bad)
    bad = dict(x, a=z(B, T, H, d))
    with pytest.raises(TypeError, match="a must"):
        api.prologue_fwd(**bad)
    with pytest.raises(ValueError, match="CUDA"):
        api.prologue_fwd(**x)


def test_tensors_on_two_devices_are_refused():
    """A pointer into another GPU's memory must never reach the kernels: the
    calls refuse CUDA tensors on more than one device before anything else
    (stand-ins for tensors on cuda:0 and cuda:1; no GPU is touched)."""
    from types import SimpleNamespace
    on = lambda i: SimpleNamespace(is_cuda=True, device=torch.device("cuda", i))
    assert api._cuda_devices((on(0), None, 3, torch.zeros(1)), {"S0": on(0)}) == {torch.device("cuda", 0)}
    assert len(api._cuda_devices((on(0),), {"S0": on(1)})) == 2
    seen = []
    guarded = api._one_device(lambda *a, **k: seen.append(1))
    with pytest.raises(ValueError, match="one CUDA device"):
        guarded(on(0), on(1))
    with pytest.raises(ValueError, match="one CUDA device"):
        guarded(on(0), ws=on(1))
    guarded(torch.zeros(1), None)  # host tensors only: passed through (the argument checks refuse them)
    assert seen == [1]
    for fn in (api.chunk_fwd, api.chunk_bwd, api.decode_step, api.decode_multi, api.varlen_fwd, api.varlen_bwd,
               api.prologue_fwd, api.prologue_bwd):
        assert getattr(fn, "__wrapped__", None) is not None, fn.__name__
