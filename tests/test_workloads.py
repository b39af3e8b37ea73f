"""The seeded generators: shapes, dtypes, ranges, determinism and the packed
document-length recipe."""
import torch

from chunked_gated_delta_ckda_b200 import workloads as W


def test_tiny_shapes_and_ranges():
    x = W.make(W.TINY)
    assert x["q"].shape == (1, 256, 2, 64) and x["q"].dtype == torch.float32
    assert torch.allclose(x["q"].norm(dim=-1), torch.ones(1, 256, 2), atol=1e-5)
    assert torch.allclose(x["k"].norm(dim=-1), torch.ones(1, 256, 2), atol=1e-5)
    assert (x["beta"] >= 0).all() and (x["beta"] <= 2).all()
    assert (x["g"] <= 0).all()
    assert set(x["sign"].unique().tolist()) <= {-1, 1}
    frac_neg = (x["sign"] == -1).float().mean().item()
    assert 0.2 < frac_neg < 0.3
    assert x["S0"] is None


def test_deterministic():
    a = W.make(W.LAYER_FWD, B=1, T=64, H=2)
    b = W.make(W.LAYER_FWD, B=1, T=64, H=2)
    for key in ("q", "k", "v", "g", "sign", "beta"):
        assert torch.equal(a[key], b[key])


def test_layer_floor_and_extremes():
    x = W.make(W.LAYER_FWDBWD, B=2, T=512, H=4)
    assert x["q"].dtype == torch.bfloat16 and x["g"].dtype == torch.float32
    assert (x["g"] >= -5).all()
    ext = (x["g"] == 0).all(dim=-1) & (x["beta"].float() == 2.0)
    frac = ext.float().mean().item()
    assert 0.02 < frac < 0.09
    assert x["dO"] is not None and x["dO"].shape == (2, 512, 4, 128)


def test_doc_lengths_recipe():
    gen = torch.Generator().manual_seed(3)
    lens = W.doc_lengths(65536, 1500.0, 16, 4096, gen)
    assert sum(lens) == 65536
    assert all(16 <= L <= 4096 for L in lens)
    assert 25 <= len(lens) <= 80
    x = W.make_varlen(W.VARLEN, total=4096, H=2)
    assert int(x["cu_seqlens"][-1]) == 4096 == x["q"].shape[1]
    assert x["cu_seqlens"].dtype == torch.int32


def test_decode_steps_independent():
    a = W.make_decode_step(W.DECODE, step=3, N=4, H=2)
    b = W.make_decode_step(W.DECODE, step=3, N=4, H=2)
    c = W.make_decode_step(W.DECODE, step=4, N=4, H=2)
    assert torch.equal(a["q"], b["q"]) and not torch.equal(a["q"], c["q"])


def test_decode_multi_slots_are_distinct_and_in_pool():
    w = W.DECODE_MULTI
    x = W.make_decode_multi(w, call=2)
    assert x["q"].shape == (w.B, w.T, w.H, w.dk) and x["beta"].shape == (w.B, w.T, w.H)
    s = x["slots"]
    assert s.dtype == torch.int32 and len(set(s.tolist())) == w.B
    assert int(s.min()) >= 0 and int(s.max()) < w.extra["n_slots"]
    assert torch.equal(s, W.make_decode_multi(w, call=3)["slots"])   # placement fixed across calls
