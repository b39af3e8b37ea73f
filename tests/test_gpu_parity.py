"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Small cases span several chunks and a ragged tail; full-size workloads are
checked on sampled heads the oracle computes one by one.  Tolerances: fp32
I/O relative L2 <= 1e-4; bf16 I/O relative L2 <= 1e-2 and max-abs <=
2e-2 * max|ref| (per whole tensor: o, final state and every gradient)."""
import numpy as np
import pytest
import torch

import oracle
from chunked_gated_delta_ckda_b200 import _abi, api
from chunked_gated_delta_ckda_b200 import workloads as W
from tests.gpu_util import (check, f64, oracle_bwd_batched, oracle_fwd_batched, random_inputs,
                            to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    _abi.library()  # fails loudly if the library is missing
    torch.manual_seed(0)


def _fwd(inp, S0=None, chunk_states=False):
    d = to_dev(inp)
    o, ST, cs = api.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"],
                              S0=None if S0 is None else S0.cuda(), save_chunk_states=chunk_states)
    torch.cuda.synchronize()
    return o, ST, cs


# ---------------------------------------------------------------------------
# forward
# ---------------------------------------------------------------------------

def test_tiny_fp32_forward_workload():
    """The tiny fp32 workload (B=1, H=2, T=256, d=64, zero initial state)."""
    inp = W.make(W.TINY)
    o, ST, _ = _fwd(inp)
    o_ref, ST_ref, _ = oracle_fwd_batched(inp)
    check("o", o, o_ref, torch.float32)
    check("ST", ST, ST_ref, torch.float32)


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,T,H,dk,dv", [(2, 200, 3, 64, 128), (1, 64, 2, 128, 64),
                                         (3, 1, 2, 64, 64), (1, 129, 1, 128, 128)])
def test_forward_ragged_with_state(io, B, T, H, dk, dv):
    inp = random_inputs(B, T, H, dk, dv, io, seed=B * 1000 + T, extreme_p=0.05)
    o, ST, cs = _fwd(inp, S0=inp["S0"], chunk_states=True)
    o_ref, ST_ref, cs_ref = oracle_fwd_batched(inp, S0=inp["S0"], chunk=64)
    check("o", o, o_ref, io)
    check("ST", ST, ST_ref, io)
    NC = (T + 63) // 64
    cs_ref = cs_ref.reshape(B, NC, H, dk, dv).transpose(0, 2, 1, 3, 4)
    check("chunk_states", cs, cs_ref, io)


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
def test_forward_strong_decay_exact_pair_path(io, d):
    """Decay strong enough (|g| ~ 3 per token) that the factored pair sums
    would overflow: the kernels must take the exact per-pair path."""
    inp = random_inputs(2, 160, 2, d, d, io, seed=5, gscale=3.0)
    o, ST, _ = _fwd(inp, S0=inp["S0"])
    o_ref, ST_ref, _ = oracle_fwd_batched(inp, S0=inp["S0"])
    check("o", o, o_ref, io)
    check("ST", ST, ST_ref, io)


def test_empty_and_zero_length():
    inp = random_inputs(2, 1, 2, 64, 64, torch.float32, seed=9)
    S0 = inp["S0"].cuda()
    e = lambda *s, dt=torch.float32: torch.empty(*s, dtype=dt, device="cuda")
    q = e(2, 0, 2, 64)
    o = e(2, 0, 2, 64)
    ST = e(2, 2, 64, 64)
    ws = api.workspace(_abi.CKDA_OP_CHUNK_FWD, 2, 0, 2, 64, 64)
    _abi.ckda_chunk_fwd(2, 0, 2, 64, 64, 0, q, q, q, q, e(2, 0, 2, 64, dt=torch.int8), e(2, 0, 2), S0,
                        o, ST, None, ws)
    torch.cuda.synchronize()
    assert torch.equal(ST, S0)
    _abi.ckda_chunk_fwd(0, 5, 2, 64, 64, 0, None, None, None, None, None, None, None, None, None,
                        None, ws)


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------

def _bwd(inp, S0, dST, cs=None):
    d = to_dev(inp)
    r = api.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], d["dO"],
                      S0=None if S0 is None else S0.cuda(), dST=None if dST is None else dST.cuda(),
                      chunk_states=cs)
    torch.cuda.synchronize()
    return r


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,T,H,dk,dv,gscale", [(2, 150, 2, 64, 64, 0.05), (1, 256, 2, 128, 128, 0.05),
                                                (1, 70, 3, 64, 128, 3.0), (2, 33, 1, 128, 64, 0.3),
                                                (1, 100, 2, 128, 128, 3.0), (3, 130, 2, 128, 128, 0.05)])
def test_backward_against_oracle(io, B, T, H, dk, dv, gscale):
    inp = random_inputs(B, T, H, dk, dv, io, seed=T + dk, gscale=gscale, extreme_p=0.05)
    got = _bwd(inp, inp["S0"], inp["dST"])
    ref = oracle_bwd_batched(inp, inp["dO"], S0=inp["S0"], dST=inp["dST"])
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        check(key, got[key], ref[key], io)


def test_backward_uses_saved_chunk_states():
    io = torch.bfloat16
    inp = random_inputs(2, 300, 2, 128, 128, io, seed=11, extreme_p=0.05)
    _, _, cs = _fwd(inp, S0=inp["S0"], chunk_states=True)
    a = _bwd(inp, inp["S0"], inp["dST"], cs=cs)
    b = _bwd(inp, inp["S0"], inp["dST"], cs=None)
    for key in a:
        check(key, a[key], f64(b[key]), io)


@pytest.mark.parametrize("with_cs,gscale", [(True, 0.3), (False, 0.3), (False, 3.0)])
def test_backward_with_saved_forward_results(with_cs, gscale):
    """The forward's saved per-chunk results stand in for the backward's
    recomputation: same kernel on the same inputs, so the gradients are
    bit-identical; and they match the oracle (gscale 3: chunks on the exact
    per-pair path)."""
    io = torch.bfloat16
    inp = random_inputs(2, 300, 2, 128, 128, io, seed=13, gscale=gscale, extreme_p=0.05)
    d = to_dev(inp)
    S0, dST = inp["S0"].cuda(), inp["dST"].cuda()
    o, ST, cs, sv = api.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], S0=S0,
                                  save_chunk_states=True, save_for_backward=True)
    assert sv is not None and sv.numel() == _abi.ckda_saved_size(2, 300, 2, 128, 128, _abi.CKDA_BF16)
    args = (d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], d["dO"])
    a = api.chunk_bwd(*args, S0=S0, dST=dST, chunk_states=cs if with_cs else None, saved=sv)
    b = api.chunk_bwd(*args, S0=S0, dST=dST, chunk_states=cs if with_cs else None)
    torch.cuda.synchronize()
    for key in a:
        assert torch.equal(a[key], b[key]), key
    ref = oracle_bwd_batched(inp, inp["dO"], S0=inp["S0"], dST=inp["dST"])
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        check(key, a[key], ref[key], io)


def test_near_unit_gates_over_a_long_chunk_chain():
    """g ~ -3e-4 per channel and token (decay ~0.9997) over 4096 tokens = 64
    chunks: the state forgets almost nothing, so the bf16 operand roundings
    of every chunk step add up the most here.  The forward (o, final state,
    chunk states) and the backward through the saved buffer, as the training
    step runs them, against the oracle."""
    io = torch.bfloat16
    B, T, H = 1, 4096, 2
    inp = random_inputs(B, T, H, 128, 128, io, seed=77, gscale=4e-4)
    d = to_dev(inp)
    S0, dST = inp["S0"].cuda(), inp["dST"].cuda()
    o, ST, cs, sv = api.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], S0=S0,
                                  save_chunk_states=True, save_for_backward=True)
    got = api.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], d["dO"], S0=S0, dST=dST,
                        saved=sv)
    torch.cuda.synchronize()
    o_ref, ST_ref, cs_ref = oracle_fwd_batched(inp, S0=inp["S0"], chunk=64)
    errs = {"o": check("o", o, o_ref, io), "ST": check("ST", ST, ST_ref, io),
            "chunk_states": check("chunk_states", cs, cs_ref.reshape(B, T // 64, H, 128, 128).transpose(0, 2, 1, 3, 4),
                                  io)}
    ref = oracle_bwd_batched(inp, inp["dO"], S0=inp["S0"], dST=inp["dST"])
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        errs[key] = check(key, got[key], ref[key], io)
    print("relative L2:", {k: "%.2e" % v for k, v in errs.items()})


def test_saved_is_ignored_without_a_saved_form():
    io = torch.float32
    inp = random_inputs(1, 100, 2, 64, 64, io, seed=14)
    d = to_dev(inp)
    o, ST, cs, sv = api.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"],
                                  save_chunk_states=True, save_for_backward=True)
    assert sv is None and _abi.ckda_saved_size(1, 100, 2, 64, 64, _abi.CKDA_F32) == 0
    junk = torch.empty(4096, dtype=torch.uint8, device="cuda")   # ignored for this configuration
    got = api.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], d["dO"],
                        chunk_states=cs, saved=junk)
    ref = oracle_bwd_batched(inp, inp["dO"])
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        check(key, got[key], ref[key], io)


@pytest.mark.parametrize("io,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_kda_mode_without_sign_tensor(io, d):
    """A null sign pointer is standard KDA (every gate sign +1): forward with
    the saved buffer, backward, decode and packed documents match the oracle
    run with an all-ones sign tensor."""
    inp = random_inputs(2, 150, 2, d, d, io, seed=21 + d, extreme_p=0.05)
    inp["sign"] = torch.ones_like(inp["sign"])
    x = to_dev(inp)
    S0, dST = inp["S0"].cuda(), inp["dST"].cuda()
    o, ST, cs, sv = api.chunk_fwd(x["q"], x["k"], x["v"], x["g"], None, x["beta"], S0=S0,
                                  save_chunk_states=True, save_for_backward=True)
    gr = api.chunk_bwd(x["q"], x["k"], x["v"], x["g"], None, x["beta"], x["dO"], S0=S0, dST=dST,
                       chunk_states=cs, saved=sv)
    torch.cuda.synchronize()
    o_ref, ST_ref, _ = oracle_fwd_batched(inp, S0=inp["S0"])
    check("o", o, o_ref, io)
    check("ST", ST, ST_ref, io)
    ref = oracle_bwd_batched(inp, inp["dO"], S0=inp["S0"], dST=inp["dST"])
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        check(key, gr[key], ref[key], io)
    # packed documents (the two batch rows as two documents)
    cu = torch.tensor([0, 150, 300], dtype=torch.int32, device="cuda")
    P = lambda t: t.reshape(1, -1, *t.shape[2:]).contiguous()
    ov, STv = api.varlen_fwd(P(x["q"]), P(x["k"]), P(x["v"]), P(x["g"]), None, P(x["beta"]), cu, 150, S0=S0)
    torch.cuda.synchronize()
    check("o (packed)", ov.reshape(o.shape), o_ref, io)
    check("ST (packed)", STv, ST_ref, io)
    # one decode step from the final state
    st = ST.clone()
    y = random_inputs(3, 1, 2, d, d, io, seed=31 + d)
    y = {k: (v[:, 0] if k in ("q", "k", "v", "g", "sign", "beta") else v) for k, v in y.items()}
    y["sign"] = torch.ones_like(y["sign"])
    yd = to_dev(y)
    st3 = st[:1].expand(3, -1, -1, -1).contiguous()
    st_ref = f64(st3)
    od = api.decode_step(yd["q"], yd["k"], yd["v"], yd["g"], None, yd["beta"], st3)
    torch.cuda.synchronize()
    od_ref, st_ref = oracle.decode(f64(y["q"]), f64(y["k"]), f64(y["v"]), f64(y["g"]), y["sign"].numpy(),
                                   f64(y["beta"]), st_ref)
    check("o (decode)", od, od_ref, io)
    check("state (decode)", st3, st_ref, io)


@pytest.mark.parametrize("B,H", [(1, 2), (2, 1)])
def test_long_sequence_segment_scan(B, H):
    """Few (sequence, head) pairs and many chunks take the segment scan (the
    sequence's chunks split into segments whose affine maps are composed in
    parallel, scanned, and re-run): T = 64 * 48 + 17 gives three segments of
    at most 17 chunks.  Forward with start state, chunk states and final
    state, and the backward's recomputed state pass, against the oracle."""
    io = torch.bfloat16
    T = 64 * 48 + 17
    inp = random_inputs(B, T, H, 128, 128, io, seed=41 + B, gscale=0.05, extreme_p=0.05)
    o, ST, cs = _fwd(inp, S0=inp["S0"], chunk_states=True)
    o_ref, ST_ref, cs_ref = oracle_fwd_batched(inp, S0=inp["S0"], chunk=64)
    check("o", o, o_ref, io)
    check("ST", ST, ST_ref, io)
    NC = (T + 63) // 64
    check("chunk states", cs, cs_ref.reshape(B, NC, H, 128, 128).transpose(0, 2, 1, 3, 4), io)
    got = _bwd(inp, inp["S0"], inp["dST"])
    ref = oracle_bwd_batched(inp, inp["dO"], S0=inp["S0"], dST=inp["dST"])
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        check(key, got[key], ref[key], io)


@pytest.mark.parametrize("B,H,use_saved", [(1, 2, True), (2, 1, False)])
def test_long_sequence_backward_segments(B, H, use_saved):
    """Few pairs over 151 chunks: the backward also splits the sequence into
    segments (the maps M_g, a provisional reverse pass per segment from zero,
    the reverse scan of the adjoint states, then every segment from its true
    end).  Gradients with S0 and dS_T against the oracle; the saved-buffer
    and recomputing paths."""
    io = torch.bfloat16
    T = 64 * 150 + 33
    inp = random_inputs(B, T, H, 128, 128, io, seed=61 + B, gscale=0.05, extreme_p=0.05)
    d = to_dev(inp)
    S0, dST = inp["S0"].cuda(), inp["dST"].cuda()
    r = api.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], S0=S0, save_for_backward=use_saved)
    got = api.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], d["dO"], S0=S0, dST=dST,
                        saved=r[3] if use_saved else None)
    torch.cuda.synchronize()
    ref = oracle_bwd_batched(inp, inp["dO"], S0=inp["S0"], dST=inp["dST"])
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        check(key, got[key], ref[key], io)


def test_long_sequence_segment_scan_many_pairs():
    """20 (sequence, head) pairs over 64 chunks: four segments of 16 chunks,
    the scan split into four value-column slices per pair.  Forward chunk
    states and final state against the oracle."""
    io = torch.bfloat16
    B, H, T = 2, 10, 64 * 63 + 9
    inp = random_inputs(B, T, H, 128, 128, io, seed=47, gscale=0.05, extreme_p=0.05)
    o, ST, cs = _fwd(inp, S0=inp["S0"], chunk_states=True)
    o_ref, ST_ref, cs_ref = oracle_fwd_batched(inp, S0=inp["S0"], chunk=64)
    check("o", o, o_ref, io)
    check("ST", ST, ST_ref, io)
    NC = (T + 63) // 64
    check("chunk states", cs, cs_ref.reshape(B, NC, H, 128, 128).transpose(0, 2, 1, 3, 4), io)


def test_backward_without_state_inputs():
    io = torch.float32
    inp = random_inputs(1, 100, 2, 64, 64, io, seed=12)
    got = _bwd(inp, None, None)
    ref = oracle_bwd_batched(inp, inp["dO"])
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        check(key, got[key], ref[key], io)


# ---------------------------------------------------------------------------
# packed variable-length forward
# ---------------------------------------------------------------------------

def _varlen(lens, io, seed, with_S0=True, gscale=0.05):
    T = int(sum(lens))
    inp = random_inputs(1, T, 2, 128, 128, io, seed=seed, gscale=gscale, extreme_p=0.05)
    N = len(lens)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    S0 = 0.1 * torch.randn(N, 2, 128, 128, generator=torch.Generator().manual_seed(seed)) if with_S0 else None
    d = to_dev(inp)
    o, ST = api.varlen_fwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], cu.cuda(),
                           max(max(lens), 1), S0=None if S0 is None else S0.cuda())
    torch.cuda.synchronize()
    P = lambda x: f64(x[0])
    o_ref, ST_ref, _ = oracle.fwd(cu.numpy().astype(np.int64), P(inp["q"]), P(inp["k"]), P(inp["v"]),
                                  P(inp["g"]), inp["sign"][0].numpy(), P(inp["beta"]), S0=f64(S0))
    return o, ST, o_ref, ST_ref


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_varlen_forward(io):
    o, ST, o_ref, ST_ref = _varlen([1, 16, 64, 65, 200, 5, 128], io, seed=21)
    check("o", o[0], o_ref, io)
    check("ST", ST, ST_ref, io)


def test_varlen_zero_length_documents_and_no_state():
    o, ST, o_ref, ST_ref = _varlen([0, 70, 0, 3, 0], torch.float32, seed=22, with_S0=False)
    check("o", o[0], o_ref, torch.float32)
    check("ST", ST, ST_ref, torch.float32)


def test_varlen_strong_decay():
    o, ST, o_ref, ST_ref = _varlen([100, 37], torch.float32, seed=23, gscale=3.0)
    check("o", o[0], o_ref, torch.float32)
    check("ST", ST, ST_ref, torch.float32)


def test_varlen_malformed_cu_seqlens_reported_on_device():
    inp = random_inputs(1, 64, 2, 64, 64, torch.float32, seed=24)
    d = to_dev(inp)
    for cu in ([0, 40, 30, 64], [0, 40, 64, 70], [1, 40, 64]):
        cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
        N = len(cu) - 1
        ws = api.workspace(_abi.CKDA_OP_VARLEN_FWD, 1, 64, 2, 64, 64, N, cache=False)
        o = torch.empty(1, 64, 2, 64, device="cuda")
        _abi.ckda_varlen_fwd(64, N, cu_t, 64, 2, 64, 64, 0, d["q"], d["k"], d["v"], d["g"], d["sign"],
                             d["beta"], None, o, None, ws)
        assert _abi.ckda_check_device_status(ws) == 7
    # a well-formed call on the same workspace clears the status
    cu_t = torch.tensor([0, 30, 64], dtype=torch.int32, device="cuda")
    _abi.ckda_varlen_fwd(64, 2, cu_t, 64, 2, 64, 64, 0, d["q"], d["k"], d["v"], d["g"], d["sign"],
                         d["beta"], None, o, None, ws)
    assert _abi.ckda_check_device_status(ws) == 0


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_decode_steps(io, dk, dv):
    N, H, steps = 5, 3, 4
    state = 0.1 * torch.randn(N, H, dk, dv, generator=torch.Generator().manual_seed(dk + dv))
    st_ref = f64(state)
    st_dev = state.cuda()
    for t in range(steps):
        x = random_inputs(N, 1, H, dk, dv, io, seed=100 * t + dk)
        x = {k: (v[:, 0] if k in ("q", "k", "v", "g", "sign", "beta") else v) for k, v in x.items()}
        d = to_dev(x)
        o = api.decode_step(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], st_dev)
        torch.cuda.synchronize()
        o_ref, st_ref = oracle.decode(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]),
                                      x["sign"].numpy(), f64(x["beta"]), st_ref)
        check("o[%d]" % t, o, o_ref, io)
        check("state[%d]" % t, st_dev, st_ref, io)


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("K", [1, 3, 8])
def test_decode_multi_pool(io, dk, dv, K):
    """Several steps per sequence on a slot pool: permuted slots, skipped
    sequences (slot -1 and slot n_slots), ragged step counts (0 .. K, one
    clamped from above), no sign tensor on one case; verify (no write-back)
    then commit, against the oracle."""
    N, H, n_slots = 6, 3, 9
    x = random_inputs(N, K, H, dk, dv, io, seed=7 * K + dk + dv)
    pool = 0.1 * torch.randn(n_slots, H, dk, dv, generator=torch.Generator().manual_seed(K + dk))
    slots = torch.tensor([4, 0, -1, 8, 2, 9], dtype=torch.int32)
    n_tok = torch.tensor([K, 0, K, 1, K + 5, max(K - 1, 0)], dtype=torch.int32)
    sign = None if (K == 3 and dk == 64) else x["sign"]
    d = to_dev(x)
    sg = None if sign is None else d["sign"]
    args = (d["q"], d["k"], d["v"], d["g"], sg, d["beta"])
    P = lambda t: f64(t)
    oargs = (P(x["q"]), P(x["k"]), P(x["v"]), P(x["g"]), None if sign is None else sign.numpy(), P(x["beta"]))
    dev_pool = pool.cuda()
    o_ver = api.decode_multi(*args, dev_pool, slots=slots.cuda(), n_tokens=None, write_state=False)
    torch.cuda.synchronize()
    assert torch.equal(dev_pool.cpu(), pool)  # verify leaves the pool untouched
    ref_o, _ = oracle.decode_multi(*oargs, P(pool), n_tokens=None, slots=slots.numpy(), write_state=False)
    check("o (verify)", o_ver, ref_o, io)
    o_com = api.decode_multi(*args, dev_pool, slots=slots.cuda(), n_tokens=n_tok.cuda(), write_state=True)
    torch.cuda.synchronize()
    ref_o, ref_pool = oracle.decode_multi(*oargs, P(pool), n_tokens=n_tok.numpy(), slots=slots.numpy())
    check("o (commit)", o_com, ref_o, io)
    check("pool", dev_pool, ref_pool, io)
    untouched = [s for s in range(n_slots) if s not in (4, 8, 2)]
    assert torch.equal(dev_pool.cpu()[untouched], pool[untouched])


@pytest.mark.parametrize("io,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_decode_multi_many_items_per_cta(io, d):
    """More (sequence, head, column slice) items than resident CTAs, so every
    CTA walks several items and prefetches the next one's state: skipped and
    zero-step sequences interleaved, ragged step counts, a permuted pool."""
    N, K, H, n_slots = 160, 3, 4, 200
    x = random_inputs(N, K, H, d, d, io, seed=91 + d)
    gen = torch.Generator().manual_seed(d)
    pool = 0.1 * torch.randn(n_slots, H, d, d, generator=gen)
    slots = torch.randperm(n_slots, generator=gen)[:N].to(torch.int32)
    slots[torch.rand(N, generator=gen) < 0.1] = -1
    n_tok = torch.randint(0, K + 1, (N,), generator=gen, dtype=torch.int32)
    d_ = to_dev(x)
    dev_pool = pool.cuda()
    o = api.decode_multi(d_["q"], d_["k"], d_["v"], d_["g"], d_["sign"], d_["beta"], dev_pool, slots=slots.cuda(),
                         n_tokens=n_tok.cuda())
    torch.cuda.synchronize()
    ref_o, ref_pool = oracle.decode_multi(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]), x["sign"].numpy(),
                                          f64(x["beta"]), f64(pool), n_tokens=n_tok.numpy(), slots=slots.numpy())
    check("o", o, ref_o, io)
    check("pool", dev_pool, ref_pool, io)


def test_decode_multi_matches_decode_steps():
    """K steps in one call against K single-step calls (the existing decode
    kernel) on the same states: both against the oracle, and close to each
    other."""
    io, N, K, H, dk, dv = torch.bfloat16, 4, 5, 2, 128, 128
    x = random_inputs(N, K, H, dk, dv, io, seed=77)
    state = 0.1 * torch.randn(N, H, dk, dv, generator=torch.Generator().manual_seed(5))
    d = to_dev(x)
    a = state.cuda()
    o_multi = api.decode_multi(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], a)
    b = state.cuda()
    outs = []
    for t in range(K):
        outs.append(api.decode_step(*(d[n][:, t].contiguous() for n in ("q", "k", "v", "g", "sign", "beta")), b))
    torch.cuda.synchronize()
    o_steps = torch.stack(outs, 1)
    ref_o, ref_pool = oracle.decode_multi(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]), x["sign"].numpy(),
                                          f64(x["beta"]), f64(state))
    check("o (multi)", o_multi, ref_o, io)
    check("o (steps)", o_steps, ref_o, io)
    check("state (multi)", a, ref_pool, io)
    check("state (steps)", b, ref_pool, io)
    assert (a - b).abs().max().item() < 1e-4


def test_decode_continues_chunked_final_state():
    """States cross the ABI in the true frame: decode after a chunked forward
    equals one forward over the concatenation."""
    io = torch.float32
    inp = random_inputs(2, 101, 2, 64, 64, io, seed=31)
    pre = {k: (v[:, :100] if k in ("q", "k", "v", "g", "sign", "beta") else v) for k, v in inp.items()}
    _, ST, _ = _fwd(pre, S0=inp["S0"])
    last = {k: inp[k][:, 100].contiguous() for k in ("q", "k", "v", "g", "sign", "beta")}
    d = to_dev(last)
    o = api.decode_step(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], ST)
    o_ref, ST_ref, _ = oracle_fwd_batched(inp, S0=inp["S0"])
    check("o_last", o, o_ref[:, 100], io)
    check("ST", ST, ST_ref, io)


# ---------------------------------------------------------------------------
# full-size workloads, sampled heads
# ---------------------------------------------------------------------------

def _sample_heads(B, H, n, seed):
    rng = np.random.default_rng(seed)
    return [(int(b), int(h)) for b, h in zip(rng.integers(0, B, n), rng.integers(0, H, n))]


def test_full_layer_fwd_bwd_sampled_heads():
    """B=8, H=16, T=4096, d=128, bf16: the forward+backward the benchmark times,
    checked on sampled (batch, head) pairs."""
    w = W.LAYER_FWDBWD
    inp = W.make(w)
    d = to_dev(inp)
    o, ST, cs, sv = api.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"],
                                  save_chunk_states=True, save_for_backward=True)
    gr = api.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], d["dO"], chunk_states=cs,
                       saved=sv)
    torch.cuda.synchronize()
    for b, h in _sample_heads(w.B, w.H, 3, seed=1):
        sub = {k: inp[k][b:b + 1, :, h:h + 1].contiguous() for k in ("q", "k", "v", "g", "sign", "beta", "dO")}
        o_ref, ST_ref, _ = oracle_fwd_batched(sub)
        check("o[%d,%d]" % (b, h), o[b:b + 1, :, h:h + 1], o_ref, w.io_dtype)
        check("ST[%d,%d]" % (b, h), ST[b:b + 1, h:h + 1], ST_ref, w.io_dtype)
        ref = oracle_bwd_batched(sub, sub["dO"])
        for key in ("dq", "dk", "dv", "dg", "dbeta"):
            check("%s[%d,%d]" % (key, b, h), gr[key][b:b + 1, :, h:h + 1], ref[key], w.io_dtype)
        check("dS0[%d,%d]" % (b, h), gr["dS0"][b:b + 1, h:h + 1], ref["dS0"], w.io_dtype)


def test_full_varlen_sampled():
    """65536 packed tokens (geometric document lengths), H=16, d=128, bf16."""
    w = W.VARLEN
    inp = W.make_varlen(w)
    d = to_dev(inp)
    cu = inp["cu_seqlens"]
    o, ST = api.varlen_fwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], cu.cuda(),
                           max(inp["lens"]))
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    docs = rng.choice(len(inp["lens"]), 3, replace=False)
    for i in docs:
        a, b = int(cu[i]), int(cu[i + 1])
        h = int(rng.integers(0, w.H))
        sl = lambda x: f64(x[0, a:b, h:h + 1])
        o_ref, ST_ref, _ = oracle.fwd([0, b - a], sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]),
                                      inp["sign"][0, a:b, h:h + 1].numpy(), sl(inp["beta"]))
        check("o[doc %d]" % i, o[0, a:b, h:h + 1], o_ref, w.io_dtype)
        check("ST[doc %d]" % i, ST[i:i + 1, h:h + 1], ST_ref, w.io_dtype)


def test_full_long_sequence_sampled():
    """One 65536-token sequence with an N(0, 0.1^2) initial state."""
    w = W.LONG
    inp = W.make(w)
    d = to_dev(inp)
    o, ST, _ = api.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], S0=d["S0"])
    torch.cuda.synchronize()
    h = 5
    sub = {k: inp[k][:, :, h:h + 1].contiguous() for k in ("q", "k", "v", "g", "sign", "beta")}
    o_ref, ST_ref, _ = oracle_fwd_batched(sub, S0=inp["S0"][:, h:h + 1])
    check("o", o[:, :, h:h + 1], o_ref, w.io_dtype)
    check("ST", ST[:, h:h + 1], ST_ref, w.io_dtype)


def test_full_decode_steps():
    """N=256, H=16, d=128 states, bf16 I/O, a few consecutive steps, all heads."""
    w = W.DECODE
    state = W.make_decode_state(w)
    st_dev = state.cuda()
    st_ref = f64(state)
    for t in range(3):
        x = W.make_decode_step(w, t)
        d = to_dev(x)
        o = api.decode_step(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], st_dev)
        torch.cuda.synchronize()
        o_ref, st_ref = oracle.decode(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]),
                                      x["sign"].numpy(), f64(x["beta"]), st_ref)
        check("o[%d]" % t, o, o_ref, w.io_dtype)
    check("state", st_dev, st_ref, w.io_dtype)


def test_decode_chain_512_steps():
    """The recurrent-decode workload's chain length: 512 consecutive single-token
    calls on fp32 states resident on the device (8 sequences x 16 heads, d=128,
    bf16 I/O, the decode workload's input generators and N(0, 0.1^2) states),
    o checked at every step and the state after the last, against the oracle
    carrying its own fp64 state through the same 512 steps."""
    w = W.DECODE
    N, steps = 8, 512
    state = W.make_decode_state(w, N=N)
    st_dev = state.cuda()
    st_ref = f64(state)
    for t in range(steps):
        x = W.make_decode_step(w, t, N=N)
        d = to_dev(x)
        o = api.decode_step(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], st_dev)
        o_ref, st_ref = oracle.decode(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["g"]),
                                      x["sign"].numpy(), f64(x["beta"]), st_ref)
        torch.cuda.synchronize()
        check("o[%d]" % t, o, o_ref, w.io_dtype)
    check("state after %d steps" % steps, st_dev, st_ref, w.io_dtype)


# ---------------------------------------------------------------------------
# token-mixer prologue
# ---------------------------------------------------------------------------

def _prologue_inputs(B, T, H, dk, dv, io, seed):
    gen = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=gen)
    x = dict(xq=r(B, T, H, dk).to(io), xk=r(B, T, H, dk).to(io), xv=r(B, T, H, dv).to(io),
             wq=0.5 * r(H * dk, 4), wk=0.5 * r(H * dk, 4), wv=0.5 * r(H * dv, 4),
             a=1.5 * r(B, T, H, dk), b=(2.0 * r(B, T, H)).to(io))
    up = dict(dq=r(B, T, H, dk).to(io), dk=r(B, T, H, dk).to(io), dv=r(B, T, H, dv).to(io),
              dg=r(B, T, H, dk), dbeta=r(B, T, H).to(io))
    return x, up


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,T,H,dk,dv,g_floor", [(2, 200, 3, 64, 128, -5.0), (1, 64, 2, 128, 64, -1.0),
                                                 (3, 5, 2, 64, 64, -5.0), (1, 129, 2, 128, 128, -0.5)])
def test_prologue_forward_backward(io, B, T, H, dk, dv, g_floor):
    """Short conv + SiLU, q/k L2 norm, signed gate, beta: forward outputs and
    every gradient against the fp64 oracle (runs of 64 tokens with a ragged
    tail, sequences shorter than the conv window, several clamp levels)."""
    x, up = _prologue_inputs(B, T, H, dk, dv, io, seed=B * 100 + T + dk)
    d = to_dev({**x, **up})
    got = api.prologue_fwd(d["xq"], d["xk"], d["xv"], d["wq"], d["wk"], d["wv"], d["a"], d["b"], g_floor=g_floor)
    gr = api.prologue_bwd(d["xq"], d["xk"], d["xv"], d["wq"], d["wk"], d["wv"], d["a"], d["b"], d["dq"], d["dk"],
                          d["dv"], d["dg"], d["dbeta"], g_floor=g_floor)
    torch.cuda.synchronize()
    X = {n: f64(t) for n, t in x.items()}
    ref = oracle.prologue_fwd(**X, g_floor=g_floor)
    for n in ("q", "k", "v", "g", "beta"):
        check(n, got[n], ref[n], io)
    assert torch.equal(got["sign"].cpu(), torch.from_numpy(ref["sign"]))
    rg = oracle.prologue_bwd(**X, **{n: f64(t) for n, t in up.items()}, g_floor=g_floor)
    for n in ("dxq", "dxk", "dxv", "dwq", "dwk", "dwv", "da", "db"):
        check(n, gr[n], rg[n], io)


def _oracle_prologue_stored(x, io, cu=None):
    """The oracle's prologue outputs as the boundary stores them (q, k, v,
    beta in the I/O dtype, g in fp32): the recurrence oracle's inputs."""
    r = oracle.prologue_fwd(**{n: f64(t) for n, t in x.items()}, g_floor=-5.0, cu_seqlens=cu)
    st = {n: torch.from_numpy(r[n]).to(io) for n in ("q", "k", "v", "beta")}
    st.update(g=torch.from_numpy(r["g"]).float(), sign=torch.from_numpy(r["sign"]))
    return st


def test_prologue_feeds_the_recurrence():
    """prologue -> chunked forward equals the oracle's prologue -> recurrence."""
    io, B, T, H, d = torch.bfloat16, 1, 150, 2, 128
    x, _ = _prologue_inputs(B, T, H, d, d, io, seed=5)
    dx = to_dev(x)
    p = api.prologue_fwd(dx["xq"], dx["xk"], dx["xv"], dx["wq"], dx["wk"], dx["wv"], dx["a"], dx["b"], g_floor=-5.0)
    o, ST, _ = api.chunk_fwd(p["q"], p["k"], p["v"], p["g"], p["sign"], p["beta"])
    torch.cuda.synchronize()
    o_ref, ST_ref, _ = oracle_fwd_batched(_oracle_prologue_stored(x, io))
    check("o", o, o_ref, io)
    check("ST", ST, ST_ref, io)


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("lens,dk,dv", [([1, 2, 0, 58, 3, 2, 64, 3, 67], 64, 128),
                                        ([61, 4, 1, 1, 1, 62, 70], 128, 64), ([130], 128, 128)])
def test_prologue_packed_documents(io, lens, dk, dv):
    """Documents packed in one row (cu_seqlens): the conv history restarts at
    every document start, forward and backward, against the oracle (documents
    of one to three tokens, an empty one, starts just before, at and after
    the kernels' 64-token run edges)."""
    T, H, g_floor = int(sum(lens)), 2, -5.0
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x, up = _prologue_inputs(1, T, H, dk, dv, io, seed=T + dk)
    d = to_dev({**x, **up})
    names = ("xq", "xk", "xv", "wq", "wk", "wv", "a", "b")
    dcu = torch.from_numpy(cu).cuda()
    got = api.prologue_fwd(*(d[n] for n in names), g_floor=g_floor, cu_seqlens=dcu)
    gr = api.prologue_bwd(*(d[n] for n in names), d["dq"], d["dk"], d["dv"], d["dg"], d["dbeta"],
                          g_floor=g_floor, cu_seqlens=dcu)
    torch.cuda.synchronize()
    X = {n: f64(t) for n, t in x.items()}
    ref = oracle.prologue_fwd(**X, g_floor=g_floor, cu_seqlens=cu)
    for n in ("q", "k", "v", "g", "beta"):
        check(n, got[n], ref[n], io)
    assert torch.equal(got["sign"].cpu(), torch.from_numpy(ref["sign"]))
    rg = oracle.prologue_bwd(**X, **{n: f64(t) for n, t in up.items()}, g_floor=g_floor, cu_seqlens=cu)
    for n in ("dxq", "dxk", "dxv", "dwq", "dwk", "dwv", "da", "db"):
        check(n, gr[n], rg[n], io)
    if len(lens) == 1:  # one document: the same kernels' arithmetic as the unpacked row
        plain = api.prologue_fwd(*(d[n] for n in names), g_floor=g_floor)
        for n in ("q", "k", "v", "g", "sign", "beta"):
            assert torch.equal(plain[n], got[n]), n


def test_prologue_packed_feeds_varlen():
    """Packed prologue -> packed recurrence equals the oracle's per-document
    prologue -> recurrence."""
    io, H, d, lens = torch.bfloat16, 2, 128, [37, 2, 90, 64]
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x, _ = _prologue_inputs(1, T, H, d, d, io, seed=9)
    dx = to_dev(x)
    p = api.prologue_fwd(*(dx[n] for n in ("xq", "xk", "xv", "wq", "wk", "wv", "a", "b")), g_floor=-5.0,
                         cu_seqlens=torch.from_numpy(cu).cuda())
    o, ST = api.varlen_fwd(p["q"], p["k"], p["v"], p["g"], p["sign"], p["beta"], torch.from_numpy(cu).cuda(),
                           max(lens))
    torch.cuda.synchronize()
    r = _oracle_prologue_stored(x, io, cu)
    P = lambda n: f64(r[n][0])
    o_ref, ST_ref, _ = oracle.fwd(cu.astype(np.int64), P("q"), P("k"), P("v"), P("g"), r["sign"][0].numpy(), P("beta"))
    check("o", o[0], o_ref, io)
    check("ST", ST, ST_ref, io)


def test_full_decode_multi_sampled():
    """The benchmark's multi-token decode (256 sequences x 4 tokens, H=16,
    d=128, 512-slot pool) in its launch configuration, checked on sampled
    sequences (all heads) and on the slots nothing touched."""
    w = W.DECODE_MULTI
    x = W.make_decode_multi(w, call=0)
    pool = W.make_decode_pool(w)
    dpool = pool.cuda()
    d = to_dev(x)
    o = api.decode_multi(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], dpool, slots=d["slots"])
    torch.cuda.synchronize()
    rng = np.random.default_rng(4)
    seqs = sorted(rng.choice(w.B, 3, replace=False).tolist())
    sub = lambda t: t[seqs]
    slots = x["slots"][seqs].numpy()
    ref_o, ref_pool = oracle.decode_multi(f64(sub(x["q"])), f64(sub(x["k"])), f64(sub(x["v"])), f64(sub(x["g"])),
                                          sub(x["sign"]).numpy(), f64(sub(x["beta"])), f64(pool), slots=slots)
    check("o (sampled sequences)", o[seqs], ref_o, w.io_dtype)
    check("pool (their slots)", dpool[torch.from_numpy(slots).long().cuda()], ref_pool[slots], w.io_dtype)
    live = set(x["slots"].tolist())
    idle = [s for s in range(pool.shape[0]) if s not in live][:8]
    assert torch.equal(dpool[idle].cpu(), pool[idle])


def test_full_prologue_sampled_heads():
    """The benchmark's prologue (B=8, T=4096, H=16, d=128, bf16) forward and
    backward, checked on sampled heads over the whole batch (the conv taps'
    gradients sum over every token of a head)."""
    w = W.LAYER_FWDBWD
    x = W.make_prologue(w)
    d = to_dev(x)
    names = ("xq", "xk", "xv", "wq", "wk", "wv", "a", "b")
    p = api.prologue_fwd(*(d[n] for n in names), g_floor=-5.0)
    gr = api.prologue_bwd(*(d[n] for n in names), d["dq"], d["dk"], d["dv"], d["dg"], d["dbeta"], g_floor=-5.0)
    torch.cuda.synchronize()
    for h in (3, 11):
        hs = slice(h, h + 1)
        X = {n: f64(x[n][:, :, hs]) for n in ("xq", "xk", "xv", "a", "b")}
        X.update({n: f64(x[n][h * 128:(h + 1) * 128]) for n in ("wq", "wk", "wv")})
        up = {n: f64(x[n][:, :, hs]) for n in ("dq", "dk", "dv", "dg", "dbeta")}
        ref = oracle.prologue_fwd(**X, g_floor=-5.0)
        for n in ("q", "k", "v", "g", "beta"):
            check("%s[h=%d]" % (n, h), p[n][:, :, hs], ref[n], w.io_dtype)
        assert torch.equal(p["sign"][:, :, hs].cpu(), torch.from_numpy(ref["sign"]))
        rg = oracle.prologue_bwd(**X, **up, g_floor=-5.0)
        for n in ("dxq", "dxk", "dxv", "da", "db"):
            check("%s[h=%d]" % (n, h), gr[n][:, :, hs], rg[n], w.io_dtype)
        for n in ("dwq", "dwk", "dwv"):
            check("%s[h=%d]" % (n, h), gr[n][h * 128:(h + 1) * 128], rg[n], w.io_dtype)


# ---------------------------------------------------------------------------
# packed documents: backward
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("io,d", [(torch.bfloat16, 128), (torch.float32, 64)])
@pytest.mark.parametrize("lens", [[200, 1, 64, 0, 130], [64 * 5 + 3], [0, 65, 0]])
def test_varlen_backward(io, d, lens):
    """Gradients over packed documents (ragged, a one-token document, empty
    documents), with per-document initial states and final-state gradients,
    on the tensor-core (bf16, d=128) and CUDA-core (fp32, d=64) paths."""
    T, H, N = int(sum(lens)), 2, len(lens)
    inp = random_inputs(1, T, H, d, d, io, seed=T + d, gscale=0.05, extreme_p=0.05)
    gen = torch.Generator().manual_seed(T + 7)
    S0 = 0.1 * torch.randn(N, H, d, d, generator=gen)
    dST = torch.randn(N, H, d, d, generator=gen)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    x = to_dev(inp)
    got = api.varlen_bwd(x["q"], x["k"], x["v"], x["g"], x["sign"], x["beta"], x["dO"], cu.cuda(),
                         max(max(lens), 1), S0=S0.cuda(), dST=dST.cuda())
    torch.cuda.synchronize()
    P = lambda t: f64(t[0])
    ref = oracle.bwd(cu.numpy().astype(np.int64), P(inp["q"]), P(inp["k"]), P(inp["v"]), P(inp["g"]),
                     inp["sign"][0].numpy(), P(inp["beta"]), P(inp["dO"]), S0=f64(S0), dST=f64(dST))
    for key in ("dq", "dk", "dv", "dg", "dbeta"):
        check(key, got[key][0], ref[key], io)
    check("dS0", got["dS0"], ref["dS0"], io)


def test_varlen_backward_with_saved_forward_results():
    """The packed forward's saved per-chunk results stand in for the packed
    backward's recomputation: bit-identical gradients, and the oracle's."""
    io, H, d = torch.bfloat16, 2, 128
    lens = [150, 0, 64, 77]
    T, N = int(sum(lens)), len(lens)
    inp = random_inputs(1, T, H, d, d, io, seed=71, gscale=0.3, extreme_p=0.05)
    gen = torch.Generator().manual_seed(72)
    S0 = (0.1 * torch.randn(N, H, d, d, generator=gen)).cuda()
    dST = torch.randn(N, H, d, d, generator=gen).cuda()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32).cuda()
    x = to_dev(inp)
    args = (x["q"], x["k"], x["v"], x["g"], x["sign"], x["beta"])
    o, ST, sv = api.varlen_fwd(*args, cu, max(lens), S0=S0, save_for_backward=True)
    assert sv is not None and sv.numel() == _abi.ckda_varlen_saved_size(T, N, H, d, d, _abi.CKDA_BF16)
    a = api.varlen_bwd(*args, x["dO"], cu, max(lens), S0=S0, dST=dST, saved=sv)
    b = api.varlen_bwd(*args, x["dO"], cu, max(lens), S0=S0, dST=dST)
    torch.cuda.synchronize()
    for key in a:
        assert torch.equal(a[key], b[key]), key
    P = lambda t: f64(t[0])
    ref = oracle.bwd(cu.cpu().numpy().astype(np.int64), P(inp["q"]), P(inp["k"]), P(inp["v"]), P(inp["g"]),
                     inp["sign"][0].numpy(), P(inp["beta"]), P(inp["dO"]), S0=f64(S0.cpu()), dST=f64(dST.cpu()))
    for key in ("dq", "dk", "dv", "dg", "dbeta"):
        check(key, a[key][0], ref[key], io)
    check("dS0", a["dS0"], ref["dS0"], io)


def test_full_varlen_backward_sampled():
    """The packed-document workload (65536 tokens, geometric document
    lengths, H=16, d=128, bf16) through the backward, checked on sampled
    documents and heads."""
    w = W.VARLEN
    inp = W.make_varlen(w)
    d = to_dev(inp)
    cu = inp["cu_seqlens"]
    gen = torch.Generator().manual_seed(9)
    dO = torch.randn(inp["q"].shape[:3] + (w.dv,), generator=gen).to(w.io_dtype)
    got = api.varlen_bwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], dO.cuda(), cu.cuda(),
                         max(inp["lens"]))
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    for i in rng.choice(len(inp["lens"]), 3, replace=False):
        a, b = int(cu[i]), int(cu[i + 1])
        h = int(rng.integers(0, w.H))
        sl = lambda x: f64(x[0, a:b, h:h + 1])
        ref = oracle.bwd([0, b - a], sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]),
                         inp["sign"][0, a:b, h:h + 1].numpy(), sl(inp["beta"]), sl(dO))
        for key in ("dq", "dk", "dv", "dg", "dbeta"):
            check("%s[doc %d]" % (key, i), got[key][0, a:b, h:h + 1], ref[key], w.io_dtype)
        check("dS0[doc %d]" % i, got["dS0"][i:i + 1, h:h + 1], ref["dS0"], w.io_dtype)
