"""ckda_chunk_fwd_noalloc: the chunked forward for callers that cannot
allocate device memory (a plug-in whose host application owns every device
allocation, or a latency-critical path that must not call cudaMalloc); its
scratch is a fixed array the library owns.

Collected last on purpose (a failure here comes after every other test has
run).  Two calls in a row through the C ABI are each checked against the fp64
oracle on the same inputs, at the parity tolerances, so the second call must
not be disturbed by what the first left in the shared array.  The capacity
limit is checked at its boundary, oversized problems are refused before
anything is enqueued, and the empty cases keep their meaning."""
import numpy as np
import pytest
import torch

from chunked_gated_delta_ckda_b200 import _abi, api
from tests.gpu_util import check, oracle_fwd_batched, random_inputs, to_dev

pytestmark = pytest.mark.gpu

CAPACITY_ERR = 8  # CKDA_ERR_NOALLOC_CAPACITY


def _noalloc(d, B, T, H, dk, dv, S0):
    """One call through the C ABI (caller-allocated outputs, no workspace)."""
    o = torch.empty(B, T, H, dv, dtype=d["q"].dtype, device="cuda")
    ST = torch.empty(B, H, dk, dv, dtype=torch.float32, device="cuda")
    cs = torch.empty(B, H, (T + 63) // 64, dk, dv, dtype=torch.float32, device="cuda")
    _abi.ckda_chunk_fwd_noalloc(B, T, H, dk, dv, api.io_code(d["q"].dtype), d["q"], d["k"], d["v"],
                                d["g"], d["sign"], d["beta"], S0, o, ST, cs)
    return o, ST, cs


def _check_against_oracle(inp, o, ST, cs, io):
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    o_ref, ST_ref, cs_ref = oracle_fwd_batched(inp, S0=inp["S0"], chunk=64)
    check("o", o, o_ref, io)
    check("ST", ST, ST_ref, io)
    NC = (T + 63) // 64
    check("chunk_states", cs, cs_ref.reshape(B, NC, H, dk, dv).transpose(0, 2, 1, 3, 4), io)


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
def test_two_calls_in_a_row_match_oracle(io):
    assert torch.cuda.is_available()
    cases = [(2, 300, 4, 128, 128, 41), (1, 200, 3, 64, 128, 42)]
    outs = []
    for B, T, H, dk, dv, seed in cases:   # two calls in a row, different shapes
        inp = random_inputs(B, T, H, dk, dv, io, seed=seed, extreme_p=0.05)
        d = to_dev(inp)
        outs.append((inp, _noalloc(d, B, T, H, dk, dv, d["S0"])))
    torch.cuda.synchronize()
    for inp, (o, ST, cs) in outs:
        _check_against_oracle(inp, o, ST, cs, io)


def test_api_wrapper_matches_oracle():
    inp = random_inputs(1, 130, 2, 128, 128, torch.bfloat16, seed=43)
    d = to_dev(inp)
    o, ST, cs = api.chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"], S0=d["S0"],
                                      save_chunk_states=True)
    torch.cuda.synchronize()
    _check_against_oracle(inp, o, ST, cs, torch.bfloat16)


def test_capacity_boundary():
    """194 chunk-heads at d = 128 fit (B=2, T=6208: 97 chunks each, H=1); 195
    (B=3, T=4160: 65 chunks each) are refused with nothing enqueued."""
    inp = random_inputs(2, 6208, 1, 128, 128, torch.bfloat16, seed=44)
    d = to_dev(inp)
    o, ST, cs = _noalloc(d, 2, 6208, 1, 128, 128, d["S0"])
    torch.cuda.synchronize()
    _check_against_oracle(inp, o, ST, cs, torch.bfloat16)

    fake = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = _abi._p(fake)
    lib = _abi.library()
    for B, T, H in ((3, 4160, 1), (1, 195 * 64, 1), (8, 4096, 16)):
        rc = lib.ckda_chunk_fwd_noalloc(B, T, H, 128, 128, 1, p, p, p, p, None, p, None, p, None, None, None)
        assert rc == CAPACITY_ERR, (B, T, H, rc)
    # at d = 64 the limit is 379 chunk-heads
    assert lib.ckda_chunk_fwd_noalloc(1, 380 * 64, 1, 64, 64, 1, p, p, p, p, None, p, None, p, None, None,
                                      None) == CAPACITY_ERR


def test_empty_problems():
    """T = 0: the final state is the initial state; B = 0: nothing to do."""
    S0 = (0.1 * torch.randn(2, 2, 128, 128, generator=torch.Generator().manual_seed(45))).cuda()
    e = lambda *s, dt=torch.bfloat16: torch.empty(*s, dtype=dt, device="cuda")
    q = e(2, 0, 2, 128)
    g = e(2, 0, 2, 128, dt=torch.float32)
    beta = e(2, 0, 2)
    ST = torch.full((2, 2, 128, 128), float("nan"), device="cuda")
    _abi.ckda_chunk_fwd_noalloc(2, 0, 2, 128, 128, 1, q, q, q, g, None, beta, S0, q, ST, None)
    torch.cuda.synchronize()
    assert torch.equal(ST, S0)
    ST.fill_(float("nan"))
    _abi.ckda_chunk_fwd_noalloc(2, 0, 2, 128, 128, 1, q, q, q, g, None, beta, None, q, ST, None)
    torch.cuda.synchronize()
    assert torch.count_nonzero(ST).item() == 0
    rc = _abi.library().ckda_chunk_fwd_noalloc(0, 64, 2, 128, 128, 1, None, None, None, None, None, None,
                                               None, None, None, None, None)
    assert rc == 0
    assert np.isfinite(ST.cpu().numpy()).all()
