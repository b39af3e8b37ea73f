"""ckda_chunk_fwd_noalloc: the chunked forward for callers that cannot
allocate device memory (its scratch is a fixed array the library owns).

Collected last on purpose.  Two calls in a row through the C ABI must match
ckda_chunk_fwd (which uses a caller workspace) within the parity tolerances,
the second call must not be disturbed by what the first left in the shared
array, and oversized problems must be refused before any work is enqueued."""
import pytest
import torch

from chunked_gated_delta_ckda_b200 import _abi, api
from tests.gpu_util import check, random_inputs, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(d, B, T, H, dk, dv, S0):
    o = torch.empty(B, T, H, dv, dtype=d["q"].dtype, device="cuda")
    ST = torch.empty(B, H, dk, dv, dtype=torch.float32, device="cuda")
    cs = torch.empty(B, H, (T + 63) // 64, dk, dv, dtype=torch.float32, device="cuda")
    _abi.ckda_chunk_fwd_noalloc(B, T, H, dk, dv, api.io_code(d["q"].dtype), d["q"], d["k"], d["v"],
                                d["g"], d["sign"], d["beta"], S0, o, ST, cs)
    return o, ST, cs


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
def test_two_calls_match_workspace_forward(io):
    assert torch.cuda.is_available()
    cases = [(2, 300, 4, 128, 128, 41), (1, 200, 3, 64, 128, 42)]
    for B, T, H, dk, dv, seed in cases:   # two calls in a row, different shapes
        inp = random_inputs(B, T, H, dk, dv, io, seed=seed, extreme_p=0.05)
        d = to_dev(inp)
        S0 = d["S0"]
        o, ST, cs = _noalloc(d, B, T, H, dk, dv, S0)
        o_ref, ST_ref, cs_ref = api.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["sign"], d["beta"],
                                              S0=S0, save_chunk_states=True)
        torch.cuda.synchronize()
        check("o", o, o_ref.double().cpu().numpy(), io)
        check("ST", ST, ST_ref.double().cpu().numpy(), io)
        check("chunk_states", cs, cs_ref.double().cpu().numpy(), io)


def test_refuses_problems_beyond_capacity():
    B, T, H, d = 8, 4096, 16, 128
    fake = torch.empty(16, dtype=torch.uint8, device="cuda")
    rc = _abi.library().ckda_chunk_fwd_noalloc(B, T, H, d, d, 1, *([_abi._p(fake)] * 6), None,
                                               _abi._p(fake), None, None, None)
    assert rc == 8   # CKDA_ERR_NOALLOC_CAPACITY, nothing enqueued
