"""Failure detection on the GPU without a fault: the library's bounded
mbarrier wait, run against a barrier nothing arrives at, gives up, the
time-out reaches the host through the workspace status word, and the
context stays usable for the next call."""
import pytest
import torch

from chunked_gated_delta_ckda_b200 import _abi
from chunked_gated_delta_ckda_b200 import workloads as W
from tests.gpu_util import check, oracle_fwd_batched
from tests.test_gpu_parity import _fwd

pytestmark = pytest.mark.gpu

SITE = 900  # the self-test wait's site code in the status word


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    _abi.library()


def test_bounded_wait_gives_up_and_reports_timeout():
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    assert ws.data_ptr() % 256 == 0
    for polls in (0, 1, 1 << 12):
        ws.fill_(0xFF)  # the call clears the status word itself
        _abi.ckda_selftest_bounded_wait(ws, polls)
        assert _abi.STATUS[_abi.ckda_check_device_status(ws)] == "CKDA_ERR_TIMEOUT"
        flags, detail = ws[:8].view(torch.int32).cpu().tolist()
        assert flags == 1 and detail == SITE, (polls, flags, detail)


def test_context_usable_after_timeouts():
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    _abi.ckda_selftest_bounded_wait(ws, 16)
    torch.cuda.synchronize()
    inp = W.make(W.TINY)
    o, ST, _ = _fwd(inp)
    o_ref, ST_ref, _ = oracle_fwd_batched(inp)
    check("o", o, o_ref, torch.float32)
    check("ST", ST, ST_ref, torch.float32)
