"""Plant plausible mistakes in a copy of the prologue oracle (CPU only) and
check that the pins of test_oracle_prologue.py catch every one of them."""
import os
import types

import pytest

import oracle
from tests import test_oracle_prologue as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "prologue.py")

MUTATIONS = {
    "taps_reversed": ("shift = WIDTH - 1 - j  # tap j reads token t - shift",
                      "shift = j"),
    "silu_dropped": ("return y * torch.sigmoid(y)", "return y"),
    "norm_over_heads": ("q = nq / torch.sqrt((nq * nq).sum(-1, keepdim=True) + EPS)",
                        "q = nq / torch.sqrt((nq * nq).sum(-2, keepdim=True) + EPS)"),
    "norm_eps_dropped": ("k = nk / torch.sqrt((nk * nk).sum(-1, keepdim=True) + EPS)",
                         "k = nk / torch.sqrt((nk * nk).sum(-1, keepdim=True))"),
    "gate_half_argument": ("alpha = torch.tanh(a)", "alpha = torch.tanh(0.5 * a)"),
    "beta_range_halved": ("beta = 2.0 * torch.sigmoid(b)", "beta = torch.sigmoid(b)"),
    "history_across_sequences": (
        "torch.cat([torch.zeros_like(x[:, :shift]), x[:, :T - shift]], dim=1)",
        "torch.cat([torch.roll(x, 1, 0)[:, T - shift:], x[:, :T - shift]], dim=1)"),
    "history_across_documents": (
        "return torch.cat([_conv_silu(x[:, s:e], w) for s, e in docs], dim=1)",
        "return _conv_silu(x, w)"),
    "gradient_through_floor": (
        "g = torch.clamp(torch.log(torch.abs(alpha)), min=g_floor)",
        "lg = torch.log(torch.abs(alpha))\n    g = torch.clamp(lg, min=g_floor).detach() + "
        "torch.where(torch.isfinite(lg), lg - lg.detach(), torch.zeros_like(lg))"),
}

# cheap pins first; the finite-difference sweep last
PINS = [pins.test_short_conv_silu_matches_numpy_convolve, pins.test_conv_restarts_at_each_sequence,
        pins.test_single_tap_reduces_to_pointwise, pins.test_signed_gate_closed_forms,
        pins.test_packed_documents_equal_batch_rows, pins.test_packed_ragged_documents_match_numpy_convolve,
        lambda: pins.test_gradients_central_differences(-1.0)]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not found once: " + name
    mod = types.ModuleType("mutated_prologue")
    exec(compile(src.replace(old, new), "mutated_prologue.py", "exec"), mod.__dict__)
    monkeypatch.setattr(oracle, "prologue_fwd", mod.prologue_fwd)
    monkeypatch.setattr(oracle, "prologue_bwd", mod.prologue_bwd)
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, RuntimeError, FloatingPointError):
            return
    pytest.fail("planted mistake %s passed every pin" % name)
