"""The fp64 oracle against its pins (library routines, closed forms, invariants, brute force)."""
import pytest

from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    ok, detail = pin()
    assert ok, detail


def test_bf16_output_rounding_alone_exceeds_literal_max_abs_bound():
    """Why the bf16 max-abs bound is applied beyond the output's own rounding: rounding an exact
    result with a few rows far above the RMS to bf16 already breaks 2e-2 * RMS, while the
    roundoff-discounted measure is zero for it."""
    import numpy as np
    import torch
    from tests.parity import BF16_UNIT_ROUNDOFF, output_errors
    r = np.random.default_rng(0)
    o = r.standard_normal((512, 64)) * 0.05
    o[7] = r.standard_normal(64) * 1.0          # one concentrated-attention row, ~20x the RMS
    ob = torch.from_numpy(o).to(torch.bfloat16).double().numpy()
    _, literal = output_errors(ob, o)
    _, discounted = output_errors(ob, o, output_roundoff=BF16_UNIT_ROUNDOFF)
    assert literal > 2e-2 and discounted == 0.0
