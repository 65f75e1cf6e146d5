"""The oracle's fused entry points (raw reference points, offsets and logits)
against their pins: torch autograd of the pages' formulation, softmax
invariants, closed forms and finite differences."""
import pytest

import oracle
import fused_pins


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", fused_pins.ALL_PINS, ids=[p.__name__ for p in fused_pins.ALL_PINS])
def test_fused_pin(orc, pin):
    pin(orc)
