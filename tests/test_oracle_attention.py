"""Oracle attention + summed weights against brute force, torch SDPA (fp64),
closed forms, invariants and a hand-worked example."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_ATTENTION_PINS, ids=lambda f: f.__name__)
def test_attention_pin(pin):
    pin()
