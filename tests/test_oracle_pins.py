"""The CPU oracle against its pins (hand-worked examples, library special
cases, brute force, closed forms, invariants).  CPU only."""
import pytest

import oracle
from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle)


def test_near_tie_rule():
    import torch
    row = torch.tensor([1.0, 0.5000001, 0.5, 0.2], dtype=torch.float64)
    b = (0.5000001, 0.5)
    assert P.near_tie_excused(b, row, [0, 2], [0, 1])          # inside the band
    assert not P.near_tie_excused((0.5, 0.5), row, [0, 2], [0, 1])   # exact tie: must match
    assert not P.near_tie_excused((0.6, 0.5), row, [0, 2], [0, 1])   # clear gap
    assert not P.near_tie_excused(None, row, [0, 2], [0, 1])
    assert not P.near_tie_excused(b, row, [0, 3], [0, 1])      # block 3 is far from the boundary
