"""The CPU oracle against its pins (exact rationals, brute force, closed forms,
invariants, hand-derived fixtures)."""
import pytest

import oracle.wushkv_oracle as orc
from tests import pins


@pytest.mark.parametrize("check", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(check):
    check(orc)
