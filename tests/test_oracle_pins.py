"""The fp64 oracle against facts outside itself (closed forms, brute force, library routines)."""
import pytest

import oracle
from tests import pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(oracle)
