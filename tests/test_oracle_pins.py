"""The fp64 CPU oracle against what the pages and the mathematics fix
(see tests/oracle_pins.py for each fact and its source)."""
import pytest

import oracle_pins as P


@pytest.mark.parametrize("check", P.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(orc, check):
    check(orc)
