"""The fp64 oracle against what the pages and the mathematics fix (CPU only)."""
import pytest

from tests import oracle_pins as pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check, oracle_lib):
    check(oracle_lib)
