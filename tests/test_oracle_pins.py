"""The fp64 oracle against its pins (closed forms, invariants, brute force,
finite differences); no GPU needed."""
import pytest

from tests import pins


@pytest.mark.parametrize("name", list(pins.PINS))
def test_pin(name):
    ok, detail = pins.run_pin(name)
    assert ok, detail
