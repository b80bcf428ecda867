"""The oracle against its pins (CPU only)."""
import pytest

from tests import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_oracle_golden_fixture(oracle_lib):
    """Regression fixture written by tests/golden/make_golden.py (which calls
    only the oracle): the oracle still produces the stored values."""
    from tests.golden import make_golden
    make_golden.check(oracle_lib)
