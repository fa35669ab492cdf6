"""The CPU oracle against facts fixed outside it (see tests/pins.py)."""
import pytest

from tests import pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check):
    check()
