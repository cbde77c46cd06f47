"""The oracle against its pins (CPU only). See tests/pins.py for what pins what."""

import pytest

from tests import pins


@pytest.mark.parametrize("pin", pins.PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()
