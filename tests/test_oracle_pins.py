"""The C oracle against its pins (values fixed by the pages and the math)."""

import pytest

from oracle import ref
from pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(ref.default())
