"""The oracle against its pins (CPU only). See pins.py for what each pin fixes."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_ORACLE_PINS + pins.ALL_MODEL_PINS,
                         ids=lambda p: p.__name__)
def test_pin(pin):
    pin()
