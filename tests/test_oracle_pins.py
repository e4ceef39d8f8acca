"""The fp64 oracle against facts fixed outside it (see ``pins.py``,
``pins_ext.py`` and ``pins_grad.py``)."""
import pytest

import oracle
import pins
import pins_ext
import pins_grad
from oracle import backward, cache_ops


@pytest.mark.parametrize("pin", pins.ALL_PINS + pins_ext.EXT_PINS,
                         ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.load())


@pytest.mark.parametrize("pin", pins_grad.GRAD_PINS, ids=lambda f: f.__name__)
def test_grad_pin(pin):
    pin(backward)


@pytest.mark.parametrize("pin", pins_ext.CACHE_PINS, ids=lambda f: f.__name__)
def test_cache_pin(pin):
    pin(cache_ops)
