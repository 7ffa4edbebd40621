"""The fp64 oracle against its pins (CPU only)."""

import importlib

import pytest

import oracle_pins

O = importlib.import_module("oracle.compressor")


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(O)
