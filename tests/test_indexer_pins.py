"""The lightning-indexer oracle against its pins (CPU only)."""

import importlib

import pytest

import indexer_pins

I = importlib.import_module("oracle.indexer")


@pytest.mark.parametrize("pin", indexer_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(I)
