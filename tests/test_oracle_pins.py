"""The CPU oracle against closed forms, torch's SDPA, brute force and invariants."""

import os

import pytest

import pins

FIXTURE = os.path.join(os.path.dirname(__file__), "golden", "block_structure_37x37_p4.txt")
PINS = pins.all_pins(FIXTURE)


@pytest.mark.parametrize("name", sorted(PINS))
def test_pin(name):
    PINS[name]()
