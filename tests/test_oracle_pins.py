"""The CPU oracle against its pins (closed forms, hand-worked examples, the
quadratic dual form, library routines, brute force, invariants)."""

import pytest

import oracle as O
import oracle_pins as pins


@pytest.fixture(scope="module")
def orc():
    return O.default()


def test_default_build_tag(orc):
    assert orc.tag == "oracle"


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)
