"""Each planted mistake in the oracle fails at least one pin.

The oracle source carries compile-time switches that each plant one plausible
mistake (a flipped conv kernel, a wrong head->group map, a wrong sign of A, a
dropped dt on the input term, y read from the old state, y read with B instead
of C, a dropped D skip, truncating bf16 rounding, a sigmoid gate, no conv
roll, swapped B/C halves, dt without its bias; for the gated RMSNorm: one
group over the whole row, eps outside the square root, no weight). Each
mutant is built on the
CPU into a temporary directory and run against the same pins as the default
build; the test asserts that some pin rejects it.
"""

import os

import pytest

import oracle as O
import oracle_pins as pins

MUTANTS = [
    "M2O_MUTANT_CONV_FLIP",
    "M2O_MUTANT_GROUP_MOD",
    "M2O_MUTANT_A_SIGN",
    "M2O_MUTANT_DROP_DT_INPUT",
    "M2O_MUTANT_Y_OLD_STATE",
    "M2O_MUTANT_Y_USES_B",
    "M2O_MUTANT_DROP_D",
    "M2O_MUTANT_BF16_TRUNC",
    "M2O_MUTANT_GATE_SIGMOID",
    "M2O_MUTANT_NO_ROLL",
    "M2O_MUTANT_SWAP_BC",
    "M2O_MUTANT_DT_NO_BIAS",
    "M2O_MUTANT_NORM_WHOLE_ROW",
    "M2O_MUTANT_NORM_EPS_OUTSIDE",
    "M2O_MUTANT_NORM_NO_WEIGHT",
]


@pytest.mark.parametrize("mutant", MUTANTS)
def test_mutant_is_caught(mutant, tmp_path):
    path = O.build(os.path.join(tmp_path, f"lib_{mutant}.so"), defines=[mutant], force=True)
    orc = O.Oracle(path)
    assert orc.tag.startswith("mutant:")
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"{mutant} passed every pin"
