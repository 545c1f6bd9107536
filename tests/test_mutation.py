"""Planted mistakes in the oracle must be caught by its pins.

Each variant is the oracle source compiled with one ``-DORACLE_MUTANT_*``
macro (a swapped nibble order, a dropped min term, ties rounded away from
zero, an off-by-one block sum, a shifted group index, a product that indexes
d and m by 256-wide groups whatever the group size, a dropped block-sum term
in the W4A8 product, a weight scale from the maximum alone instead of the
range, an activation scale of amax/128, a W4A8 product that takes each
block's scale from the next block, and a weight quantiser that stores a -0
group minimum as found instead of +0).  The mistake lives in the oracle on the CPU; no GPU
code is involved.  Every variant must fail at least one pin.
"""
import pytest

import oracle
import oracle_pins

MUTANTS = [
    "SWAP_NIBBLES",
    "DROP_MIN",
    "ROUND_AWAY",
    "BLOCKSUM_OFF_BY_ONE",
    "GROUP_INDEX",
    "GROUP_FIXED_256",
    "MMQ_DROP_BLOCKSUM",
    "RANGE_NO_MIN",
    "SCALE_128",
    "MMQ_NEXT_BLOCK_SCALE",
    "SIGNED_ZERO",
]


@pytest.mark.parametrize("mutant", MUTANTS)
def test_mutant_is_caught(tmp_path, mutant):
    path = oracle.compile_oracle(str(tmp_path / f"liboracle_{mutant}.so"),
                                 defines=(f"ORACLE_MUTANT_{mutant}",), openmp=False)
    o = oracle.Oracle(oracle.load(path))
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(o)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {mutant}"
    if mutant == "GROUP_FIXED_256":
        # the mistake only shows at group 32: the group-32 pins must see it
        assert any(name.startswith("pin_g32_") for name in failed), failed
