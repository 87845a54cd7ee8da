"""The float64 oracle against facts outside itself (see tests/oracle_pins.py),
and a check that each planted mistake in the oracle trips at least one pin."""
import pytest

import oracle
from tests import oracle_pins as P


@pytest.fixture(scope="module")
def o():
    return oracle.get()


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(o, pin):
    pin(o)


# mutant id -> the mistake planted in oracle/q4_0_oracle.c
MUTANTS = {
    1: "nibbles swapped in pack",
    2: "zero point 7 instead of 8",
    3: "sign of (q - 8) flipped",
    4: "last block of each row dropped from the sum",
    5: "fp16 exponent bias off by one",
    6: "output written transposed",
    7: "gather reads the next row",
    8: "quantization scale with the wrong sign",
    9: "quantization takes the last of equal extreme magnitudes",
    10: "quantization truncates instead of rounding",
    11: "silu with the wrong sign in the exponent",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m])
def test_planted_mistake_is_caught(mutant):
    om = oracle.Oracle(mutant)
    failed = []
    for pin in P.ALL_PINS:
        try:
            pin(om)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught mutant {mutant} ({MUTANTS[mutant]})"
