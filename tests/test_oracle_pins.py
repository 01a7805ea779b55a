"""The CPU oracle against its pins (binary16 format, packing rule, exact arithmetic,
closed forms, one-hot selection, scale duplication, numpy BLAS, the quantiser's
worked example and properties) and a check that
each planted mistake in the oracle breaks at least one pin."""
import numpy as np
import pytest

import oracle
import pins


@pytest.fixture(scope="module")
def o():
    return oracle.load()


@pytest.mark.parametrize("pin", pins.PINS, ids=lambda f: f.__name__)
def test_pin(o, pin):
    assert pin(o)


def test_exact_whole_tiny_config(o):
    # The whole 4 x 512 x 512 tiny config against the integer brute force.
    assert pins.pin_exact_tiny_config(o)


MUTANTS = {
    1: "nibble order swapped when decoding",
    2: "nibble read as unsigned",
    3: "scale row off by one at group boundaries",
    4: "scales read transposed",
    5: "float32 accumulation",
    6: "result rounded through float32 first",
    7: "truncation instead of round-to-nearest-even",
    8: "last partial group dropped",
    9: "activations read transposed",
    10: "low code not masked when packing",
    11: "tiled layout in natural nibble order",
    12: "last row of each expert segment dropped",
    13: "quantiser scale taken as max/8",
    14: "quantiser rounds halves to even",
    15: "quantiser scale from the whole column",
    16: "8-bit codes read as unsigned",
    17: "8-bit tiled layout with the bytes of a chunk reversed",
    18: "8-bit quantiser scale taken as max/128",
    19: "8-bit quantiser rounds halves to even",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m].replace(" ", "_"))
def test_planted_mistake_is_caught(mutant, tmp_path):
    m = oracle.load_mutant(mutant, str(tmp_path))
    failing = []
    for pin in pins.PINS:
        try:
            ok = pin(m)
        except Exception:
            ok = False
        if not ok:
            failing.append(pin.__name__)
            break
    assert failing, f"mutant {mutant} ({MUTANTS[mutant]}) passes every pin"


def test_oracle_uses_threads(o):
    assert o.threads() >= 1
