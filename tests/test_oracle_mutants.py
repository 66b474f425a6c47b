"""Each planted oracle mistake must be caught by at least one pin (CPU only).

The mutants are compile-time variants of the C oracle (PKV_ORACLE_MUTANT):
1 interleaved GQA head map, 2 page/row index swapped, 3 scale dropped,
4 causal edge off by one, 5 newest key dropped in decode, 6 softmax
normaliser dropped, 7 token-major page layout, 8 cache-write slot off by one,
9 scores taken against V, 10 merge weight sign flipped, 11 int8 code range
128 instead of 127, 12 int8 rounding toward zero, 13 int8 V rows scaled by the
K scale, 14 sliding window one key too wide, 15 RoPE pairs adjacent elements,
16 RoPE turns the wrong way, 17 RoPE frequency exponent halved, 18 sign of
the scale dropped.
"""
import pytest

import oracle
import oracle_pins

MUTANTS = list(range(1, 19))


@pytest.mark.parametrize("mutant", MUTANTS)
def test_mutant_is_caught(mutant):
    orc = oracle.Oracle(mutant=mutant)
    assert orc.mutant == mutant
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except Exception:            # AssertionError, or the oracle rejecting its own output
            caught.append(pin.__name__)
    assert caught, f"mutant {mutant} passed every pin"
