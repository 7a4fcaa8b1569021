"""Plant one known mistake at a time in the oracle (on the CPU) and check
that the pins catch it without help from the brute force."""
import pytest

import oracle
from tests import pins

INDEPENDENT = [n for n in pins.PINS if n != "brute_force_tiny"]


@pytest.mark.parametrize("code", sorted(oracle.mutation.NAMES))
def test_mutation_is_caught(code):
    with oracle.mutation(code):
        failed = [n for n in INDEPENDENT if not pins.run_pin(n)[0]]
        brute_ok = pins.run_pin("brute_force_tiny")[0]
    assert failed, "mutation %s went unnoticed by every pin" % oracle.mutation.NAMES[code]
    # the brute force is independent code, so it must see every mutation that
    # the tiny workload can express (V != H there, so not the transposition)
    if oracle.mutation.NAMES[code] != "dh_transposed":
        assert not brute_ok


def test_pins_hold_again_after_mutations():
    assert all(pins.run_pin(n)[0] for n in pins.PINS)
