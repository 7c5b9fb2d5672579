"""Plant each listed mistake in the oracle (on the CPU) and require that at
least one pin fails: evidence that the pins can tell a wrong oracle from a
right one."""
import pytest

from oracle import oracle as O
from tests import pins

FAULTS = [f for f in O.FAULTS if f != "none"]


@pytest.mark.parametrize("fault", FAULTS)
def test_planted_mistake_is_caught(fault):
    caught = []
    O.set_fault(fault)
    try:
        for pin in pins.ALL_PINS:
            try:
                pin()
            except AssertionError:
                caught.append(pin.__name__)
    finally:
        O.set_fault("none")
    assert caught, f"no pin catches the planted mistake {fault!r}"
