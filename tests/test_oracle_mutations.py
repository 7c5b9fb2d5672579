"""Plant each listed mistake in the oracle (on the CPU, in the oracle's
mutation build) and require that at least one pin fails: evidence that the
pins can tell a wrong oracle from a right one."""
import pytest

from oracle import oracle as O
from tests import pins

FAULTS = [f for f in O.FAULTS if f != "none"]


@pytest.mark.parametrize("fault", FAULTS)
def test_planted_mistake_is_caught(fault):
    caught = []
    with O.planted(fault):
        for pin in pins.ALL_PINS:
            try:
                pin()
            except AssertionError:
                caught.append(pin.__name__)
    assert O.planted_fault() == "none"
    assert caught, f"no pin catches the planted mistake {fault!r}"


def test_oracle_proper_has_no_mutation_hook():
    """The oracle the tests compare against is the build without planted
    mistakes: it exports no fault setter."""
    lib = O.lib()
    assert not hasattr(lib, "qo_set_fault")
