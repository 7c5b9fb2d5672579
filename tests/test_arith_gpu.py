"""The library's fast reciprocal and division by qmax (used for the scales on
the hot path) against the IEEE correctly rounded routines, bit for bit, on
every input in their range (qstate_selfcheck, through the C ABI)."""
import pytest

pytestmark = pytest.mark.gpu


def test_fast_arithmetic_matches_ieee_everywhere():
    from ssm_decode_step_b200 import qstate as Q
    assert Q.selfcheck() == [0, 0, 0]
