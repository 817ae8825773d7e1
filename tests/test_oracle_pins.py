"""The fp64 oracle against its pins (closed forms, invariants, library routines,
brute-force dense evaluation). CPU only."""

import pytest

from oracle_checks import ALL_CHECKS


@pytest.mark.parametrize("check", ALL_CHECKS, ids=[c.__name__ for c in ALL_CHECKS])
def test_oracle_pin(oracle_lib, check):
    check(oracle_lib)
