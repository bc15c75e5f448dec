"""The fp64 oracle against closed forms, library routines, the brute-force
SSD matrix, an independent chunked form and invariants (CPU only)."""
import pytest

import oracle_checks


@pytest.mark.parametrize("check", oracle_checks.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check()
