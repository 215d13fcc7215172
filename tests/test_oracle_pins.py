"""The oracle against closed forms, brute force, textbook special cases and
invariants (CPU only)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda f: f.__name__[6:])
def test_pin(check):
    check()
