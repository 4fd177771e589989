"""The CPU oracle against closed forms, invariants, brute force, torch's fp64
attention and the pages' printed figures (no GPU)."""
import pytest

from oracle import vsa_oracle
from tests import oracle_pins


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(vsa_oracle)
