"""The fp64 oracle against what the pages and the mathematics fix (CPU only)."""
import pytest

import oracle.moe_oracle as O
from tests import pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(check):
    check(O)
