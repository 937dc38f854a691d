"""The CPU oracle against facts other than itself (no GPU needed)."""
import pytest

import pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(orc, check):
    check(orc)


def test_oracle_reports_threads(orc):
    assert orc.num_threads() >= 1
