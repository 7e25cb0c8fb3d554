"""The CPU oracle against its pins (see tests/pins.py for what pins what)."""
import pytest

import pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(orc, check):
    check(orc)


def test_permuted_rows(orc):
    assert orc.permuted_rows(512, 8, 2) == 1024
    assert orc.permuted_rows(128, 64, 6, C=16, capped=True) == 64 * 16 + 6 * (128 - 16)
    assert orc.permuted_rows(10, 64, 6, C=16, capped=True) == 64 * 16
    assert orc.permuted_rows(10, 4, 2, C=0, capped=True) == 20
