"""The fp64 oracle pinned to things other than itself (no GPU needed)."""
import pytest

import oracle
import oracle_checks as oc


@pytest.mark.parametrize("check", oc.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(orc, check):
    check(orc)


def test_textbook_bf16(orc):
    oc.check_textbook(orc, dtype=oracle.BF16)


def test_append_bf16_bits_untouched(orc):
    oc.check_append(orc, dtype=oracle.BF16)
