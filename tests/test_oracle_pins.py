"""The CPU oracle against what the pages and the mathematics fix (no GPU)."""

import pytest

import oracle_checks as oc


@pytest.mark.parametrize("check", oc.BLOCK_CHECKS, ids=lambda f: f.__name__)
def test_block_arithmetic_pins(check, golden):
    check(golden)


@pytest.mark.parametrize("check", oc.PLAIN_BLOCK_CHECKS, ids=lambda f: f.__name__)
def test_block_manager_pins(check):
    check()


@pytest.mark.parametrize("check", oc.ATTENTION_CHECKS, ids=lambda f: f.__name__)
def test_attention_pins(check):
    check()
