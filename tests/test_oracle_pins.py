"""The oracle against facts outside itself: E4M3 closed forms and a library decoder, a
hand-worked case, brute force with exact rationals, a single-head special case, invariants,
the page's layer pattern and hand-counted overlaps."""

import pytest

from pins import PIN_CHECKS


@pytest.mark.parametrize("check", PIN_CHECKS, ids=[c.__name__ for c in PIN_CHECKS])
def test_pin(check):
    check()
