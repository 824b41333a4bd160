"""The CPU oracle against closed forms, library routines, brute force and finite differences."""
import pytest

from tests import pins


@pytest.mark.parametrize("check", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(check):
    check()


def test_nystrom_form_is_not_injective_everywhere():
    # The pages' injectivity claim is for the exact whitened map; the Nystrom rows
    # collide on a positive-measure set. The constructed pair must collide exactly
    # (up to rounding) while the queries differ.
    dc, dq = pins.nystrom_collision_example()
    assert dq > 0.3
    assert dc < 1e-15
