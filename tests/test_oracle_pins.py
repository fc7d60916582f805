"""The CPU oracle against facts fixed outside it (brute force, closed forms, the pages' examples)."""
import pytest

from tests.pins import PINS


@pytest.mark.parametrize("name", sorted(PINS))
def test_pin(name):
    fn, tol = PINS[name]
    err = fn()
    assert err <= tol, f"{name}: error {err:.3e} above {tol:.1e}"
