"""The oracle against its pins (closed forms, identities, hand-worked examples)."""
import pytest

import oracle_pins as P


@pytest.mark.parametrize("name", sorted(P.ALL_PINS))
def test_pin(name):
    fn, tol = P.ALL_PINS[name]
    err = fn()
    assert err <= tol, "%s: error %.3e above %.1e" % (name, err, tol)
