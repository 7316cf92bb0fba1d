"""The float64 oracle against its pins (CPU only)."""
import pytest

from oracle import oracle
from oracle_pins import PINS


@pytest.fixture(scope="module")
def ref():
    return oracle.default()


@pytest.mark.parametrize("name", sorted(PINS))
def test_pin(ref, name):
    PINS[name](ref)


def test_rejects_bad_sizes(ref):
    import numpy as np
    u = np.zeros((1, 1, 2))
    with pytest.raises(ValueError):
        ref.selective_scan(u, u, np.zeros((1, 300)), np.zeros((1, 300, 2)), np.zeros((1, 300, 2)))


def test_empty_sequence(ref):
    import numpy as np
    u = np.zeros((2, 3, 0))
    out, last = ref.selective_scan(u, u, -np.ones((3, 4)), np.zeros((2, 4, 0)), np.zeros((2, 4, 0)))
    assert out.shape == (2, 3, 0)
    assert np.array_equal(last, np.zeros((2, 3, 4)))
