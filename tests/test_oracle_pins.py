"""The fp64 oracle against facts the pages and the mathematics fix (CPU only)."""
import pytest

import oracle
from tests import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle.load())


def test_golden_coefficients_are_the_pages():
    assert pins.QUINTIC == (3.4445, -4.7750, 2.0315)
    assert pins.CUBIC == (1.5, -0.5, 0.0)
    assert pins.HYBRID[0] == (3.445, -4.7750, 2.0315) and pins.HYBRID[-1] == (2.0, -1.5, 0.5)
    assert len(pins.HYBRID) == 10


def test_hybrid_schedule_lands_on_one():
    """The eight-plus-two schedule maps every normalised singular value in [1e-3, 1] close to 1
    (scalar map only; the matrix iteration is pinned to it by pin_spectral_map)."""
    import numpy as np
    x = np.geomspace(1e-3, 1.0, 2000)
    y = pins.scalar_map(x, pins.HYBRID)
    assert y.min() > 0.9999 and y.max() < 1.0021, (y.min(), y.max())


def test_thread_count_does_not_change_result():
    import numpy as np
    G = pins.rng(5).standard_normal((37, 61))
    a = oracle.newton_schulz(G, [pins.QUINTIC] * 5, nthreads=1)
    b = oracle.newton_schulz(G, [pins.QUINTIC] * 5, nthreads=7)
    assert np.array_equal(a, b)


def test_rejects_bad_arguments():
    import numpy as np
    with pytest.raises(ValueError):
        oracle.newton_schulz(np.zeros((0, 3)), [pins.QUINTIC])
