"""The fp64 oracle checked against facts that do not come from the oracle itself."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.default())


def test_threads_do_not_change_results():
    import numpy as np
    rng = np.random.default_rng(7)
    p, q, m1, m2, r, N = 4, 4, 4, 4, 2, 33
    S = np.ones((p, q)); A = rng.standard_normal((r, p, q)); B = rng.standard_normal((r, m1, m2))
    x = rng.standard_normal((N, p * m1)); G = rng.standard_normal((N, q * m2))
    orc = oracle.default()
    n0 = orc.get_threads()
    try:
        orc.set_threads(1)
        y1 = orc.forward(x, S, A, B); g1 = orc.backward(x, S, A, B, G)
        orc.set_threads(max(2, n0))
        y2 = orc.forward(x, S, A, B); g2 = orc.backward(x, S, A, B, G)
    finally:
        orc.set_threads(n0)
    assert np.array_equal(y1, y2)
    for k in g1:
        assert np.array_equal(g1[k], g2[k])
