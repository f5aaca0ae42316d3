"""The committed float64 oracle against its pins (CPU only)."""
import pytest

import oracle
from tests import pins


@pytest.fixture(scope="module")
def o():
    return oracle.default()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(o, pin):
    pin(o)


def test_threads_do_not_change_results(o):
    import numpy as np

    rng = np.random.default_rng(5)
    T, Hq, Hk, D = 64, 4, 2, 16
    stride = (Hq + 2 * Hk) * D
    x = rng.standard_normal((T, stride)).astype(np.float32)
    g = (1 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    a = o.per_head(x, "fp32", T, Hq, Hk, D, stride, g, g, 1e-6, nthreads=1)
    b = o.per_head(x, "fp32", T, Hq, Hk, D, stride, g, g, 1e-6, nthreads=4)
    assert np.array_equal(a, b)
