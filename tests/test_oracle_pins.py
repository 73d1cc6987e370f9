"""The float64 oracle against the pins of ``oracle_pins`` (CPU only)."""
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_threads_do_not_change_results(orc):
    """The token loop may run on several threads; the row arithmetic is the same."""
    import numpy as np
    x, g = oracle_pins.bf16_inputs(64, 1024, seed=21)
    y1, r1 = orc.rmsnorm(x, g, 4, 1e-6, "bf16", nthreads=1)
    y8, r8 = orc.rmsnorm(x, g, 4, 1e-6, "bf16", nthreads=8)
    assert np.array_equal(y1, y8) and np.array_equal(r1, r8)
    assert np.array_equal(orc.partial_sumsq(x, 4, "bf16", 1), orc.partial_sumsq(x, 4, "bf16", 8))


def test_rejects_bad_arguments(orc):
    import numpy as np
    x, g = oracle_pins.bf16_inputs(2, 24, seed=1)
    with pytest.raises(ValueError):
        orc.partial_sumsq(x, 5, "bf16")       # D % P != 0
    with pytest.raises(ValueError):
        orc.rmsnorm(x, g, 2, -1.0, "bf16")    # eps < 0
    with pytest.raises(ValueError):
        orc.rmsnorm(x.astype(np.float32), g, 2, 1e-6, "bf16")
