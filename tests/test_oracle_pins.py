"""The oracle against its pins (CPU only)."""
import pytest

from tests.oracle_pins import PINS


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_thread_count_independent(oracle_lib):
    import numpy as np
    from oracle import oracle as O
    r = np.random.default_rng(3)
    q, k, v, do = (r.standard_normal((70, 16)) for _ in range(4))
    base = O.bwd(q, k, v, do, 0.25, True, nthreads=1, lib=oracle_lib)
    for t in (2, 7, 16):
        other = O.bwd(q, k, v, do, 0.25, True, nthreads=t, lib=oracle_lib)
        for a, b in zip(base, other):
            assert np.array_equal(a, b)
