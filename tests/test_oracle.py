"""The fp64 oracle against its pins (CPU only)."""
import pytest

import oracle
import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.default())


def test_row_subset_leaves_other_rows():
    import numpy as np
    import torch
    q, k, v, qg, kg, vg = oracle_pins._six(1, 2, 30, 8, 11)
    out = np.full((1, 2, 30, 8), 123.0)
    oracle.forward(q, k, v, qg, kg, vg, window=4, bh_range=(1, 2), row_range=(5, 9), out=out)
    full = oracle.forward(q, k, v, qg, kg, vg, window=4)
    assert np.all(out[0, 0] == 123.0)
    assert np.all(out[0, 1, :5] == 123.0) and np.all(out[0, 1, 9:] == 123.0)
    assert np.array_equal(out[0, 1, 5:9], full[0, 1, 5:9])


def test_bad_arguments():
    q, k, v, qg, kg, vg = oracle_pins._six(1, 1, 8, 4, 12)
    with pytest.raises(RuntimeError):
        oracle.forward(q, k, v, qg, kg, vg, window=3)          # odd non-causal window
    with pytest.raises(RuntimeError):
        oracle.forward(q, k, v, qg, kg, vg, window=4, dilation=[0])
